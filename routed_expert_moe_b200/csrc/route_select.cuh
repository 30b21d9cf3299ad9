// Token selection shared by the router kernels (route.cu, route_tc.cu): the
// exact fixed-point logit, the certified ranking of approximate logits, the
// exact ranking of the candidates the bound leaves open, and the renormalised
// routing weights.
//
// The method (bloomery issue page, s.2 "Checkpoint facts": top-6 routing over
// 128 experts; audio.cpp model page, "CPU weight offload": the router and the
// routing-weight formulas): keep the K largest logits (ties to the lower
// expert index), weights = softmax over the kept logits.  Ranking is defined
// on logits summed in fixed point (every bf16 x bf16 product, exact in fp32,
// rounded to the grid 2^-40 and summed exactly in int64).
#pragma once
#include <cstdint>
#include <climits>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {

// warp arg-max of (value, -index)
__device__ __forceinline__ void warp_argmax_i64(long long& v, int& e) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const long long ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oe = __shfl_xor_sync(0xffffffffu, e, off);
        if (ov > v || (ov == v && oe < e)) {
            v = ov;
            e = oe;
        }
    }
}

// Exact fixed-point logit (units of 2^-40) of expert e for token row xr:
// every bf16 product (exact in fp32) scaled by 2^40 and rounded to the
// nearest integer, summed exactly; one warp, 16-byte loads issued eight
// fragments per lane at a time so that their latencies overlap.
static __device__ long long exact_logit(const uint16_t* xr, const uint16_t* wrow, int H, const float* bias, int e,
                                 int lane) {
    constexpr int B = 8;
    const uint4* xv = reinterpret_cast<const uint4*>(xr);
    const uint4* wv = reinterpret_cast<const uint4*>(wrow);
    const int nv = H / 8;
    long long acc = 0;
    for (int v0 = lane; v0 < nv; v0 += 32 * B) {
        uint4 a[B], b[B];
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const int v = v0 + 32 * i;
            a[i] = b[i] = make_uint4(0, 0, 0, 0);
            if (v < nv) {
                a[i] = xv[v];
                b[i] = wv[v];
            }
        }
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const uint32_t aa[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
            const uint32_t bb[4] = {b[i].x, b[i].y, b[i].z, b[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float p0 = __fmul_rn(__uint_as_float(aa[j] << 16), __uint_as_float(bb[j] << 16));
                const float p1 =
                    __fmul_rn(__uint_as_float(aa[j] & 0xFFFF0000u), __uint_as_float(bb[j] & 0xFFFF0000u));
                acc += __float2ll_rn(__fmul_rn(p0, 0x1p40f));
                acc += __float2ll_rn(__fmul_rn(p1, 0x1p40f));
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (bias) acc += __float2ll_rn(__fmul_rn(bias[e], 0x1p40f));
    return acc;
}

constexpr int TK_MAXK = 16;       // K <= 16

// Relative bound of an approximate logit l~ (in units of ||x|| ||w_e||, which
// bounds sum_h |x_h w_eh| by Cauchy-Schwarz) for a summation whose fp32 part
// rounds at most n32 times along any product's path (g_n32, u = 2^-24) and
// whose fp64 part adds at most d64 times (d64 2^-52 >= g_d64 at u = 2^-53);
// 2^-40 is slack for the roundings of the bound's own arithmetic.
__host__ __device__ inline double router_k_rel(int n32, int d64) {
    const double g = (double)n32 * 0x1p-24;
    return g / (1.0 - g) + (double)d64 * 0x1p-52 + 0x1p-40;
}

// Order-preserving integer key of a double (unsigned order = numeric order;
// -0 is mapped with +0 by adding 0.0 first).
__device__ __forceinline__ unsigned long long order_key(double v) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(v + 0.0);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Per-block constants of the bound: the largest ||w_e|| (from the fp32 squared
// norms Q, inflated by 1 + (H+64) 2^-23 to an upper bound) and the largest
// |b_e|.  One warp; every lane returns both.
__device__ __forceinline__ void bound_constants(const double* Q, const float* bias, int H, int E, int lane,
                                                double& wnmax, double& bmax) {
    double q = 0.0, b = 0.0;
    for (int e = lane; e < E; e += 32) {
        q = fmax(q, Q[e]);
        if (bias) b = fmax(b, fabs((double)bias[e]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        q = fmax(q, __shfl_xor_sync(0xffffffffu, q, off));
        b = fmax(b, __shfl_xor_sync(0xffffffffu, b, off));
    }
    wnmax = sqrt(q * (1.0 + (double)(H + 64) * 0x1p-23));
    bmax = b;
}

// Ranks one token's approximate logits l~ (one warp, E <= 256): the K best
// (ties to the lower index) into out_e/out_l (shared memory of this token,
// written by lane 0), and whether every gap among the K+1 best exceeds
// 2 eps*, where eps* bounds every |(l~_e + b_e) - l_e| against the exact
// fixed-point logit l_e.  When it does not, the token's candidates (every
// expert whose exact logit could still be in the top K) are appended to the
// block's list under `slot`.  The ranking compares order-preserving integer
// keys of l~ + b.
template <int NJ>
__device__ __forceinline__ bool rank_packed(const double* Lrow, double eps_star, const float* bias, int E, int K,
                                            int lane, int slot, int* out_e, double* out_l, uint8_t* c_tok,
                                            uint16_t* c_e, int* n_cand) {
    auto lval = [&](int e) {
        double l = Lrow[e];
        if (bias) l += (double)bias[e];
        return l;
    };
    // Packed keys: the order key of l~ + b with its low 8 bits replaced by 255 - e.  One 64-bit
    // maximum then ranks by value and breaks ties toward the lower index; two values whose keys
    // differ only in those 8 bits are within 2^-44 of each other relatively, and the bound below
    // is widened by 2^-43 max |l~ + b| so that such a pair is never certified.  The exact values
    // are read back for the gaps and the weights.  Empty slots: key 0, below every real key.
    unsigned long long pk[NJ];
    double amax = 0.0;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        pk[j] = 0ull;
        if (e < E) {
            const double l = lval(e);
            amax = fmax(amax, fabs(l));
            pk[j] = (order_key(l) & ~0xFFull) | (unsigned long long)(255 - e);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const double eps = eps_star + amax * 0x1p-43;
    auto cx = [&](int i, int j) {   // (i, j) in descending order after the exchange
        const unsigned long long a = pk[i], b = pk[j];
        pk[i] = a > b ? a : b;
        pk[j] = a > b ? b : a;
    };
    if constexpr (NJ == 4) {
        cx(0, 1); cx(2, 3); cx(0, 2); cx(1, 3); cx(1, 2);
    } else {
        // Batcher's odd-even merge sort of 8
        cx(0, 1); cx(2, 3); cx(4, 5); cx(6, 7);
        cx(0, 2); cx(1, 3); cx(4, 6); cx(5, 7);
        cx(1, 2); cx(5, 6);
        cx(0, 4); cx(1, 5); cx(2, 6); cx(3, 7);
        cx(2, 4); cx(3, 5);
        cx(1, 2); cx(3, 4); cx(5, 6);
    }

    // the K+1 best (ties to the lower index): the best of the lanes' heads, popped
    const int nsel = min(K + 1, E);
    double prev = 0.0, lk = 0.0;
    bool certified = true;
    for (int k = 0; k < nsel; ++k) {
        unsigned long long b = pk[0];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, b, off);
            b = o > b ? o : b;
        }
        const int be = 255 - (int)(b & 0xFFull);
        const double bv = lval(be);
        if (k < K) {
            if (lane == 0) {
                out_e[k] = be;
                out_l[k] = bv;
            }
            lk = bv;
        }
        if (k > 0 && !(prev - bv > 2.0 * eps)) certified = false;
        prev = bv;
        if (pk[0] == b) {   // the lane that held it (keys are unique)
#pragma unroll
            for (int j = 0; j + 1 < NJ; ++j) pk[j] = pk[j + 1];
            pk[NJ - 1] = 0ull;
        }
    }
    if (!certified) {
        // candidates: every expert that could still be in the exact top K
        const unsigned long long thr = order_key(lk - 2.0 * eps);
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int e = lane + 32 * j;
            const bool c = e < E && order_key(lval(e)) >= thr;
            const uint32_t m = __ballot_sync(0xffffffffu, c);
            int base = 0;
            if (lane == 0 && m) base = atomicAdd(n_cand, __popc(m));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (c) {
                const int i = base + __popc(m & ((1u << lane) - 1u));
                c_tok[i] = (uint8_t)slot;
                c_e[i] = (uint16_t)e;
            }
        }
    }
    __syncwarp();
    return certified;
}

__device__ __forceinline__ bool rank_certified_eps(const double* Lrow, double eps_star, const float* bias, int E,
                                                   int K, int lane, int slot, int* out_e, double* out_l,
                                                   uint8_t* c_tok, uint16_t* c_e, int* n_cand) {
    return E <= 128 ? rank_packed<4>(Lrow, eps_star, bias, E, K, lane, slot, out_e, out_l, c_tok, c_e, n_cand)
                    : rank_packed<8>(Lrow, eps_star, bias, E, K, lane, slot, out_e, out_l, c_tok, c_e, n_cand);
}

// rank_certified_eps with the bound of the fp32-chain logits: k_rel bounds
// |l~ - l| / (||x|| ||w_e||) for the caller's summation (see router_k_rel) and
//   eps* = k_rel ||x|| max_e ||w_e|| + (H+1) 2^-41 + (2 ||x|| max_e ||w_e|| + max_e |b_e| + 1) 2^-50
// bounds every |l~_e - l_e| (the last term covers the fp64 roundings of l~ + b).
__device__ __forceinline__ bool rank_certified(const double* Lrow, double xsq, const float* bias, int H, int E,
                                               int K, double k_rel, double wnmax, double bmax, int lane, int slot,
                                               int* out_e, double* out_l, bool& range_bad, uint8_t* c_tok,
                                               uint16_t* c_e, int* n_cand) {
    const double xnorm = sqrt(xsq * (1.0 + (double)(H + 64) * 0x1p-23));   // fp32 norm sum -> upper bound
    const double xw = xnorm * wnmax;
    if (xw >= 0x1p22 || bmax >= 0x1p21) range_bad = true;
    const double eps_star = k_rel * xw + (double)(H + 1) * 0x1p-41 + (2.0 * xw + bmax + 1.0) * 0x1p-50;
    return rank_certified_eps(Lrow, eps_star, bias, E, K, lane, slot, out_e, out_l, c_tok, c_e, n_cand);
}

// Exact fixed-point logits of the block's listed candidates, one warp each;
// token slot s of the list is token t_base + s.
__device__ __forceinline__ void exact_candidates(int nc, const uint8_t* c_tok, const uint16_t* c_e,
                                                 long long* c_val, int64_t t_base, const uint16_t* x,
                                                 const uint16_t* wr, int H, const float* bias, int warp,
                                                 int n_warps, int lane) {
    for (int i = warp; i < nc; i += n_warps) {
        const int e = c_e[i];
        const long long v = exact_logit(x + (t_base + c_tok[i]) * H, wr + (int64_t)e * H, H, bias, e, lane);
        if (lane == 0) c_val[i] = v;
    }
}

// Finishes one token (one warp): if its order was not certified, ranks its
// candidates by exact logit (ties to the lower index) into out_e/out_l; then
// the renormalised softmax over the K kept logits (w_k = exp(l_k - l_0) / z,
// z summed in order k = 0..K-1), and the K (index, weight) pairs of row t.
__device__ __forceinline__ void finish_token(bool certified, int slot, int64_t t, int nc, uint8_t* c_tok,
                                             const uint16_t* c_e, const long long* c_val, int K, int* out_e,
                                             double* out_l, int lane, int32_t* idx, float* w) {
    if (!certified) {
        for (int k = 0; k < K; ++k) {
            long long bv = LLONG_MIN;
            int be = 0x7fffffff, bi = -1;
            for (int i = lane; i < nc; i += 32) {
                if (c_tok[i] != slot) continue;   // other tokens, or already taken (0xFF)
                const long long v = c_val[i];
                const int e = c_e[i];
                if (bi < 0 || v > bv || (v == bv && e < be)) {
                    bv = v;
                    be = e;
                    bi = i;
                }
            }
            int src_e = be;
            warp_argmax_i64(bv, src_e);
            if (bi >= 0 && be == src_e) c_tok[bi] = 0xFF;   // taken (this lane held it)
            if (lane == 0) {
                out_e[k] = src_e;
                out_l[k] = (double)bv * 0x1p-40;
            }
            __syncwarp();
        }
    }
    // lane k < K holds term k
    const double l0 = out_l[0];
    const float ex = lane < K ? expf((float)(out_l[lane < K ? lane : 0] - l0)) : 0.0f;
    float z = 0.0f;
    for (int k = 0; k < K; ++k) z += __shfl_sync(0xffffffffu, ex, k);
    if (lane < K) {
        idx[t * K + lane] = out_e[lane];
        w[t * K + lane] = ex / z;
    }
}

}  // namespace moe
