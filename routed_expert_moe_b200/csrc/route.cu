// Router: logits, top-K with exact ranking, renormalised softmax weights.
//
// The method (bloomery issue page, s.2 "Checkpoint facts": top-6 routing over
// 128 experts; audio.cpp model page, "CPU weight offload": the router and the
// routing-weight formulas) is: l = x Wr^T (+ b), keep the K largest logits
// (ties to the lower expert index), weights = softmax over the kept logits.
//
// Ranking is defined on logits summed in fixed point (every bf16 x bf16
// product, exact in fp32, rounded to the grid 2^-40 and summed exactly in
// int64), which makes the order independent of summation order.  The kernels
// never need that sum for most tokens:
//   1. router_logits_kernel computes l~ in fp32 over chunks of RT_HC = 16
//      terms, chunk sums accumulated in fp64, plus the squared norms of x and Wr.
//      |l~ - l_fx| <= eps_e = (g_RT_HC + 2^-45) ||x|| ||w_e|| + (H+1) 2^-41
//      (the squared norms are fp32 sums of exact squares, at most H terms per
//      value, so they are inflated by 1 + (H+64) 2^-23 to stay upper bounds)
//      (Cauchy-Schwarz bounds sum|x_h w_eh|; g_n = n u / (1 - n u), u = 2^-24).
//   2. router_topk_kernel (one warp per token) ranks l~; if every gap among
//      the K+1 best exceeds 2 eps* (eps* = max_e eps_e) the order is certified.
//      Otherwise it recomputes l_fx exactly for the candidates
//      {e : l~_e >= l~_(K) - 2 eps*} (no other expert can reach the top K)
//      and ranks those; the candidates of a block's 8 tokens are computed by
//      all its warps together.
// Both kernels use only CUDA cores: the contraction is 2.8 GFLOP at 4096
// tokens, and a tensor-core accumulation has no error bound to certify.
#include <cstdint>
#include <cfloat>
#include <climits>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {

constexpr int RT_TE = 128;      // experts per block tile
constexpr int RT_HC = 16;       // terms per fp32 partial sum
constexpr int RT_THREADS = 256;

struct RouterLogitsArgs {
    const uint16_t* x;    // [T][H] bf16
    const uint16_t* wr;   // [E][H] bf16
    int64_t T;
    int H, E, S, nchunks;
    double* P;            // [S][T][E] partial logits
    double* xn2;          // [S][T]  partial ||x||^2
    double* wn2;          // [S][E]  partial ||w_e||^2
};

// One block: 16*TPT tokens x 128 experts over one split of the hidden
// dimension.  Thread (tg, eg) owns tokens TPT*tg .. +TPT-1 x experts
// 8eg..8eg+7.  Each 16-term chunk is a chain of fp32 FMAs from zero (the
// products are exact), added into an fp64 total; smem tiles are
// double-buffered.  TPT = 4 for large batches (64-token tiles), 1 for small
// ones so that a decode batch still spreads over the whole GPU.
template <int TPT>
__global__ void __launch_bounds__(RT_THREADS) router_logits_kernel(RouterLogitsArgs a) {
    constexpr int RT_TT = 16 * TPT;
    __shared__ __align__(16) float xs[2][RT_HC][RT_TT];
    __shared__ __align__(16) float ws[2][RT_HC][RT_TE];

    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * RT_TT;
    const int e0 = blockIdx.y * RT_TE;
    const int s = blockIdx.z;
    const int c_begin = (int)((int64_t)s * a.nchunks / a.S);
    const int c_end = (int)((int64_t)(s + 1) * a.nchunks / a.S);

    const int tg = tid / 16;    // tokens TPT*tg .. TPT*tg+TPT-1
    const int eg = tid % 16;    // experts 4eg..4eg+3 and 64+4eg..64+4eg+3 (16-byte smem reads, no stride)
    const int l_row = tid / 2, l_half = tid % 2;   // staging: row tid/2, 8 terms at 8*(tid%2)

    double acc[TPT * 8];
#pragma unroll
    for (int i = 0; i < TPT * 8; ++i) acc[i] = 0.0;
    float xsq = 0.0f, wsq = 0.0f;  // squared norms of this thread's staged row halves (fp32; see below)

    auto load = [&](int c, uint4& xv, uint4& wv) {
        const int h = c * RT_HC + l_half * 8;
        xv = make_uint4(0, 0, 0, 0);
        wv = make_uint4(0, 0, 0, 0);
        const int64_t t = t0 + l_row;
        if (tid < 2 * RT_TT && t < a.T && h < a.H) xv = *reinterpret_cast<const uint4*>(a.x + t * a.H + h);
        const int e = e0 + l_row;
        if (e < a.E && h < a.H) wv = *reinterpret_cast<const uint4*>(a.wr + (int64_t)e * a.H + h);
    };
    auto store = [&](int buf, const uint4& xv, const uint4& wv) {
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
        if (tid < 2 * RT_TT) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float lo = __uint_as_float(xw[q] << 16), hi = __uint_as_float(xw[q] & 0xFFFF0000u);
                xs[buf][l_half * 8 + 2 * q][l_row] = lo;
                xs[buf][l_half * 8 + 2 * q + 1][l_row] = hi;
                xsq = __fmaf_rn(hi, hi, __fmaf_rn(lo, lo, xsq));
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = __uint_as_float(ww[q] << 16), hi = __uint_as_float(ww[q] & 0xFFFF0000u);
            ws[buf][l_half * 8 + 2 * q][l_row] = lo;
            ws[buf][l_half * 8 + 2 * q + 1][l_row] = hi;
            wsq = __fmaf_rn(hi, hi, __fmaf_rn(lo, lo, wsq));
        }
    };

    uint4 xv, wv;
    if (c_begin < c_end) {
        load(c_begin, xv, wv);
        store(0, xv, wv);
    }
    __syncthreads();
    for (int c = c_begin; c < c_end; ++c) {
        const int buf = (c - c_begin) & 1;
        if (c + 1 < c_end) load(c + 1, xv, wv);
        float p[TPT * 8];
#pragma unroll
        for (int i = 0; i < TPT * 8; ++i) p[i] = 0.0f;
#pragma unroll
        for (int h = 0; h < RT_HC; ++h) {
            float xr[TPT];
            if constexpr (TPT == 4) {
                const float4 xx = *reinterpret_cast<const float4*>(&xs[buf][h][4 * tg]);
                xr[0] = xx.x;
                xr[1] = xx.y;
                xr[2] = xx.z;
                xr[3] = xx.w;
            } else {
                xr[0] = xs[buf][h][tg];
            }
            const float4 wa = *reinterpret_cast<const float4*>(&ws[buf][h][4 * eg]);
            const float4 wb = *reinterpret_cast<const float4*>(&ws[buf][h][64 + 4 * eg]);
            const float wr8[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int i = 0; i < TPT; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) p[i * 8 + j] = __fmaf_rn(xr[i], wr8[j], p[i * 8 + j]);
        }
#pragma unroll
        for (int i = 0; i < TPT * 8; ++i) acc[i] += (double)p[i];
        if (c + 1 < c_end) store(buf ^ 1, xv, wv);
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int64_t t = t0 + TPT * tg + i;
        if (t >= a.T) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = e0 + (j < 4 ? 4 * eg + j : 64 + 4 * eg + j - 4);
            if (e < a.E) a.P[((int64_t)s * a.T + t) * a.E + e] = acc[i * 8 + j];
        }
    }

    // squared norms of this split's range: the two halves of a row sit in adjacent lanes
    xsq = __fadd_rn(xsq, __shfl_xor_sync(0xffffffffu, xsq, 1));
    wsq = __fadd_rn(wsq, __shfl_xor_sync(0xffffffffu, wsq, 1));
    if (l_half == 0) {
        const int64_t t = t0 + l_row;
        if (blockIdx.y == 0 && tid < 2 * RT_TT && t < a.T) a.xn2[(int64_t)s * a.T + t] = (double)xsq;
        const int e = e0 + l_row;
        if (blockIdx.x == 0 && e < a.E) a.wn2[(int64_t)s * a.E + e] = (double)wsq;
    }
}

struct RouterTopkArgs {
    const double* P;
    const double* xn2;
    const double* wn2;
    const uint16_t* x;
    const uint16_t* wr;
    const float* bias;    // [E] or null
    int64_t T;
    int H, E, K, S;
    int32_t* idx;         // [T][K]
    float* w;             // [T][K]
};

constexpr int TK_MAXJ = 8;        // experts per lane (E <= 256)
constexpr int TK_WARPS = 8;       // tokens per block
constexpr int TK_CAP = TK_WARPS * 256;

// warp arg-max of (value, -index)
__device__ __forceinline__ void warp_argmax(double& v, int& e) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oe = __shfl_xor_sync(0xffffffffu, e, off);
        if (ov > v || (ov == v && oe < e)) {
            v = ov;
            e = oe;
        }
    }
}

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
// nearest integer, summed exactly; 16-byte loads, one warp.
__device__ long long exact_logit(const uint16_t* xr, const uint16_t* wrow, int H, const float* bias, int e,
                                 int lane) {
    const uint4* xv = reinterpret_cast<const uint4*>(xr);
    const uint4* wv = reinterpret_cast<const uint4*>(wrow);
    long long acc = 0;
    for (int v = lane; v < H / 8; v += 32) {
        const uint4 a = xv[v], b = wv[v];
        const uint32_t aa[4] = {a.x, a.y, a.z, a.w};
        const uint32_t bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float p0 = __fmul_rn(__uint_as_float(aa[j] << 16), __uint_as_float(bb[j] << 16));
            const float p1 = __fmul_rn(__uint_as_float(aa[j] & 0xFFFF0000u), __uint_as_float(bb[j] & 0xFFFF0000u));
            acc += __float2ll_rn(__fmul_rn(p0, 0x1p40f));
            acc += __float2ll_rn(__fmul_rn(p1, 0x1p40f));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (bias) acc += __float2ll_rn(__fmul_rn(bias[e], 0x1p40f));
    return acc;
}

// One warp per token ranks l~; tokens whose order the bound leaves open put
// their candidates in a block-wide list whose exact logits all 8 warps
// compute together, then finish their selection from it.
__global__ void __launch_bounds__(TK_WARPS * 32, 2) router_topk_kernel(RouterTopkArgs a, DevCtx ctx) {
    __shared__ uint8_t c_tok[TK_CAP];
    __shared__ uint16_t c_e[TK_CAP];
    __shared__ long long c_val[TK_CAP];
    __shared__ double Ls[TK_WARPS][256];   // sum over splits of the partial logits
    __shared__ double Qs[256];             // sum over splits of ||w_e||^2
    __shared__ double Xs[TK_WARPS];        // sum over splits of ||x||^2
    __shared__ int n_cand;

    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    const int64_t t_base = (int64_t)blockIdx.x * TK_WARPS;
    const int64_t t = t_base + warp;
    const bool active = t < a.T;
    if (threadIdx.x == 0) n_cand = 0;
    // the block's (token, expert) partial sums: consecutive threads take
    // consecutive experts, and every load is independent of the others
    {
        const int n_tok = (int)min((int64_t)TK_WARPS, a.T - t_base);
        const int pairs = n_tok * a.E;
        const int64_t stride = a.T * a.E;
        for (int i0 = threadIdx.x; i0 < pairs; i0 += 4 * TK_WARPS * 32) {
            // four pairs per thread, their loads for every split issued together
            int64_t off[4];
            bool ok[4];
            double acc[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = i0 + k * TK_WARPS * 32;
                ok[k] = i < pairs;
                const int w = ok[k] ? i / a.E : 0, e = ok[k] ? i % a.E : 0;
                off[k] = (t_base + w) * a.E + e;
                acc[k] = 0.0;
            }
#pragma unroll 8
            for (int s = 0; s < a.S; ++s) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (ok[k]) acc[k] += a.P[(int64_t)s * stride + off[k]];
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = i0 + k * TK_WARPS * 32;
                if (ok[k]) Ls[i / a.E][i % a.E] = acc[k];
            }
        }
        for (int e = threadIdx.x; e < a.E; e += TK_WARPS * 32) {
            double q = 0.0;
            for (int s = 0; s < a.S; ++s) q += a.wn2[(int64_t)s * a.E + e];
            Qs[e] = q;
        }
        if (threadIdx.x < n_tok) {
            double q = 0.0;
            for (int s = 0; s < a.S; ++s) q += a.xn2[(int64_t)s * a.T + t_base + threadIdx.x];
            Xs[threadIdx.x] = q;
        }
    }
    __syncthreads();

    const int nj = (a.E + 31) / 32;
    // g_16 + 2^-45 (fp64 sums of the chunk and split partials), with slack for the norm sums
    const double kRel = (16.0 * 0x1p-24) / (1.0 - 16.0 * 0x1p-24) + 0x1p-45 + 0x1p-40;
    const double kFx = (double)(a.H + 1) * 0x1p-41;

    double L[TK_MAXJ];
    bool certified = true;
    bool range_bad = false;
    int out_e[16];
    double out_l[16];
    if (active) {
        const double kNorm = 1.0 + (double)(a.H + 64) * 0x1p-23;   // fp32 norm sums -> upper bounds
        const double xnorm = sqrt(Xs[warp] * kNorm);
        double eps_star = 0.0;
#pragma unroll
        for (int j = 0; j < TK_MAXJ; ++j) {
            L[j] = -DBL_MAX;
            const int e = lane + 32 * j;
            if (j < nj && e < a.E) {
                double l = Ls[warp][e];
                if (a.bias) {
                    const double b = (double)a.bias[e];
                    if (fabs(b) >= 0x1p21) range_bad = true;
                    l += b;
                }
                const double wnorm = sqrt(Qs[e] * kNorm);
                if (xnorm * wnorm >= 0x1p22) range_bad = true;
                eps_star = fmax(eps_star, kRel * xnorm * wnorm + kFx + fabs(l) * 0x1p-50);
                L[j] = l;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            eps_star = fmax(eps_star, __shfl_xor_sync(0xffffffffu, eps_star, off));

        // the K+1 best by l~ (ties to the lower index)
        const int nsel = min(a.K + 1, a.E);
        uint32_t taken = 0;
        double prev = 0.0;
        for (int k = 0; k < nsel; ++k) {
            double bv = -DBL_MAX;
            int be = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < TK_MAXJ; ++j) {
                const int e = lane + 32 * j;
                if (j < nj && e < a.E && !((taken >> j) & 1u)) {
                    if (L[j] > bv || (L[j] == bv && e < be)) {
                        bv = L[j];
                        be = e;
                    }
                }
            }
            warp_argmax(bv, be);
            if (k < a.K) {
                out_e[k] = be;
                out_l[k] = bv;
            }
            if (k > 0 && !(prev - bv > 2.0 * eps_star)) certified = false;
            prev = bv;
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
        }
        if (!certified) {
            // candidates: every expert that could still be in the exact top K
            const double thr = out_l[a.K - 1] - 2.0 * eps_star;
#pragma unroll
            for (int j = 0; j < TK_MAXJ; ++j) {
                const int e = lane + 32 * j;
                const bool c = j < nj && e < a.E && L[j] >= thr;
                const uint32_t m = __ballot_sync(0xffffffffu, c);
                int base = 0;
                if (lane == 0 && m) base = atomicAdd(&n_cand, __popc(m));
                base = __shfl_sync(0xffffffffu, base, 0);
                if (c) {
                    const int i = base + __popc(m & ((1u << lane) - 1u));
                    c_tok[i] = (uint8_t)warp;
                    c_e[i] = (uint16_t)e;
                }
            }
        }
    }
    __syncthreads();
    const int nc = n_cand;
    for (int i = warp; i < nc; i += TK_WARPS) {
        const int64_t tt = (int64_t)blockIdx.x * TK_WARPS + c_tok[i];
        const int e = c_e[i];
        const long long v = exact_logit(a.x + tt * a.H, a.wr + (int64_t)e * a.H, a.H, a.bias, e, lane);
        if (lane == 0) c_val[i] = v;
    }
    __syncthreads();

    if (!active) return;
    if (!certified) {
        for (int k = 0; k < a.K; ++k) {
            long long bv = LLONG_MIN;
            int be = 0x7fffffff, bi = -1;
            for (int i = lane; i < nc; i += 32) {
                if (c_tok[i] != warp) continue;   // other tokens, or already taken (0xFF)
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
            __syncwarp();
            out_e[k] = src_e;
            out_l[k] = (double)bv * 0x1p-40;
        }
    }
    if (__any_sync(0xffffffffu, range_bad) && lane == 0) record_error(ctx.err, MOE_ERANGE);

    // renormalised softmax over the selected logits
    float z = 0.0f;
    float ex[16];
    for (int k = 0; k < a.K; ++k) {
        ex[k] = expf((float)(out_l[k] - out_l[0]));
        z += ex[k];
    }
    for (int k = lane; k < a.K; k += 32) {
        int ek = 0;
        float wk = 0.0f;
        for (int q = 0; q < a.K; ++q)
            if (q == k) {
                ek = out_e[q];
                wk = ex[q] / z;
            }
        a.idx[t * a.K + k] = ek;
        a.w[t * a.K + k] = wk;
    }
}

// ----------------------------------------------------------------------------- host

struct RouterPlan {
    int S;
    int nchunks;
    size_t p_bytes, xn_bytes, wn_bytes;
};

static int router_tt(int64_t T) { return T > 256 ? 64 : 16; }

RouterPlan router_plan(int64_t T, int H, int E, int num_sms) {
    RouterPlan p;
    p.nchunks = (H + RT_HC - 1) / RT_HC;
    const int tt = router_tt(T);
    const int64_t tiles = ((T + tt - 1) / tt) * ((E + RT_TE - 1) / RT_TE);
    // about one wave of blocks; at least 4 chunks per split, at most 32 splits
    int64_t want = tiles > 0 ? ((int64_t)num_sms + tiles - 1) / tiles : 1;
    if (tiles * want > (int64_t)num_sms && want > 1) want -= 1;
    int64_t cap = p.nchunks / 4 > 0 ? p.nchunks / 4 : 1;
    if (cap > 32) cap = 32;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    p.S = (int)want;
    p.p_bytes = (size_t)p.S * (size_t)T * (size_t)E * sizeof(double);
    p.xn_bytes = (size_t)p.S * (size_t)T * sizeof(double);
    p.wn_bytes = (size_t)p.S * (size_t)E * sizeof(double);
    return p;
}

cudaError_t launch_route(const uint16_t* x, const uint16_t* wr, const float* bias, int64_t T, int H,
                         int E, int K, int32_t* idx, float* w, double* P, double* xn2, double* wn2,
                         const RouterPlan& plan, const DevCtx& ctx, cudaStream_t stream,
                         void (*between)(cudaStream_t)) {
    if (T == 0) return cudaSuccess;
    RouterLogitsArgs la{x, wr, T, H, E, plan.S, plan.nchunks, P, xn2, wn2};
    const int tt = router_tt(T);
    dim3 grid((unsigned)((T + tt - 1) / tt), (unsigned)((E + RT_TE - 1) / RT_TE), (unsigned)plan.S);
    if (tt == 64)
        router_logits_kernel<4><<<grid, RT_THREADS, 0, stream>>>(la);
    else
        router_logits_kernel<1><<<grid, RT_THREADS, 0, stream>>>(la);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (between) between(stream);
    RouterTopkArgs ta{P, xn2, wn2, x, wr, bias, T, H, E, K, plan.S, idx, w};
    const unsigned blocks = (unsigned)((T + TK_WARPS - 1) / TK_WARPS);
    router_topk_kernel<<<blocks, TK_WARPS * 32, 0, stream>>>(ta, ctx);
    return cudaGetLastError();
}

}  // namespace moe
