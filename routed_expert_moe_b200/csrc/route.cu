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
//   1. router_logits_kernel computes l~ in fp32 over chunks of RT_HC terms,
//      chunk sums accumulated in fp64, plus the squared norms of x and Wr.
//      |l~ - l_fx| <= eps_e = (g_RT_HC + 2^-45) ||x|| ||w_e|| + (H+1) 2^-41
//      (Cauchy-Schwarz bounds sum|x_h w_eh|; g_n = n u / (1 - n u), u = 2^-24).
//   2. router_topk_kernel (one warp per token) ranks l~; if every gap among
//      the K+1 best exceeds 2 eps* (eps* = max_e eps_e) the order is certified.
//      Otherwise it recomputes l_fx exactly for the candidates
//      {e : l~_e >= l~_(K) - 2 eps*} (no other expert can reach the top K)
//      and ranks those.
// Both kernels use only CUDA cores: the contraction is 2.8 GFLOP at 4096
// tokens, and a tensor-core accumulation has no error bound to certify.
#include <cstdint>
#include <cfloat>
#include <climits>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {

constexpr int RT_TT = 32;       // tokens per block tile
constexpr int RT_TE = 64;       // experts per block tile
constexpr int RT_HC = 32;       // terms per fp32 partial sum
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

__global__ void __launch_bounds__(RT_THREADS) router_logits_kernel(RouterLogitsArgs a) {
    __shared__ __align__(16) float xs[RT_HC][RT_TT];
    __shared__ __align__(16) float ws[RT_HC][RT_TE];

    const int tid = threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.x * RT_TT;
    const int e0 = blockIdx.y * RT_TE;
    const int s = blockIdx.z;
    const int c_begin = (int)((int64_t)s * a.nchunks / a.S);
    const int c_end = (int)((int64_t)(s + 1) * a.nchunks / a.S);

    const int tg = tid / 16;    // tokens 2*tg, 2*tg+1
    const int eg = tid % 16;    // experts 4*eg .. 4*eg+3

    // staging assignment: threads 0..127 load x (token tid/4, vector tid%4),
    // all 256 load w (expert tid/4, vector tid%4); a vector is 8 bf16.
    const int xl_t = tid / 4, xl_v = tid % 4;
    const int wl_e = tid / 4, wl_v = tid % 4;

    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;

    auto load_chunk = [&](int c, uint4& xv, uint4& wv) {
        const int h = c * RT_HC;
        xv = make_uint4(0, 0, 0, 0);
        wv = make_uint4(0, 0, 0, 0);
        if (tid < 128) {
            const int64_t t = t0 + xl_t;
            const int hh = h + xl_v * 8;
            if (t < a.T && hh < a.H) xv = *reinterpret_cast<const uint4*>(a.x + t * a.H + hh);
        }
        {
            const int e = e0 + wl_e;
            const int hh = h + wl_v * 8;
            if (e < a.E && hh < a.H)
                wv = *reinterpret_cast<const uint4*>(a.wr + (int64_t)e * a.H + hh);
        }
    };
    auto store_chunk = [&](const uint4& xv, const uint4& wv) {
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
        if (tid < 128) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                xs[xl_v * 8 + 2 * q][xl_t] = __uint_as_float(xw[q] << 16);
                xs[xl_v * 8 + 2 * q + 1][xl_t] = __uint_as_float(xw[q] & 0xFFFF0000u);
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            ws[wl_v * 8 + 2 * q][wl_e] = __uint_as_float(ww[q] << 16);
            ws[wl_v * 8 + 2 * q + 1][wl_e] = __uint_as_float(ww[q] & 0xFFFF0000u);
        }
    };

    uint4 xv, wv;
    if (c_begin < c_end) load_chunk(c_begin, xv, wv);
    for (int c = c_begin; c < c_end; ++c) {
        __syncthreads();
        store_chunk(xv, wv);
        __syncthreads();
        if (c + 1 < c_end) load_chunk(c + 1, xv, wv);
        float p[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) p[i] = 0.0f;
#pragma unroll 8
        for (int h = 0; h < RT_HC; ++h) {
            const float2 xx = *reinterpret_cast<const float2*>(&xs[h][2 * tg]);
            const float4 w4 = *reinterpret_cast<const float4*>(&ws[h][4 * eg]);
            p[0] = __fmaf_rn(xx.x, w4.x, p[0]);
            p[1] = __fmaf_rn(xx.x, w4.y, p[1]);
            p[2] = __fmaf_rn(xx.x, w4.z, p[2]);
            p[3] = __fmaf_rn(xx.x, w4.w, p[3]);
            p[4] = __fmaf_rn(xx.y, w4.x, p[4]);
            p[5] = __fmaf_rn(xx.y, w4.y, p[5]);
            p[6] = __fmaf_rn(xx.y, w4.z, p[6]);
            p[7] = __fmaf_rn(xx.y, w4.w, p[7]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += (double)p[i];
    }

#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int64_t t = t0 + 2 * tg + i;
        if (t >= a.T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + 4 * eg + j;
            if (e < a.E) a.P[((int64_t)s * a.T + t) * a.E + e] = acc[i * 4 + j];
        }
    }

    // squared norms of this split's range (fp64 sums of exact squares)
    const int warp = tid / 32, lane = tid % 32;
    const int h_lo = c_begin * RT_HC;
    const int h_hi = min(c_end * RT_HC, a.H);
    if (blockIdx.y == 0) {
        for (int i = warp; i < RT_TT; i += RT_THREADS / 32) {
            const int64_t t = t0 + i;
            if (t >= a.T) break;
            double q = 0.0;
            for (int h = h_lo + lane; h < h_hi; h += 32) {
                const double v = (double)bf16_bits_to_float(a.x[t * a.H + h]);
                q += v * v;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
            if (lane == 0) a.xn2[(int64_t)s * a.T + t] = q;
        }
    }
    if (blockIdx.x == 0) {
        for (int i = warp; i < RT_TE; i += RT_THREADS / 32) {
            const int e = e0 + i;
            if (e >= a.E) break;
            double q = 0.0;
            for (int h = h_lo + lane; h < h_hi; h += 32) {
                const double v = (double)bf16_bits_to_float(a.wr[(int64_t)e * a.H + h]);
                q += v * v;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
            if (lane == 0) a.wn2[(int64_t)s * a.E + e] = q;
        }
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

constexpr int TK_MAXJ = 8;   // experts per lane (E <= 256)

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

__global__ void __launch_bounds__(256) router_topk_kernel(RouterTopkArgs a, DevCtx ctx) {
    const int lane = threadIdx.x % 32;
    const int64_t t = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (t >= a.T) return;

    const int nj = (a.E + 31) / 32;
    // g_32 + 2^-45, with a little slack for the fp64 norm sums and sqrt
    const double kRel = (32.0 * 0x1p-24) / (1.0 - 32.0 * 0x1p-24) + 0x1p-45 + 0x1p-40;
    const double kFx = (double)(a.H + 1) * 0x1p-41;

    double xn2 = 0.0;
    for (int s = 0; s < a.S; ++s) xn2 += a.xn2[(int64_t)s * a.T + t];
    const double xnorm = sqrt(xn2);

    double L[TK_MAXJ];
    double wnorm[TK_MAXJ];
    double eps_star = 0.0;
    bool range_bad = false;
#pragma unroll
    for (int j = 0; j < TK_MAXJ; ++j) {
        L[j] = -DBL_MAX;
        wnorm[j] = 0.0;
        const int e = lane + 32 * j;
        if (j < nj && e < a.E) {
            double l = 0.0, q = 0.0;
            for (int s = 0; s < a.S; ++s) {
                l += a.P[((int64_t)s * a.T + t) * a.E + e];
                q += a.wn2[(int64_t)s * a.E + e];
            }
            double b = 0.0;
            if (a.bias) {
                b = (double)a.bias[e];
                if (fabs(b) >= 0x1p21) range_bad = true;
            }
            l += b;
            wnorm[j] = sqrt(q);
            if (xnorm * wnorm[j] >= 0x1p22) range_bad = true;
            const double eps = kRel * xnorm * wnorm[j] + kFx + fabs(l) * 0x1p-50;
            eps_star = fmax(eps_star, eps);
            L[j] = l;
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        eps_star = fmax(eps_star, __shfl_xor_sync(0xffffffffu, eps_star, off));

    // the K+1 best by l~ (ties to the lower index)
    const int nsel = min(a.K + 1, a.E);
    uint32_t taken = 0;
    int sel_e[17];
    double sel_l[17];
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
        sel_e[k] = be;
        sel_l[k] = bv;
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
    }

    bool certified = true;
    for (int i = 0; i + 1 < nsel; ++i)
        if (!(sel_l[i] - sel_l[i + 1] > 2.0 * eps_star)) certified = false;

    int out_e[16];
    double out_l[16];
    if (certified) {
        for (int k = 0; k < a.K; ++k) {
            out_e[k] = sel_e[k];
            out_l[k] = sel_l[k];
        }
    } else {
        // exact fixed-point logits of every candidate
        const double thr = sel_l[a.K - 1] - 2.0 * eps_star;
        long long lfx[TK_MAXJ];
        uint32_t cand = 0;
#pragma unroll
        for (int j = 0; j < TK_MAXJ; ++j) {
            lfx[j] = LLONG_MIN;
            const int e = lane + 32 * j;
            if (j < nj && e < a.E && L[j] >= thr) cand |= 1u << j;
        }
        const uint16_t* xr = a.x + t * a.H;
        for (int j = 0; j < nj; ++j) {
            uint32_t m = __ballot_sync(0xffffffffu, (cand >> j) & 1u);
            while (m) {
                const int src = __ffs(m) - 1;
                m &= m - 1;
                const int e = src + 32 * j;
                const uint16_t* wrow = a.wr + (int64_t)e * a.H;
                long long acc = 0;
                for (int h = lane; h < a.H; h += 32) {
                    const float p = __fmul_rn(bf16_bits_to_float(xr[h]), bf16_bits_to_float(wrow[h]));
                    acc += __float2ll_rn(__fmul_rn(p, 0x1p40f));
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (a.bias) acc += __float2ll_rn(__fmul_rn(a.bias[e], 0x1p40f));
                if (lane == src) lfx[j] = acc;
            }
        }
        uint32_t used = 0;
        for (int k = 0; k < a.K; ++k) {
            long long bv = LLONG_MIN;
            int be = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < TK_MAXJ; ++j) {
                const int e = lane + 32 * j;
                if (((cand >> j) & 1u) && !((used >> j) & 1u)) {
                    if (lfx[j] > bv || (lfx[j] == bv && e < be)) {
                        bv = lfx[j];
                        be = e;
                    }
                }
            }
            warp_argmax_i64(bv, be);
            out_e[k] = be;
            out_l[k] = (double)bv * 0x1p-40;
            if ((be & 31) == lane) used |= 1u << (be >> 5);
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
        // registers indexed by a lane-dependent k: select through a small loop
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

RouterPlan router_plan(int64_t T, int H, int E, int num_sms) {
    RouterPlan p;
    p.nchunks = (H + RT_HC - 1) / RT_HC;
    const int64_t tiles = ((T + RT_TT - 1) / RT_TT) * ((E + RT_TE - 1) / RT_TE);
    int64_t want = tiles > 0 ? (2 * (int64_t)num_sms + tiles - 1) / tiles : 1;
    // keep at least 4 chunks per split so the fp64 partial traffic stays small
    const int64_t cap = (p.nchunks + 3) / 4;
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
    dim3 grid((unsigned)((T + RT_TT - 1) / RT_TT), (unsigned)((E + RT_TE - 1) / RT_TE),
              (unsigned)plan.S);
    router_logits_kernel<<<grid, RT_THREADS, 0, stream>>>(la);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (between) between(stream);
    RouterTopkArgs ta{P, xn2, wn2, x, wr, bias, T, H, E, K, plan.S, idx, w};
    const unsigned blocks = (unsigned)((T + 7) / 8);
    router_topk_kernel<<<blocks, 256, 0, stream>>>(ta, ctx);
    return cudaGetLastError();
}

}  // namespace moe
