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
#include <atomic>
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "route_select.cuh"

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
    pdl_enter();
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
    int H, E, K, S, nchunks;
    int32_t* idx;         // [T][K]
    float* w;             // [T][K]
};

constexpr int TK_WARPS = 8;       // tokens per block
constexpr int TK_CAP = TK_WARPS * 256;

// One warp per token ranks l~; tokens whose order the bound leaves open put
// their candidates in a block-wide list whose exact logits all 8 warps
// compute together, then finish their selection from it.
__global__ void __launch_bounds__(TK_WARPS * 32, 2) router_topk_kernel(RouterTopkArgs a, DevCtx ctx) {
    pdl_enter();
    __shared__ uint8_t c_tok[TK_CAP];
    __shared__ uint16_t c_e[TK_CAP];
    __shared__ long long c_val[TK_CAP];
    __shared__ double Ls[TK_WARPS][256];   // sum over splits of the partial logits
    __shared__ double Qs[256];             // sum over splits of ||w_e||^2
    __shared__ double Xs[TK_WARPS];        // sum over splits of ||x||^2
    __shared__ int s_oe[TK_WARPS][TK_MAXK];
    __shared__ double s_ol[TK_WARPS][TK_MAXK];
    __shared__ double s_bound[2];
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

    if (warp == 0) {
        double wn, bm;
        bound_constants(Qs, a.bias, a.H, a.E, lane, wn, bm);
        if (lane == 0) {
            s_bound[0] = wn;
            s_bound[1] = bm;
        }
    }
    __syncthreads();
    // fp32 chains of RT_HC terms; fp64: the chunk sums of one split, then the S split partials
    const int per_split = (a.nchunks + a.S - 1) / a.S;
    const double k_rel = router_k_rel(RT_HC, per_split + a.S + 1);
    bool certified = true;
    bool range_bad = false;
    if (active)
        certified = rank_certified(Ls[warp], Xs[warp], a.bias, a.H, a.E, a.K, k_rel, s_bound[0], s_bound[1], lane,
                                   warp, s_oe[warp], s_ol[warp], range_bad, c_tok, c_e, &n_cand);
    __syncthreads();
    const int nc = n_cand;
    exact_candidates(nc, c_tok, c_e, c_val, t_base, a.x, a.wr, a.H, a.bias, warp, TK_WARPS, lane);
    __syncthreads();

    if (!active) return;
    if (__any_sync(0xffffffffu, range_bad) && lane == 0) record_error(ctx.err, MOE_ERANGE);
    finish_token(certified, warp, t, nc, c_tok, c_e, c_val, a.K, s_oe[warp], s_ol[warp], lane, a.idx, a.w);
}

// ----------------------------------------------------------------------------- small batches
//
// One cluster of 8 CTAs per group of TB tokens computes the whole router in
// one launch.  CTA r of the cluster owns experts [r*ceil(E/8), ...), whose
// router rows are one contiguous block of W_r: two bulk copies bring that
// block and the group's x rows into shared memory.  A warp handles experts
// e and e+8 of the slice over one half of H (16 warps: 8 expert pairs x 2
// halves); each lane takes pairs of 16-byte fragments, which give, per token,
// a chain of 16 fp32 FMAs from zero, added into an fp64 total; the warp sums
// its lanes' totals in fp64 and the two halves are added in fp64.  The logits
// and the squared weight norms go to the leader CTA's shared memory
// (distributed shared memory); after the cluster barrier the leader's warps
// run the same certified selection as router_topk_kernel, one token each.

constexpr int RS_CLUSTER = 8;
constexpr int RS_THREADS = 512;
constexpr int RS_WARPS = RS_THREADS / 32;
constexpr int RS_PAIRW = 8;                      // warps per half of H (expert pairs in flight)
constexpr int RS_SPLIT = RS_WARPS / RS_PAIRW;    // halves of H
static_assert(RS_SPLIT == 2, "the fp64 depth of the bound counts one add of the halves");

struct RouterSmallArgs {
    const uint16_t* x;
    const uint16_t* wr;
    const float* bias;
    int64_t T;
    int H, E, K;
    int32_t* idx;
    float* w;
    const uint8_t* warm;    // bytes the next kernels read first (null: none): prefetched into L2
    int64_t warm_bytes;     // a multiple of 16 (0 when warm is null)
};

constexpr int64_t RS_WARM_PIECE = 32 * 1024;   // bytes of one L2 prefetch

__host__ __device__ constexpr int rs_epc(int E) { return (E + RS_CLUSTER - 1) / RS_CLUSTER; }
__host__ __device__ constexpr size_t rs_align(size_t v) { return (v + 15) & ~size_t(15); }

// dynamic shared memory of one CTA: xs [TB][H] bf16 | ws [epc][H] bf16 | Ls [TB][E] f64 |
// Qs [E] f64 | Xs [TB] f64 | xred [TB][RS_WARPS] f32 | Ph [2][epc][TB] f64 | Qh [2][epc] f32 |
// c_val [TB*E] i64 | c_e [TB*E] u16 | c_tok [TB*E] u8 | n_cand, abort flag | mbarrier
__host__ __device__ inline size_t rs_smem_bytes(int TB, int H, int E) {
    size_t o = rs_align((size_t)TB * H * 2) + rs_align((size_t)rs_epc(E) * H * 2);
    o += rs_align((size_t)TB * E * 8) + rs_align((size_t)E * 8) + rs_align((size_t)TB * 8);
    o += rs_align((size_t)TB * RS_WARPS * 4);
    o += rs_align((size_t)RS_SPLIT * rs_epc(E) * TB * 8) + rs_align((size_t)RS_SPLIT * rs_epc(E) * 4);
    o += rs_align((size_t)TB * E * 8) + rs_align((size_t)TB * E * 2) + rs_align((size_t)TB * E) + 16 + 16;
    return o;
}

__device__ __forceinline__ void bf16x8(const uint4& v, float (&f)[8]) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        f[2 * q] = __uint_as_float(u[q] << 16);
        f[2 * q + 1] = __uint_as_float(u[q] & 0xFFFF0000u);
    }
}

template <int TB>
__global__ void __cluster_dims__(RS_CLUSTER, 1, 1) __launch_bounds__(RS_THREADS)
    router_small_kernel(RouterSmallArgs a, DevCtx ctx) {
    // Clusters past the batch's groups only warm L2: they prefetch the bytes the expert FFN
    // reads first (its first experts' up weights) while the router and the permutation run,
    // when the memory system is otherwise idle.  They run on SMs the router leaves free, so
    // that no routing warp waits on the prefetches' issue; pieces of 32 KB, strided over their
    // lanes.  They start before the wait on the preceding kernel (the weight banks are not
    // written by it, and a prefetch changes no data), so the copies overlap its tail too.
    const int64_t n_groups = (a.T + TB - 1) / TB;
    if ((int64_t)(blockIdx.x / RS_CLUSTER) >= n_groups) {
        const int64_t first = n_groups * RS_CLUSTER * 32;
        const int64_t pieces = (a.warm_bytes + RS_WARM_PIECE - 1) / RS_WARM_PIECE;
        const int64_t stride = ((int64_t)gridDim.x - n_groups * RS_CLUSTER) * 32;
        for (int64_t q = (int64_t)blockIdx.x * 32 + threadIdx.x % 32 - first; threadIdx.x < 32 && q < pieces;
             q += stride) {
            const int64_t off = q * RS_WARM_PIECE;
            bulk_prefetch_l2(a.warm + off, (uint32_t)min(RS_WARM_PIECE, a.warm_bytes - off));
        }
        return;
    }
    pdl_enter();
    namespace cg = cooperative_groups;
    extern __shared__ __align__(16) unsigned char rs_smem[];
    const int H = a.H, E = a.E;
    const int epc = rs_epc(E);
    unsigned char* p = rs_smem;
    uint16_t* xs = reinterpret_cast<uint16_t*>(p);
    p += rs_align((size_t)TB * H * 2);
    uint16_t* ws = reinterpret_cast<uint16_t*>(p);
    p += rs_align((size_t)epc * H * 2);
    double* Ls = reinterpret_cast<double*>(p);
    p += rs_align((size_t)TB * E * 8);
    double* Qs = reinterpret_cast<double*>(p);
    p += rs_align((size_t)E * 8);
    double* Xs = reinterpret_cast<double*>(p);
    p += rs_align((size_t)TB * 8);
    float* xred = reinterpret_cast<float*>(p);
    p += rs_align((size_t)TB * RS_WARPS * 4);
    double* Ph = reinterpret_cast<double*>(p);   // [half][local expert][token] partial logits
    p += rs_align((size_t)RS_SPLIT * epc * TB * 8);
    float* Qh = reinterpret_cast<float*>(p);     // [half][local expert] partial squared norms
    p += rs_align((size_t)RS_SPLIT * epc * 4);
    long long* c_val = reinterpret_cast<long long*>(p);
    p += rs_align((size_t)TB * E * 8);
    uint16_t* c_e = reinterpret_cast<uint16_t*>(p);
    p += rs_align((size_t)TB * E * 2);
    uint8_t* c_tok = p;
    p += rs_align((size_t)TB * E);
    int* n_cand = reinterpret_cast<int*>(p);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(p + 4);
    p += 16;
    uint64_t* bar = reinterpret_cast<uint64_t*>(p);

    cg::cluster_group cluster = cg::this_cluster();
    const unsigned rank = cluster.block_rank();
    const bool leader = rank == 0;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int64_t t_base = (int64_t)(blockIdx.x / RS_CLUSTER) * TB;
    const int n_tok = (int)min((int64_t)TB, a.T - t_base);
    const int HV = H / 8;   // 16-byte fragments per row
    const int e_lo = (int)rank * epc, e_hi = min(E, e_lo + epc);
    const int n_e = max(0, e_hi - e_lo);

    // 1. the group's x rows and this CTA's router rows, one bulk copy each
    if (tid == 0) {
        *n_cand = 0;
        *abort_flag = 0;
        mbar_init(smem_u32(bar), 1);
        fence_mbar_init();
        const uint32_t xb = (uint32_t)n_tok * H * 2, wb = (uint32_t)n_e * H * 2;
        mbar_arrive_expect_tx(smem_u32(bar), xb + wb);
        bulk_load_1d(smem_u32(xs), a.x + t_base * H, xb, smem_u32(bar));
        if (wb) bulk_load_1d(smem_u32(ws), a.wr + (int64_t)e_lo * H, wb, smem_u32(bar));
    }
    __syncthreads();
    if (!mbar_wait(smem_u32(bar), 0, ctx, abort_flag)) mbar_wait_drain(smem_u32(bar), 0, ctx.timeout_ns);

    // the leader's ||x||^2 (fp32 sums of exact squares)
    if (leader) {
        for (int t = 0; t < n_tok; ++t) {
            float q = 0.0f;
            for (int v = tid; v < HV; v += RS_THREADS) {
                float f[8];
                bf16x8(*reinterpret_cast<const uint4*>(xs + (size_t)t * H + 8 * v), f);
#pragma unroll
                for (int j = 0; j < 8; ++j) q = __fmaf_rn(f[j], f[j], q);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) q = __fadd_rn(q, __shfl_xor_sync(0xffffffffu, q, off));
            if (lane == 0) xred[t * RS_WARPS + warp] = q;
        }
        __syncthreads();
        if (tid < n_tok) {
            float q = 0.0f;
            for (int i = 0; i < RS_WARPS; ++i) q = __fadd_rn(q, xred[tid * RS_WARPS + i]);
            Xs[tid] = (double)q;
        }
    }

    // 2. this CTA's experts: warp w takes local experts w + 16m and w + 16m + 8
    double* Ls_lead = cluster.map_shared_rank(Ls, 0);
    double* Qs_lead = cluster.map_shared_rank(Qs, 0);
    // warp (pair, half): local experts pair + 16m and pair + 16m + 8, fragments [vs, ve) of H
    const int pair = warp % RS_PAIRW, half = warp / RS_PAIRW;
    const int hv_half = (HV + RS_SPLIT - 1) / RS_SPLIT;
    const int vs = half * hv_half, ve = min(HV, vs + hv_half);
    for (int l0 = pair; l0 < n_e; l0 += 2 * RS_PAIRW) {
        const int l1 = l0 + RS_PAIRW;
        const bool has1 = l1 < n_e;
        const uint16_t* w0 = ws + (size_t)l0 * H;
        const uint16_t* w1 = ws + (size_t)(has1 ? l1 : l0) * H;
        double acc0[TB], acc1[TB];
#pragma unroll
        for (int t = 0; t < TB; ++t) acc0[t] = acc1[t] = 0.0;
        float q0 = 0.0f, q1 = 0.0f;
        for (int v0 = vs + lane; v0 < ve; v0 += 64) {
            const int v1 = v0 + 32;
            const bool ok1 = v1 < ve;
            const uint4 z4 = make_uint4(0, 0, 0, 0);
            float a0[16], a1[16];
            {
                float f[8];
                bf16x8(*reinterpret_cast<const uint4*>(w0 + 8 * v0), f);
#pragma unroll
                for (int j = 0; j < 8; ++j) a0[j] = f[j];
                bf16x8(ok1 ? *reinterpret_cast<const uint4*>(w0 + 8 * v1) : z4, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) a0[8 + j] = f[j];
                bf16x8(*reinterpret_cast<const uint4*>(w1 + 8 * v0), f);
#pragma unroll
                for (int j = 0; j < 8; ++j) a1[j] = f[j];
                bf16x8(ok1 ? *reinterpret_cast<const uint4*>(w1 + 8 * v1) : z4, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) a1[8 + j] = f[j];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                q0 = __fmaf_rn(a0[j], a0[j], q0);
                q1 = __fmaf_rn(a1[j], a1[j], q1);
            }
#pragma unroll
            for (int t = 0; t < TB; ++t) {
                float xv[16];
                {
                    float f[8];
                    bf16x8(*reinterpret_cast<const uint4*>(xs + (size_t)t * H + 8 * v0), f);
#pragma unroll
                    for (int j = 0; j < 8; ++j) xv[j] = f[j];
                    bf16x8(ok1 ? *reinterpret_cast<const uint4*>(xs + (size_t)t * H + 8 * v1) : z4, f);
#pragma unroll
                    for (int j = 0; j < 8; ++j) xv[8 + j] = f[j];
                }
                float c0 = 0.0f, c1 = 0.0f;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    c0 = __fmaf_rn(xv[j], a0[j], c0);
                    c1 = __fmaf_rn(xv[j], a1[j], c1);
                }
                acc0[t] += (double)c0;
                acc1[t] += (double)c1;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
            for (int t = 0; t < TB; ++t) {
                acc0[t] += __shfl_xor_sync(0xffffffffu, acc0[t], off);
                acc1[t] += __shfl_xor_sync(0xffffffffu, acc1[t], off);
            }
            q0 = __fadd_rn(q0, __shfl_xor_sync(0xffffffffu, q0, off));
            q1 = __fadd_rn(q1, __shfl_xor_sync(0xffffffffu, q1, off));
        }
        if (lane < TB) {
            // lane t parks token t's two partial logits (registers indexed at compile time)
#pragma unroll
            for (int t = 0; t < TB; ++t)
                if (t == lane) {
                    Ph[((size_t)half * epc + l0) * TB + t] = acc0[t];
                    if (has1) Ph[((size_t)half * epc + l1) * TB + t] = acc1[t];
                }
        }
        if (lane == 0) {
            Qh[half * epc + l0] = q0;
            if (has1) Qh[half * epc + l1] = q1;
        }
    }
    __syncthreads();
    // the two halves of each (expert, token) logit, added in fp64, go to the leader
    for (int i = tid; i < n_e * TB; i += RS_THREADS) {
        const int l = i / TB, t = i % TB;
        Ls_lead[t * E + e_lo + l] = Ph[(size_t)l * TB + t] + Ph[((size_t)epc + l) * TB + t];
    }
    for (int l = tid; l < n_e; l += RS_THREADS) Qs_lead[e_lo + l] = (double)__fadd_rn(Qh[l], Qh[epc + l]);
    // every CTA's stores to the leader become visible to it here
    cluster.sync();
    if (!leader) return;

    // 3. selection, one warp per token (the leader's shared memory only)
    __shared__ int s_oe[RS_WARPS][TK_MAXK];
    __shared__ double s_ol[RS_WARPS][TK_MAXK];
    __shared__ double s_bound[2];
    if (warp == 0) {
        double wn, bm;
        bound_constants(Qs, a.bias, H, E, lane, wn, bm);
        if (lane == 0) {
            s_bound[0] = wn;
            s_bound[1] = bm;
        }
    }
    __syncthreads();
    // fp32 chains of 16 terms; fp64: the lane's chain sums over its half of H, 5 warp levels,
    // the add of the two halves (and one spare)
    const double k_rel = router_k_rel(16, ((HV + RS_SPLIT - 1) / RS_SPLIT + 63) / 64 + 7);
    const bool active = warp < n_tok;
    bool certified = true;
    bool range_bad = false;
    if (active)
        certified = rank_certified(Ls + (size_t)warp * E, Xs[warp], a.bias, H, E, a.K, k_rel, s_bound[0],
                                   s_bound[1], lane, warp, s_oe[warp], s_ol[warp], range_bad, c_tok, c_e, n_cand);
    __syncthreads();
    const int nc = *n_cand;
    exact_candidates(nc, c_tok, c_e, c_val, t_base, a.x, a.wr, H, a.bias, warp, RS_WARPS, lane);
    __syncthreads();
    if (!active) return;
    if (__any_sync(0xffffffffu, range_bad) && lane == 0) record_error(ctx.err, MOE_ERANGE);
    finish_token(certified, warp, t_base + warp, nc, c_tok, c_e, c_val, a.K, s_oe[warp], s_ol[warp], lane, a.idx,
                 a.w);
}

// ----------------------------------------------------------------------------- large batches
//
// One cluster of CS CTAs per tile of BT = NTH/4 tokens (all E <= 128
// experts): CTA r of the cluster takes stages [r n/CS, (r+1) n/CS) of the
// hidden dimension, 32 values each, staged in shared memory as fp32 (double
// buffered).  Thread (ty, tx) owns 4 tokens x 8 experts; per stage each
// (token, expert) gets a chain of 32 fp32 FMAs from zero, added into an fp32
// total (so a product passes through at most 31 + m roundings, m = stages per
// CTA).  The CTA's fp32 partial logits and squared norms stay in its shared
// memory; after the cluster barrier CTA r sums, in fp64, the CS partials of
// its own BT/CS tokens over distributed shared memory, ranks them (one warp
// per token), computes the exact logits of every open candidate with the
// whole CTA, and finishes them.

constexpr int RF_HS = 32;       // hidden values per stage and per fp32 chain
constexpr int RF_E = 128;       // experts per tile (E <= 128)

struct RouterFusedArgs {
    const uint16_t* x;
    const uint16_t* wr;
    const float* bias;
    int64_t T;
    int H, E, K;
    int n_stages;         // ceil(H / RF_HS)
    int32_t* idx;
    float* w;
};

template <int NTH, int CS>
struct RfLayout {
    static constexpr int WARPS = NTH / 32;
    static constexpr int BT = NTH / 4;          // tokens per tile (16-byte x fragments per stage = NTH)
    static constexpr int TPC = BT / CS;         // tokens each CTA selects
    static constexpr int TPW = (TPC + WARPS - 1) / WARPS;
    static constexpr int NWF = 4 * RF_E;        // 16-byte w fragments per stage
    static constexpr size_t stage_floats = (size_t)RF_HS * (BT + RF_E);
    static constexpr size_t ring_bytes = 2 * stage_floats * 4;
    static constexpr size_t pl_bytes = (size_t)BT * RF_E * 4;
    // the candidate lists of the selection reuse the ring after the partials are read
    static constexpr size_t o_cv = 0;
    static constexpr size_t o_ce = o_cv + (size_t)TPC * RF_E * 8;
    static constexpr size_t o_ct = o_ce + (size_t)TPC * RF_E * 2;
    static constexpr size_t cand_end = o_ct + (size_t)TPC * RF_E;
    static constexpr size_t main_bytes =
        ((ring_bytes > pl_bytes ? ring_bytes : pl_bytes) > cand_end ? (ring_bytes > pl_bytes ? ring_bytes : pl_bytes)
                                                                    : (cand_end + 15) / 16 * 16);
    static constexpr size_t o_xq = main_bytes;
    static constexpr size_t o_wq = o_xq + NTH * 4;
    static constexpr size_t o_xp = o_wq + NWF * 4;
    static constexpr size_t o_wp = o_xp + BT * 4;
    static constexpr size_t o_ls = o_wp + RF_E * 4;
    static constexpr size_t o_qs = o_ls + (size_t)TPC * RF_E * 8;
    static constexpr size_t o_xs = o_qs + RF_E * 8;
    static constexpr size_t o_oe = o_xs + ((TPC * 8 + 15) / 16) * 16;   // [TPC][TK_MAXK] int
    static constexpr size_t o_ol = o_oe + (size_t)TPC * TK_MAXK * 4;       // [TPC][TK_MAXK] double
    static constexpr size_t o_nc = o_ol + (size_t)TPC * TK_MAXK * 8 + 16;   // + the two bound constants
    static constexpr size_t bytes = o_nc + 16;
};

template <int NTH, int CS>
__global__ void __cluster_dims__(CS, 1, 1) __launch_bounds__(NTH, 1)
    router_fused_kernel(RouterFusedArgs a, DevCtx ctx) {
    pdl_enter();
    namespace cg = cooperative_groups;
    using L = RfLayout<NTH, CS>;
    constexpr int BT = L::BT, TPC = L::TPC, WARPS = L::WARPS, TPW = L::TPW, NWF = L::NWF;
    constexpr int NW = (NWF + NTH - 1) / NTH;   // w fragments per thread and stage (the last may be empty)
    extern __shared__ __align__(16) unsigned char rf_smem[];
    float* ring = reinterpret_cast<float*>(rf_smem);
    float* Pl = ring;                             // [BT][RF_E] after the main loop
    long long* c_val = reinterpret_cast<long long*>(rf_smem + L::o_cv);   // after the partials are read
    uint16_t* c_e = reinterpret_cast<uint16_t*>(rf_smem + L::o_ce);
    uint8_t* c_tok = rf_smem + L::o_ct;
    float* xq = reinterpret_cast<float*>(rf_smem + L::o_xq);
    float* wq = reinterpret_cast<float*>(rf_smem + L::o_wq);
    float* xpart = reinterpret_cast<float*>(rf_smem + L::o_xp);
    float* wpart = reinterpret_cast<float*>(rf_smem + L::o_wp);
    double* Ls = reinterpret_cast<double*>(rf_smem + L::o_ls);
    double* Qs = reinterpret_cast<double*>(rf_smem + L::o_qs);
    double* Xs = reinterpret_cast<double*>(rf_smem + L::o_xs);
    int* s_oe = reinterpret_cast<int*>(rf_smem + L::o_oe);
    double* s_ol = reinterpret_cast<double*>(rf_smem + L::o_ol);
    int* n_cand = reinterpret_cast<int*>(rf_smem + L::o_nc);

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int ty = tid / 16, tx = tid % 16;     // tokens 4ty..4ty+3; experts 4tx.. and 64+4tx..
    const int64_t t0 = (int64_t)(blockIdx.x / CS) * BT;
    const int H = a.H, E = a.E;
    const int s_begin = rank * a.n_stages / CS, s_end = (rank + 1) * a.n_stages / CS;

    // staging: x fragment tid is row tid % BT, 8 values at 8 (tid / BT); w fragment
    // i = tid + NTH k is row i % 128, 8 values at 8 (i / 128).  Consecutive lanes take
    // consecutive rows, so the transposed fp32 stores are conflict-free.  Each fragment
    // slot keeps the fp32 sum of its squares.
    uint4 xv, wv[NW];
    float xsq = 0.0f, wsq[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) wsq[k] = 0.0f;
    auto load = [&](int st) {
        const int h0 = st * RF_HS;
        {
            const int row = tid % BT, h = h0 + 8 * (tid / BT);
            const int64_t t = t0 + row;
            xv = make_uint4(0, 0, 0, 0);
            if (t < a.T && h < H) xv = *reinterpret_cast<const uint4*>(a.x + t * H + h);
        }
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            const int i = tid + NTH * k, row = i % RF_E, h = h0 + 8 * (i / RF_E);
            wv[k] = make_uint4(0, 0, 0, 0);
            if (i < NWF && row < E && h < H) wv[k] = *reinterpret_cast<const uint4*>(a.wr + (int64_t)row * H + h);
        }
    };
    auto store = [&](int buf) {
        float* xs = ring + (size_t)buf * L::stage_floats;   // [RF_HS][BT]
        float* ws = xs + RF_HS * BT;                        // [RF_HS][RF_E]
        {
            const int row = tid % BT, f8 = 8 * (tid / BT);
            float f[8];
            bf16x8(xv, f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                xs[(f8 + j) * BT + row] = f[j];
                xsq = __fmaf_rn(f[j], f[j], xsq);
            }
        }
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            const int i = tid + NTH * k, row = i % RF_E, f8 = 8 * (i / RF_E);
            if (i < NWF) {
                float f[8];
                bf16x8(wv[k], f);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ws[(f8 + j) * RF_E + row] = f[j];
                    wsq[k] = __fmaf_rn(f[j], f[j], wsq[k]);
                }
            }
        }
    };

    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

    if (s_begin < s_end) {
        load(s_begin);
        store(0);
    }
    __syncthreads();
    for (int st = s_begin; st < s_end; ++st) {
        const int buf = (st - s_begin) & 1;
        if (st + 1 < s_end) load(st + 1);
        const float* xs = ring + (size_t)buf * L::stage_floats;
        const float* ws = xs + RF_HS * BT;
        float c[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) c[i][j] = 0.0f;
#pragma unroll
        for (int h = 0; h < RF_HS; ++h) {
            const float4 xx = *reinterpret_cast<const float4*>(xs + h * BT + 4 * ty);
            const float4 wa = *reinterpret_cast<const float4*>(ws + h * RF_E + 4 * tx);
            const float4 wb = *reinterpret_cast<const float4*>(ws + h * RF_E + 64 + 4 * tx);
            const float xr[4] = {xx.x, xx.y, xx.z, xx.w};
            const float w8[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) c[i][j] = __fmaf_rn(xr[i], w8[j], c[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = __fadd_rn(acc[i][j], c[i][j]);
        if (st + 1 < s_end) store(buf ^ 1);
        __syncthreads();
    }

    // this CTA's partials: logits [BT][RF_E] (over the ring, which is no longer read) and norms
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float* row = Pl + (4 * ty + i) * RF_E;
        *reinterpret_cast<float4*>(row + 4 * tx) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        *reinterpret_cast<float4*>(row + 64 + 4 * tx) = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
    xq[tid] = xsq;
#pragma unroll
    for (int k = 0; k < NW; ++k)
        if (tid + NTH * k < NWF) wq[tid + NTH * k] = wsq[k];
    if (tid == 0) *n_cand = 0;
    __syncthreads();
    if (tid < BT) {
        float q = 0.0f;
#pragma unroll
        for (int g = 0; g < 4; ++g) q = __fadd_rn(q, xq[g * BT + tid]);
        xpart[tid] = q;
    }
    if (tid < RF_E) {
        float q = 0.0f;
#pragma unroll
        for (int g = 0; g < 4; ++g) q = __fadd_rn(q, wq[g * RF_E + tid]);
        wpart[tid] = q;
    }
    cluster.sync();

    // CTA `rank` selects tokens rank*TPC .. +TPC-1 of the tile: fp64 sums of the CS partials
    {
        const float* Pr[CS];
        const float* Wr[CS];
        const float* Xr[CS];
#pragma unroll
        for (int r = 0; r < CS; ++r) {
            Pr[r] = cluster.map_shared_rank(Pl, r);
            Wr[r] = cluster.map_shared_rank(wpart, r);
            Xr[r] = cluster.map_shared_rank(xpart, r);
        }
        for (int i = tid; i < TPC * RF_E / 4; i += NTH) {
            const int tl = (4 * i) / RF_E, e = (4 * i) % RF_E;
            const int t = rank * TPC + tl;
            float4 v[CS];
#pragma unroll
            for (int r = 0; r < CS; ++r) v[r] = *reinterpret_cast<const float4*>(Pr[r] + t * RF_E + e);
            double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll
            for (int r = 0; r < CS; ++r) {
                s0 += (double)v[r].x;
                s1 += (double)v[r].y;
                s2 += (double)v[r].z;
                s3 += (double)v[r].w;
            }
            double* dst = Ls + tl * RF_E + e;
            dst[0] = s0;
            dst[1] = s1;
            dst[2] = s2;
            dst[3] = s3;
        }
        if (tid < RF_E) {
            double q = 0.0;
#pragma unroll
            for (int r = 0; r < CS; ++r) q += (double)Wr[r][tid];
            Qs[tid] = q;
        }
        if (tid < TPC) {
            double q = 0.0;
#pragma unroll
            for (int r = 0; r < CS; ++r) q += (double)Xr[r][rank * TPC + tid];
            Xs[tid] = q;
        }
    }
    // no CTA reuses or releases its shared memory while another still reads it
    cluster.sync();
    if (warp == 0) {
        double wn, bm;
        bound_constants(Qs, a.bias, H, E, lane, wn, bm);
        if (lane == 0) {
            s_ol[TPC * TK_MAXK] = wn;
            s_ol[TPC * TK_MAXK + 1] = bm;
        }
    }
    __syncthreads();
    const double wnmax = s_ol[TPC * TK_MAXK], bmax = s_ol[TPC * TK_MAXK + 1];

    // rank every token of this CTA, then one exact pass over all open candidates, then finish
    const int m = (a.n_stages + CS - 1) / CS;
    const double k_rel = router_k_rel(RF_HS + m, CS + 1);
    const int64_t ts0 = t0 + (int64_t)rank * TPC;
    bool cert[TPW];
    bool range_bad = false;
#pragma unroll
    for (int k = 0; k < TPW; ++k) {
        const int slot = warp + WARPS * k;
        cert[k] = true;
        if (slot < TPC && ts0 + slot < a.T)
            cert[k] = rank_certified(Ls + (size_t)slot * RF_E, Xs[slot], a.bias, H, E, a.K, k_rel, wnmax, bmax, lane,
                                     slot, s_oe + slot * TK_MAXK, s_ol + slot * TK_MAXK, range_bad, c_tok, c_e,
                                     n_cand);
    }
    __syncthreads();
    const int nc = *n_cand;
    exact_candidates(nc, c_tok, c_e, c_val, ts0, a.x, a.wr, H, a.bias, warp, WARPS, lane);
    __syncthreads();
    if (__any_sync(0xffffffffu, range_bad) && lane == 0) record_error(ctx.err, MOE_ERANGE);
#pragma unroll
    for (int k = 0; k < TPW; ++k) {
        const int slot = warp + WARPS * k;
        if (slot < TPC && ts0 + slot < a.T)
            finish_token(cert[k], slot, ts0 + slot, nc, c_tok, c_e, c_val, a.K, s_oe + slot * TK_MAXK,
                         s_ol + slot * TK_MAXK, lane, a.idx, a.w);
    }
}

// ----------------------------------------------------------------------------- host

// Batch-size boundaries of the router shapes, from CUDA-graph timings on
// B200 (H=2688, E=128, K=6): the expert-split clusters up to 256 tokens
// (14 us at 64), the two-kernel router up to 1023, the tensor-core router
// (route_tc.cu) from 1024 tokens (43 / 54 / 75 / 131 us at 1024 / 2048 / 4096 /
// 8192, against 50 / 83 / 98 / 193 for the best of the other large-batch shapes).
constexpr int64_t kRouterSmallMaxDefault = 256;
constexpr int64_t kRouterSplitMin = 3072;
constexpr int64_t kRouterTcMin = 1024;  // batches from this size take the tensor-core router (E <= 128)
constexpr size_t kRouterSmallSmemMax = 200 * 1024;

static int router_tt(int64_t T) { return T > 256 ? 64 : 16; }

// Whether a batch takes the tensor-core router (route_tc.cu): by size, or always under
// hook value 3; never for E > 128, K > 16 or a batch the expert-split clusters take.
static bool router_tc(int64_t T, int H, int E);

RouterPlan router_plan(int64_t T, int H, int E, int num_sms) {
    RouterPlan p;
    p.num_sms = num_sms;
    p.tc = router_tc(T, H, E) ? 1 : 0;
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
    if (E <= RF_E) {
        // room for the tensor-core router's slices whenever it could run (sizes do not depend
        // on the test hooks that choose the path)
        const size_t tcb = route_tc_scratch_bytes(T, H, E);
        if (tcb > p.p_bytes) p.p_bytes = tcb;
    }
    p.xn_bytes = (size_t)p.S * (size_t)T * sizeof(double);
    p.wn_bytes = (size_t)p.S * (size_t)E * sizeof(double);
    return p;
}

// Largest batch the one-launch cluster router takes (tokens); larger batches
// use the tiled logits kernel and router_topk_kernel.
std::atomic<int64_t> g_router_small_max{kRouterSmallMaxDefault};
// 0: by batch size; 1: every larger batch takes the two-kernel router; 2: every larger
// batch with E <= 128 takes the hidden-split clusters; 3: every larger batch with E <= 128
// takes the tensor-core router
std::atomic<int> g_router_split{0};

void set_router_small_max(int64_t v) { g_router_small_max.store(v < 0 ? kRouterSmallMaxDefault : v); }
void set_router_split(int v) { g_router_split.store(v >= 1 && v <= 3 ? v : 0); }

// How many clusters of the split-cluster router fit on the device at once (a
// cluster sits inside one GPC, so this is not the SM count over CS); cached
// per device.
template <int NTH, int CS>
static int64_t fused_max_clusters(int num_sms) {
    static std::atomic<int> cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load();
        if (c > 0) return c;
    }
    using L = RfLayout<NTH, CS>;
    auto kfn = router_fused_kernel<NTH, CS>;
    int n = 0;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3((unsigned)(CS * (num_sms / CS)));
        cfg.blockDim = dim3(NTH);
        cfg.dynamicSmemBytes = L::bytes;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    if (n < 1) n = num_sms / CS > 0 ? num_sms / CS : 1;
    if (dev >= 0 && dev < 64) cache[dev].store(n);
    return n;
}

// Time model of one tiling: waves of clusters x the work of one CTA (tokens x stages).
template <int NTH, int CS>
static int64_t fused_cost(int64_t T, int num_sms) {
    using L = RfLayout<NTH, CS>;
    const int64_t tiles = (T + L::BT - 1) / L::BT;
    const int64_t act = fused_max_clusters<NTH, CS>(num_sms);
    return (tiles + act - 1) / act * (int64_t)(L::BT * 8 / CS);
}

template <int NTH, int CS>
static cudaError_t launch_router_fused(const RouterFusedArgs& ra, const DevCtx& ctx, cudaStream_t stream) {
    using L = RfLayout<NTH, CS>;
    auto kfn = router_fused_kernel<NTH, CS>;
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (err != cudaSuccess) return err;
    const unsigned tiles = (unsigned)((ra.T + L::BT - 1) / L::BT);
    return launch_k(kfn, dim3(tiles * CS), dim3(NTH), L::bytes, stream, ra, ctx);
}

// Clusters of the expert-split router that fit on the current device at once (its clusters
// of 8 CTAs of one SM each must fit inside GPCs: 15 on a 148-SM B200), queried once per device.
static int router_small_max_clusters(int TB, int H, int E) {
    static std::atomic<int> cache[2][64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    const int slot = TB == 4 ? 0 : 1;
    int n = cache[slot][dev].load();
    if (n > 0) return n;
    const size_t smem = rs_smem_bytes(TB, H, E);
    auto kfn = TB == 4 ? router_small_kernel<4> : router_small_kernel<8>;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(RS_CLUSTER);
    cfg.blockDim = dim3(RS_THREADS);
    cfg.dynamicSmemBytes = smem;
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        n = 1;
    }
    cache[slot][dev].store(n);
    return n;
}

// Tokens per cluster of the expert-split router (0: the batch does not take it): 4 when the
// batch's clusters of 4 tokens fit on the device at once, else 8 (a second wave of clusters
// would double the time: at 64 tokens, 16 clusters of 4 against 15 that fit).
static int router_small_tb(int64_t T, int H, int E, bool query) {
    if (T > g_router_small_max.load() || rs_smem_bytes(4, H, E) > kRouterSmallSmemMax) return 0;
    if (rs_smem_bytes(8, H, E) > kRouterSmallSmemMax) return 4;
    if (!query) return 8;
    return (T + 3) / 4 <= router_small_max_clusters(4, H, E) ? 4 : 8;
}

static bool router_tc(int64_t T, int H, int E) {
    if (E > RF_E || router_small_tb(T, H, E, false) > 0) return false;
    const int mode = g_router_split.load();
    return mode == 3 || (mode == 0 && T >= kRouterTcMin);
}

template <int TB>
static cudaError_t launch_router_small(const RouterSmallArgs& ra, const DevCtx& ctx, cudaStream_t stream) {
    const size_t smem = rs_smem_bytes(TB, ra.H, ra.E);
    auto kfn = router_small_kernel<TB>;
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const unsigned groups = (unsigned)((ra.T + TB - 1) / TB);
    // clusters that only warm L2: those the device still fits beside the batch's groups
    const int fit = ra.warm ? router_small_max_clusters(TB, ra.H, ra.E) : 0;
    const unsigned warm = fit > (int)groups ? (unsigned)fit - groups : 0;
    return launch_k(kfn, dim3((groups + warm) * RS_CLUSTER), dim3(RS_THREADS), smem, stream, ra, ctx);
}

// Kernel launches launch_route makes for these sizes under the current hooks:
// the same tests, in the same order, as launch_route below.
int route_launches(int64_t T, int H, int E) {
    if (T == 0) return 0;
    if (router_small_tb(T, H, E, false) > 0) return 1;   // expert-split clusters
    if (router_tc(T, H, E)) return 3;                    // slices, integer products, selection
    const int split_mode = g_router_split.load();
    if (E <= RF_E && split_mode != 1 && (split_mode == 2 || T >= kRouterSplitMin)) return 1;   // hidden-split
    return 2;   // logits, then top-K
}

cudaError_t launch_route(const uint16_t* x, const uint16_t* wr, const float* bias, int64_t T, int H,
                         int E, int K, int32_t* idx, float* w, double* P, double* xn2, double* wn2,
                         const RouterPlan& plan, const DevCtx& ctx, cudaStream_t stream,
                         void (*between)(cudaStream_t), const void* warm, int64_t warm_bytes) {
    if (T == 0) return cudaSuccess;
    if (plan.tc) return launch_route_tc(x, wr, bias, T, H, E, K, idx, w, P, plan.num_sms, ctx, stream, between);
    const int tb = router_small_tb(T, H, E, true);
    if (tb > 0) {
        RouterSmallArgs ra{x, wr, bias, T, H, E, K, idx, w, static_cast<const uint8_t*>(warm),
                           warm ? (warm_bytes & ~(int64_t)15) : 0};
        if (ra.warm_bytes <= 0) ra.warm = nullptr;
        const cudaError_t err = tb == 4 ? launch_router_small<4>(ra, ctx, stream)
                                        : launch_router_small<8>(ra, ctx, stream);
        if (err == cudaSuccess && between) between(stream);   // one launch: nothing between
        return err;
    }
    const int split_mode = g_router_split.load();
    if (E <= RF_E && split_mode != 1 && (split_mode == 2 || T >= kRouterSplitMin)) {
        RouterFusedArgs fa{x, wr, bias, T, H, E, K, (H + RF_HS - 1) / RF_HS, idx, w};
        // the tiling with the fewest waves x work per CTA (ties: larger tiles, fewer CTAs)
        const int64_t k0 = fused_cost<512, 4>(T, plan.num_sms), k1 = fused_cost<512, 8>(T, plan.num_sms),
                      k2 = fused_cost<256, 8>(T, plan.num_sms);
        const cudaError_t err = (k0 <= k1 && k0 <= k2) ? launch_router_fused<512, 4>(fa, ctx, stream)
                                : (k1 <= k2)           ? launch_router_fused<512, 8>(fa, ctx, stream)
                                                       : launch_router_fused<256, 8>(fa, ctx, stream);
        if (err == cudaSuccess && between) between(stream);
        return err;
    }
    RouterLogitsArgs la{x, wr, T, H, E, plan.S, plan.nchunks, P, xn2, wn2};
    const int tt = router_tt(T);
    dim3 grid((unsigned)((T + tt - 1) / tt), (unsigned)((E + RT_TE - 1) / RT_TE), (unsigned)plan.S);
    cudaError_t err = tt == 64 ? launch_k(router_logits_kernel<4>, grid, dim3(RT_THREADS), 0, stream, la)
                               : launch_k(router_logits_kernel<1>, grid, dim3(RT_THREADS), 0, stream, la);
    if (err != cudaSuccess) return err;
    if (between) between(stream);
    RouterTopkArgs ta{P, xn2, wn2, x, wr, bias, T, H, E, K, plan.S, plan.nchunks, idx, w};
    const unsigned blocks = (unsigned)((T + TK_WARPS - 1) / TK_WARPS);
    return launch_k(router_topk_kernel, dim3(blocks), dim3(TK_WARPS * 32), 0, stream, ta, ctx);
}

}  // namespace moe
