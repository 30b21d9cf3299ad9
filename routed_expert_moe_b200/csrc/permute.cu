// Token permutation into expert-contiguous rows, the GEMM tile schedule, and
// the row gather that feeds the up-projection.
//
// The grouped expert products (audio.cpp model page, "CPU weight offload")
// run on rows grouped by expert.  The grouping is a stable counting sort of
// the assignments i = t*K + k by expert: a histogram, an exclusive scan, and
// a scatter that keeps ascending i inside each expert's segment.  The sort
// is one block: at 24,576 assignments it is a few microseconds, and one
// block keeps the stable ranks free of any cross-block protocol.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int PM_THREADS = 1024;
constexpr int64_t kPermuteOneBlockMax = 4096;   // assignments sorted by the single-block kernel

// Tile schedule: expert e's segment [offsets[e], offsets[e+1]) is cut into
// near-equal blocks of at most bn rows, each a multiple of 16 rows except the
// last: per = round16(ceil(cnt / ceil(cnt / bn))), nblk = ceil(cnt / per).
// Entry {e, row0, nrows, 0}.  Called by the whole block; nb_s is shared
// scratch of E ints.  With ns > 0 the ns chunks of the shared expert follow
// as entries e = E + j over rows row0 + j * Tsh .. row0 + (j + 1) * Tsh, cut
// the same way.
__device__ __forceinline__ int sched_per(int c, int bn) {
    const int nb = (c + bn - 1) / bn;
    const int per = (c + nb - 1) / nb;
    return (per + 15) & ~15;
}

// In-place exclusive scan of v[0..n) (n <= 256) by the first 256 threads of
// the block (blockDim.x >= 256); returns the total to every thread.
__device__ int block_exclusive_scan256(int* v, int n) {
    __shared__ int warp_tot[8];
    __shared__ int total;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    int x = 0, incl = 0;
    if (tid < 256) {
        x = tid < n ? v[tid] : 0;
        incl = x;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int w = 0; w < 8; ++w) {
            const int y = warp_tot[w];
            warp_tot[w] = run;
            run += y;
        }
        total = run;
    }
    __syncthreads();
    if (tid < n) v[tid] = warp_tot[warp] + incl - x;
    __syncthreads();
    return total;
}

__device__ void build_schedule(const int* seg_off, int E, int bn, int* nb_s, int4* sched,
                               int* n_sched, int ns, int Tsh, int row0) {
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) {
        const int c = seg_off[e + 1] - seg_off[e];
        nb_s[e] = c > 0 ? (c + sched_per(c, bn) - 1) / sched_per(c, bn) : 0;
    }
    __syncthreads();
    const int total = block_exclusive_scan256(nb_s, E);
    const int pers = ns > 0 && Tsh > 0 ? sched_per(Tsh, bn) : 16;
    const int nbs = ns > 0 && Tsh > 0 ? (Tsh + pers - 1) / pers : 0;
    if (tid == 0) *n_sched = total + ns * nbs;
    for (int q = tid; q < ns * nbs; q += blockDim.x) {
        const int j = q / nbs, r0 = (q % nbs) * pers;
        sched[total + q] = make_int4(E + j, row0 + j * Tsh + r0, min(pers, Tsh - r0), 0);
    }
    for (int e = tid; e < E; e += blockDim.x) {
        const int off = seg_off[e], c = seg_off[e + 1] - off;
        if (c <= 0) continue;
        const int per = sched_per(c, bn);
        for (int r0 = 0, b = 0; r0 < c; r0 += per, ++b)
            sched[nb_s[e] + b] = make_int4(e, off + r0, min(per, c - r0), 0);
    }
}

struct PermuteArgs {
    const int32_t* idx;
    int64_t n;       // T*K
    int E;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm_src;
    int32_t* inv_row;
    int4* sched;     // may be null
    int* n_sched;
    int bn;
    int ns;          // shared-expert chunks in the schedule (rows n + j * (n / K) ..)
    int K;
};

// NT threads (a power of two, 256..1024): the fewest warps that hold the assignments, so that
// the per-warp count table and its column scans stay short for small batches.
template <int NT>
__global__ void __launch_bounds__(NT) permute_kernel(PermuteArgs a, DevCtx ctx) {
    constexpr int NW = NT / 32;
    pdl_enter();
    extern __shared__ int sm[];
    const int E = a.E;
    int* hist = sm;               // [E]
    int* base = hist + E;         // [E] next free row of each expert
    int* tot = base + E;          // [E] chunk totals
    int* offs = tot + E;          // [E+1]
    int* wtab = offs + E + 1;     // [NW][E] per-warp counts of the chunk
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const uint32_t lt_mask = (1u << lane) - 1u;

    for (int e = tid; e < E; e += NT) hist[e] = 0;
    __syncthreads();
    int bad = 0;
    for (int64_t i = tid; i < a.n; i += NT) {
        const int e = a.idx[i];
        if (e < 0 || e >= E) {
            bad = 1;
            continue;
        }
        atomicAdd(&hist[e], 1);
    }
    if (__syncthreads_or(bad)) {
        if (tid == 0) record_error(ctx.err, MOE_EINDEX);
    }
    for (int e = tid; e < E; e += NT) offs[e] = hist[e];
    __syncthreads();
    const int total = block_exclusive_scan256(offs, E);
    for (int e = tid; e < E; e += NT) {
        base[e] = offs[e];
        a.offsets[e] = offs[e];
        a.counts[e] = hist[e];
    }
    if (tid == 0) {
        offs[E] = total;
        a.offsets[E] = total;
    }
    __syncthreads();

    for (int64_t c0 = 0; c0 < a.n; c0 += NT) {
        const int64_t i = c0 + tid;
        int e = i < a.n ? a.idx[i] : -1;
        if (e >= E) e = -1;
        for (int q = tid; q < NW * E; q += NT) wtab[q] = 0;
        __syncthreads();
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int rank_w = __popc(peers & lt_mask);
        if (e >= 0 && rank_w == 0) wtab[warp * E + e] = __popc(peers);
        __syncthreads();
        for (int ex = tid; ex < E; ex += NT) {
            int run = 0;
            for (int w = 0; w < NW; ++w) {
                const int v = wtab[w * E + ex];
                wtab[w * E + ex] = run;
                run += v;
            }
            tot[ex] = run;
        }
        __syncthreads();
        if (e >= 0) {
            const int r = base[e] + wtab[warp * E + e] + rank_w;
            a.perm_src[r] = (int32_t)i;
            a.inv_row[i] = r;
        }
        __syncthreads();
        for (int ex = tid; ex < E; ex += NT) base[ex] += tot[ex];
        __syncthreads();
    }
    if (a.sched) build_schedule(offs, E, a.bn, hist, a.sched, a.n_sched, a.ns, (int)(a.n / a.K), (int)a.n);
}

// ---- multi-block permutation for large batches: one chunk of PM_THREADS
// assignments per block; the stable rank inside a chunk is computed exactly
// as in the single-block kernel, and chunks are ordered by their index.

__global__ void __launch_bounds__(PM_THREADS) perm_hist_kernel(const int32_t* __restrict__ idx, int64_t n, int E,
                                                               int* __restrict__ bcount, DevCtx ctx) {
    pdl_enter();
    __shared__ int hist[256];
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += PM_THREADS) hist[e] = 0;
    __syncthreads();
    const int64_t i = (int64_t)blockIdx.x * PM_THREADS + tid;
    int bad = 0;
    if (i < n) {
        const int e = idx[i];
        if (e < 0 || e >= E)
            bad = 1;
        else
            atomicAdd(&hist[e], 1);
    }
    if (__syncthreads_or(bad) && tid == 0) record_error(ctx.err, MOE_EINDEX);
    for (int e = tid; e < E; e += PM_THREADS) bcount[(int64_t)blockIdx.x * E + e] = hist[e];
}

// counts, offsets, per-(chunk, expert) bases, and the GEMM schedule
__global__ void __launch_bounds__(256) perm_scan_kernel(const int* __restrict__ bcount, int G, int E,
                                                        int* __restrict__ bbase, int32_t* counts,
                                                        int32_t* offsets, int4* sched, int* n_sched, int bn,
                                                        int ns, int Tsh, int row0) {
    pdl_enter();
    __shared__ int offs[257];
    __shared__ int nb[256];
    const int tid = threadIdx.x;
    int tot = 0;
    if (tid < E)
        for (int b = 0; b < G; ++b) tot += bcount[(int64_t)b * E + tid];
    if (tid < E) offs[tid] = tot;
    __syncthreads();
    const int total = block_exclusive_scan256(offs, E);
    if (tid == 0) {
        offs[E] = total;
        offsets[E] = total;
    }
    if (tid < E) {
        counts[tid] = tot;
        offsets[tid] = offs[tid];
        int run = offs[tid];
        for (int b = 0; b < G; ++b) {
            bbase[(int64_t)b * E + tid] = run;
            run += bcount[(int64_t)b * E + tid];
        }
    }
    __syncthreads();
    if (sched) build_schedule(offs, E, bn, nb, sched, n_sched, ns, Tsh, row0);
}

__global__ void __launch_bounds__(PM_THREADS) perm_scatter_kernel(const int32_t* __restrict__ idx, int64_t n,
                                                                  int E, const int* __restrict__ bbase,
                                                                  int32_t* __restrict__ perm_src,
                                                                  int32_t* __restrict__ inv_row) {
    pdl_enter();
    extern __shared__ int wtab[];   // [32][E]
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int64_t i = (int64_t)blockIdx.x * PM_THREADS + tid;
    int e = i < n ? idx[i] : -1;
    if (e >= E) e = -1;
    for (int q = tid; q < 32 * E; q += PM_THREADS) wtab[q] = 0;
    __syncthreads();
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int rank_w = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank_w == 0) wtab[warp * E + e] = __popc(peers);
    __syncthreads();
    for (int ex = tid; ex < E; ex += PM_THREADS) {
        int run = bbase[(int64_t)blockIdx.x * E + ex];
        for (int w = 0; w < 32; ++w) {
            const int v = wtab[w * E + ex];
            wtab[w * E + ex] = run;
            run += v;
        }
    }
    __syncthreads();
    if (e >= 0) {
        const int r = wtab[warp * E + e] + rank_w;
        perm_src[r] = (int32_t)i;
        inv_row[i] = r;
    }
}

__global__ void schedule_kernel(const int32_t* offsets, int E, int bn, int4* sched, int* n_sched, int ns,
                                int Tsh, int row0) {
    pdl_enter();
    __shared__ int offs[257];
    __shared__ int nb[256];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) offs[e] = offsets[e];
    __syncthreads();
    build_schedule(offs, E, bn, nb, sched, n_sched, ns, Tsh, row0);
}

// x / s rounded to nearest from y = RN(1/s): q = RN(x y), r = x - s q (exact,
// one FMA), q' = RN(q + r y) -- Markstein's correction of a reciprocal
// quotient (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  Zeros and
// non-finite q are returned as they are (the correction would lose the sign
// of a zero or turn an overflow into NaN).  The library's tests compare the
// E4M3 codes this produces with those of a correctly rounded division for
// every bf16 input at the scales in use.
__device__ __forceinline__ float div_by_scale(float x, float s, float y) {
    const float q = __fmul_rn(x, y);
    if (q == 0.0f || !isfinite(q)) return q;
    const float r = __fmaf_rn(-q, s, x);
    return __fmaf_rn(r, y, q);
}

// xp[r] = x[perm_src[r] / K], or its E4M3 codes e4m3(x / x_scale) (fp8);
// with perm_src == null the rows are taken in order (xp[r] = x[r]).  Rows
// r >= routed_rows are the shared expert's: xp[r] = x[(r - routed_rows) % T].  One
// warp per row, four 16-byte loads per lane in flight before their stores.
__global__ void gather_rows_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm_src,
                                   int64_t rows, int64_t routed_rows, int K, int64_t T, int H,
                                   void* __restrict__ xp, int fp8, float x_scale, int* zero, int64_t n_zero,
                                   DevCtx ctx) {
    pdl_enter();
    // counters of the kernel that follows (the one-launch FFN), zero before it starts
    // (zero is 16-byte aligned: whole int4s, then the tail)
    {
        const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, step = (int64_t)gridDim.x * blockDim.x;
        for (int64_t i = i0; i < n_zero / 4; i += step) reinterpret_cast<int4*>(zero)[i] = make_int4(0, 0, 0, 0);
        for (int64_t i = (n_zero & ~int64_t(3)) + i0; i < n_zero; i += step) zero[i] = 0;
    }
    constexpr int B = 4;
    const int lane = threadIdx.x % 32;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    const int nv = H / 8;
    const float y = fp8 ? __frcp_rn(x_scale) : 1.0f;
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
        int64_t t = r;
        if (r >= routed_rows) {
            t = (r - routed_rows) % T;
        } else if (perm_src) {
            const int32_t src = perm_src[r];
            t = src / K;
            if (src < 0 || t >= T) {
                if (lane == 0) record_error(ctx.err, MOE_EINDEX);
                continue;
            }
        }
        const uint4* xr = reinterpret_cast<const uint4*>(x + t * H);
        for (int v0 = lane; v0 < nv; v0 += 32 * B) {
            uint4 q[B];
#pragma unroll
            for (int i = 0; i < B; ++i)
                if (v0 + 32 * i < nv) q[i] = xr[v0 + 32 * i];
            if (!fp8) {
                uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(xp) + r * H);
#pragma unroll
                for (int i = 0; i < B; ++i)
                    if (v0 + 32 * i < nv) out[v0 + 32 * i] = q[i];
            } else {
                uint2* out = reinterpret_cast<uint2*>(static_cast<uint8_t*>(xp) + r * H);
#pragma unroll
                for (int i = 0; i < B; ++i) {
                    if (v0 + 32 * i >= nv) continue;
                    const uint32_t wv[4] = {q[i].x, q[i].y, q[i].z, q[i].w};
                    uint32_t packed[2] = {0, 0};
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t bits = (j & 1) ? (wv[j / 2] & 0xFFFF0000u) : (wv[j / 2] << 16);
                        const float f = div_by_scale(__uint_as_float(bits), x_scale, y);
                        const uint32_t c = __nv_cvt_float_to_fp8(f, __NV_SATFINITE, __NV_E4M3);
                        packed[j / 4] |= c << (8 * (j % 4));
                    }
                    out[v0 + 32 * i] = make_uint2(packed[0], packed[1]);
                }
            }
        }
    }
}

// ----------------------------------------------------------------------------- host

size_t permute_smem_bytes(int E) { return (size_t)(4 * E + 1 + 32 * E) * sizeof(int); }

// Scratch ints the multi-block path needs (0 when the single-block kernel runs).
size_t permute_scratch_ints(int64_t n, int E) {
    if (n <= kPermuteOneBlockMax) return 0;
    const int64_t G = (n + PM_THREADS - 1) / PM_THREADS;
    return (size_t)(2 * G * E);
}

cudaError_t launch_permute(const int32_t* idx, int64_t n, int K, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm_src, int32_t* inv_row, int4* sched, int* n_sched, int bn, int ns,
                           int* scratch, const DevCtx& ctx, cudaStream_t stream) {
    if (n <= kPermuteOneBlockMax) {
        PermuteArgs a{idx, n, E, counts, offsets, perm_src, inv_row, sched, n_sched, bn, ns, K};
        if (n <= 256) return launch_k(permute_kernel<256>, dim3(1), dim3(256), permute_smem_bytes(E), stream, a, ctx);
        if (n <= 512) return launch_k(permute_kernel<512>, dim3(1), dim3(512), permute_smem_bytes(E), stream, a, ctx);
        return launch_k(permute_kernel<1024>, dim3(1), dim3(1024), permute_smem_bytes(E), stream, a, ctx);
    }
    if (!scratch) return cudaErrorInvalidValue;
    const int G = (int)((n + PM_THREADS - 1) / PM_THREADS);
    int* bcount = scratch;
    int* bbase = scratch + (size_t)G * E;
    cudaError_t err = launch_k(perm_hist_kernel, dim3(G), dim3(PM_THREADS), 0, stream, idx, n, E, bcount, ctx);
    if (err != cudaSuccess) return err;
    err = launch_k(perm_scan_kernel, dim3(1), dim3(256), 0, stream, bcount, G, E, bbase, counts, offsets, sched,
                   n_sched, bn, ns, (int)(n / K), (int)n);
    if (err != cudaSuccess) return err;
    return launch_k(perm_scatter_kernel, dim3(G), dim3(PM_THREADS), (size_t)32 * E * sizeof(int), stream, idx, n,
                    E, bbase, perm_src, inv_row);
}

cudaError_t launch_schedule(const int32_t* offsets, int E, int bn, int4* sched, int* n_sched, int ns, int64_t T,
                            int K, cudaStream_t stream) {
    return launch_k(schedule_kernel, dim3(1), dim3(256), 0, stream, offsets, E, bn, sched, n_sched, ns, (int)T,
                    (int)(T * K));
}

cudaError_t launch_gather(const uint16_t* x, const int32_t* perm_src, int64_t rows, int64_t routed_rows, int K,
                          int64_t T, int H, void* xp, bool fp8, float x_scale, int num_sms, const DevCtx& ctx,
                          cudaStream_t stream, int* zero, int64_t n_zero) {
    if (rows == 0) return cudaSuccess;
    int64_t blocks = (rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    return launch_k(gather_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, x, perm_src, rows, routed_rows,
                    K, T, H, xp, fp8 ? 1 : 0, x_scale, zero, n_zero, ctx);
}

// ----------------------------------------------------------------------------- expert-parallel regrouping

// Rows received by an expert's owner arrive source-major: for each source rank p,
// its rows for local expert 0, then 1, ... (each block in the source's order).  The
// grouped layout the expert FFN reads is expert-major, then source, then arrival
// order.  One block: thread 0 builds the small prefix tables (W * E_loc <= 256
// entries), then every thread places rows i, i + blockDim.x, ...:
//   received row i = (source p, local expert e, j-th of that block)
//   grouped row     = off[e] + before[p][e] + j
// with off[e] = rows of experts < e (all sources) and before[p][e] = rows of
// expert e from sources < p.  perm[grouped] = i and inv[i] = grouped.
constexpr int RG_THREADS = 512;
constexpr int RG_MAX_ENTRIES = 256;

__global__ void __launch_bounds__(RG_THREADS) ep_regroup_kernel(const int64_t* __restrict__ rc, int W, int E_loc,
                                                                int64_t R, int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                                                DevCtx ctx) {
    pdl_enter();
    __shared__ int64_t src_base[RG_MAX_ENTRIES + 1];               // [W + 1]
    __shared__ int64_t within[RG_MAX_ENTRIES + RG_MAX_ENTRIES];    // [W][E_loc + 1]
    __shared__ int64_t before[RG_MAX_ENTRIES];                     // [W][E_loc]
    __shared__ int64_t off[RG_MAX_ENTRIES + 1];                    // [E_loc + 1]
    __shared__ int bad;
    if (threadIdx.x == 0) {
        bad = 0;
        int64_t total = 0;
        for (int p = 0; p < W; ++p) {
            src_base[p] = total;
            int64_t w = 0;
            within[p * (E_loc + 1)] = 0;
            for (int e = 0; e < E_loc; ++e) {
                const int64_t c = rc[(int64_t)p * E_loc + e];
                if (c < 0) bad = 1;
                w += c;
                within[p * (E_loc + 1) + e + 1] = w;
            }
            total += w;
        }
        src_base[W] = total;
        if (total != R) bad = 1;
        int64_t o = 0;
        for (int e = 0; e < E_loc; ++e) {
            off[e] = o;
            int64_t b = 0;
            for (int p = 0; p < W; ++p) {
                before[p * E_loc + e] = b;
                b += rc[(int64_t)p * E_loc + e];
            }
            o += b;
        }
        off[E_loc] = o;
        if (bad) record_error(ctx.err, MOE_EINDEX);
        for (int e = 0; e <= E_loc && !bad; ++e) offsets[e] = (int32_t)off[e];
    }
    __syncthreads();
    if (bad) return;
    for (int64_t i = threadIdx.x; i < R; i += blockDim.x) {
        int lo = 0, hi = W;                      // last p with src_base[p] <= i
        while (hi - lo > 1) {
            const int mid = (lo + hi) / 2;
            if (src_base[mid] <= i) lo = mid; else hi = mid;
        }
        const int p = lo;
        const int64_t local = i - src_base[p];
        const int64_t* wp = within + p * (E_loc + 1);
        int a = 0, b = E_loc;                    // last e with wp[e] <= local (wp[E_loc] > local)
        while (b - a > 1) {
            const int mid = (a + b) / 2;
            if (wp[mid] <= local) a = mid; else b = mid;
        }
        const int e = a;
        const int64_t pos = off[e] + before[p * E_loc + e] + (local - wp[e]);
        perm[pos] = (int32_t)i;
        inv[i] = (int32_t)pos;
    }
}

cudaError_t launch_ep_regroup(const int64_t* recv_counts, int W, int E_loc, int64_t R, int32_t* offsets,
                              int32_t* perm, int32_t* inv, const DevCtx& ctx, cudaStream_t stream) {
    if (W < 1 || E_loc < 1 || (int64_t)W * E_loc > RG_MAX_ENTRIES) return cudaErrorInvalidValue;
    return launch_k(ep_regroup_kernel, dim3(1), dim3(RG_THREADS), 0, stream, recv_counts, W, E_loc, R, offsets, perm,
                    inv, ctx);
}

}  // namespace moe
