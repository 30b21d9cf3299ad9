// Grouped expert GEMM on CTA pairs (tcgen05.mma.cta_group::2) for batches
// with many rows per expert (prefill chunks).
//
// Same products as grouped_gemm.cu (bloomery issue page, s.2 "Checkpoint
// facts" and s.3: ungated ReLU^2 experts with up/down parts), same swap-AB
// orientation, but one MMA covers 256 weight rows: each CTA of a 2-CTA
// cluster holds 128 of them and HALF of the expert's token rows, and the
// pair's tensor cores multiply the full 256 x N product, each CTA keeping its
// 128 x N accumulator in its own TMEM.  Every activation tile is therefore
// read once per 256 weight rows instead of once per 128, and each SM's ring
// stage is 16 KB of weights + N/2 rows of activations, which keeps the ring
// six stages deep at N = 256.
//
// Protocol per stage:
//   both producers   wait their own `empty` slot, then load their weight rows
//                    and their half of the token rows into their own smem,
//                    completing on the LEADER's `full` barrier;
//   leader producer  also arms that barrier with the bytes of both halves;
//   leader MMA       waits `full`, issues 4 MMAs (K = 16 bf16 / 32 e4m3), and
//                    commits to `empty` of both CTAs (multicast commit);
//   after a unit     it commits to `tfull` of both CTAs; both epilogues read
//                    their own TMEM and release the accumulator on the
//                    leader's `tempty` (the peer's warps arrive remotely).
// All loads are plain (non-multicast) tensor copies.  Every wait is bounded.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int P2_THREADS = 192;
constexpr int P2_BM = 128;                  // weight rows per CTA (256 per pair)
constexpr int P2_ROW_BYTES = 128;
constexpr int P2_A_BYTES = P2_BM * P2_ROW_BYTES;
constexpr int P2_TMEM_COLS = 512;

struct Gemm2Args {
    const int4* sched;
    const int* n_sched;
    int m_pairs;             // ceil(Nout / 256)
    int Nout;
    int k_stages;
    int n_stages;
    int b_stage_bytes;       // (bn_max / 2) * 128
    void* out;
    int64_t out_ld;
    const float* w_scale;
    float in_scale;
    float out_scale;
};

struct Gemm2Maps {
    CUtensorMap a128, a64;
    CUtensorMap b128, b64, b16, b8;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cluster address of the same shared location in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// tensor copy into this CTA's smem that completes on a barrier of the pair
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar_cluster, int x,
                                                 int y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

template <bool FP8>
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    if constexpr (FP8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
            "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
    }
}

// arrive on the barrier at this smem offset in both CTAs of the pair once the
// issuing thread's MMAs are complete
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}"
        ::"r"(bar)
        : "memory");
}

// arrive on a barrier of this CTA once the issuing thread's pair MMAs are complete
__device__ __forceinline__ void mma_commit_pair_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t holder_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// weight rows this CTA loads for unit pair `mp`: 0, 64 or 128
__device__ __forceinline__ int pair_a_rows(int Nout, int mp, int rank) {
    const int valid = Nout - (mp * 2 + rank) * P2_BM;
    return valid <= 0 ? 0 : (valid <= 64 ? 64 : 128);
}

template <bool FP8, bool UP>
__global__ void __launch_bounds__(P2_THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ Gemm2Maps maps, Gemm2Args g, DevCtx ctx) {
    constexpr int KEL = P2_ROW_BYTES / (FP8 ? 1 : 2);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NS = g.n_stages;
    uint8_t* smA = smem;
    uint8_t* smB = smA + (size_t)NS * P2_A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smB + (size_t)NS * g.b_stage_bytes);
    uint64_t* full = bars;            // leader only
    uint64_t* empty = bars + NS;      // both
    uint64_t* tfull = bars + 2 * NS;  // both
    uint64_t* tempty = tfull + 2;     // leader only: 4 epilogue warps x 2 CTAs
    uint64_t* drain = tempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x / 2, n_pairs = gridDim.x / 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 8);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&maps.a128);
        tma_prefetch_desc(&maps.b128);
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(tmem_holder), P2_TMEM_COLS);
    tc_fence_before();
    cluster_sync();   // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();   // after the local setup: nothing above reads what an earlier kernel writes

    const int n_units = (*g.n_sched) * g.m_pairs;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = pair; u < n_units && ok; u += n_pairs) {
                const int4 sc = g.sched[u / g.m_pairs];
                const int mp = u % g.m_pairs;
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const int half = n_mma / 2;                       // multiple of 8
                const int n8 = half / 8;
                const int n128 = n8 / 16, n64 = (n8 % 16) / 8, n16 = (n8 % 8) / 2, r8 = n8 % 2;
                const int a_mine = pair_a_rows(g.Nout, mp, (int)rank);
                const int a_total = pair_a_rows(g.Nout, mp, 0) + pair_a_rows(g.Nout, mp, 1);
                const uint32_t bytes_total = (uint32_t)((a_total + n_mma) * P2_ROW_BYTES);
                const int a_y = sc.x * g.Nout + (mp * 2 + (int)rank) * P2_BM;
                const int b_y = sc.y + (int)rank * half;
                for (int ks = 0; ks < g.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb_local = smem_u32(&full[stage]);
                    if (rank == 0) mbar_arrive_expect_tx(fb_local, bytes_total);
                    const uint32_t fb = map_to_rank(fb_local, 0);
                    const int kx = ks * KEL;
                    const uint32_t a_dst = smem_u32(smA + (size_t)stage * P2_A_BYTES);
                    const uint32_t b_dst = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
                    if (a_mine) tma_load_2d_pair(a_dst, a_mine == 128 ? &maps.a128 : &maps.a64, fb, kx, a_y, pol_w);
                    int row = 0;
                    for (int j = 0; j < n128; ++j, row += 128)
                        tma_load_2d_pair(b_dst + row * P2_ROW_BYTES, &maps.b128, fb, kx, b_y + row, pol_x);
                    for (int j = 0; j < n64; ++j, row += 64)
                        tma_load_2d_pair(b_dst + row * P2_ROW_BYTES, &maps.b64, fb, kx, b_y + row, pol_x);
                    for (int j = 0; j < n16; ++j, row += 16)
                        tma_load_2d_pair(b_dst + row * P2_ROW_BYTES, &maps.b16, fb, kx, b_y + row, pol_x);
                    for (int j = 0; j < r8; ++j, row += 8)
                        tma_load_2d_pair(b_dst + row * P2_ROW_BYTES, &maps.b8, fb, kx, b_y + row, pol_x);
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                const uint64_t t0 = globaltimer();
                while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            bool issued = false;
            for (int u = pair; u < n_units && ok; u += n_pairs) {
                const int4 sc = g.sched[u / g.m_pairs];
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = make_idesc(FP8 ? 0u : 1u, 2 * P2_BM, n_mma);
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
                for (int ks = 0; ks < g.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&full[stage]), phase, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smA + (size_t)stage * P2_A_BYTES);
                    const uint32_t b_base = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_pair<FP8>(d_tmem, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32), idesc,
                                      (ks | kk) != 0 ? 1u : 0u);
                    issued = true;
                    mma_commit_pair(smem_u32(&empty[stage]));
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(smem_u32(&tfull[acc]));
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (!ok && issued) {
                mma_commit_pair_local(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else {
        const int q = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        const float inv_out = (FP8 && UP) ? __frcp_rn(g.out_scale) : 1.0f;
        for (int u = pair; u < n_units; u += n_pairs) {
            const int4 sc = g.sched[u / g.m_pairs];
            const int mp = u % g.m_pairs;
            if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, ctx, abort_flag)) break;
            tc_fence_after();
            const int f = (mp * 2 + (int)rank) * P2_BM + q * 32 + lane;
            const bool fvalid = f < g.Nout;
            float scale = 1.0f;
            if constexpr (FP8) scale = __fmul_rn(g.w_scale[sc.x], g.in_scale);
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
            const int nchunks = (sc.z + 15) / 16;
            for (int c = 0; c < nchunks; ++c) {
                uint32_t v[16];
                tmem_ld16(t_row + (uint32_t)(c * 16), v);
                if (fvalid) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int r = c * 16 + j;
                        if (r < sc.z) {
                            float z = __uint_as_float(v[j]);
                            if constexpr (FP8) z = __fmul_rn(z, scale);
                            const int64_t o = (int64_t)(sc.y + r) * g.out_ld + f;
                            if constexpr (UP) {
                                const float a = z > 0.0f ? __fmul_rn(z, z) : 0.0f;
                                if constexpr (FP8) {
                                    static_cast<uint8_t*>(g.out)[o] = (uint8_t)__nv_cvt_float_to_fp8(
                                        __fmul_rn(a, inv_out), __NV_SATFINITE, __NV_E4M3);
                                } else {
                                    static_cast<__nv_bfloat16*>(g.out)[o] = __float2bfloat16_rn(a);
                                }
                            } else {
                                static_cast<__nv_bfloat16*>(g.out)[o] = __float2bfloat16_rn(z);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(&tempty[acc]), 0));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();   // no barrier of either CTA is used after this point
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, P2_TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode2_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

static bool make_map2(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, bool fp8, int box_rows) {
    EncodeTiledFn fn = encode2_fn();
    if (!fn) return false;
    const int es = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * es)};
    cuuint32_t box[2] = {(cuuint32_t)(P2_ROW_BYTES / es), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool FP8, bool UP>
static cudaError_t launch_pair(const Gemm2Maps& maps, const Gemm2Args& g, int64_t max_units, int num_sms, size_t smem,
                        const DevCtx& ctx, cudaStream_t stream) {
    auto kfn = grouped_gemm_pair_kernel<FP8, UP>;
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(P2_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    // every pair must be resident at once (the kernel is persistent)
    int max_clusters = 0;
    cfg.gridDim = dim3(2 * (unsigned)(num_sms / 2));
    if (cudaOccupancyMaxActiveClusters(&max_clusters, kfn, &cfg) != cudaSuccess || max_clusters < 1)
        max_clusters = num_sms / 2;
    int64_t pairs = max_units < max_clusters ? max_units : max_clusters;
    if (pairs < 1) pairs = 1;
    cfg.gridDim = dim3(2 * (unsigned)pairs);
    return cudaLaunchKernelEx(&cfg, kfn, maps, g, ctx);
}

}  // namespace

// Stage bytes and ring depth of the pair kernel for token blocks of up to bn rows.
static size_t gemm_pair_smem(int bn, int* n_stages) {
    const int stage = P2_A_BYTES + (bn / 2) * P2_ROW_BYTES;
    int ns = (200 * 1024) / stage;
    if (ns > 8) ns = 8;
    if (ns < 2) ns = 2;
    *n_stages = ns;
    return 1024 + (size_t)ns * stage + (size_t)(2 * ns + 5) * 8 + 16;
}

// One grouped projection on CTA pairs (see grouped_gemm.cu for the operands).
cudaError_t launch_grouped_gemm_pair(bool fp8, bool up, const void* W, int E, int Nout, int Kdim, const void* act,
                                     int64_t rows, const int4* sched, const int* n_sched, int bn, int max_sched,
                                     void* out, const float* w_scale, float in_scale, float out_scale,
                                     int num_sms, const DevCtx& ctx, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    Gemm2Maps maps;
    if (!make_map2(&maps.a128, W, (int64_t)E * Nout, Kdim, fp8, 128) ||
        !make_map2(&maps.a64, W, (int64_t)E * Nout, Kdim, fp8, 64) ||
        !make_map2(&maps.b128, act, rows, Kdim, fp8, 128) || !make_map2(&maps.b64, act, rows, Kdim, fp8, 64) ||
        !make_map2(&maps.b16, act, rows, Kdim, fp8, 16) || !make_map2(&maps.b8, act, rows, Kdim, fp8, 8))
        return cudaErrorInvalidValue;
    Gemm2Args g;
    g.sched = sched;
    g.n_sched = n_sched;
    g.m_pairs = (Nout + 2 * P2_BM - 1) / (2 * P2_BM);
    g.Nout = Nout;
    const int es = fp8 ? 1 : 2;
    g.k_stages = (int)(((int64_t)Kdim * es + P2_ROW_BYTES - 1) / P2_ROW_BYTES);
    const size_t smem = gemm_pair_smem(bn, &g.n_stages);
    g.b_stage_bytes = (bn / 2) * P2_ROW_BYTES;
    g.out = out;
    g.out_ld = Nout;
    g.w_scale = w_scale;
    g.in_scale = in_scale;
    g.out_scale = out_scale;
    const int64_t max_units = (int64_t)max_sched * g.m_pairs;
    if (fp8)
        return up ? launch_pair<true, true>(maps, g, max_units, num_sms, smem, ctx, stream)
                  : launch_pair<true, false>(maps, g, max_units, num_sms, smem, ctx, stream);
    return up ? launch_pair<false, true>(maps, g, max_units, num_sms, smem, ctx, stream)
              : launch_pair<false, false>(maps, g, max_units, num_sms, smem, ctx, stream);
}

}  // namespace moe
