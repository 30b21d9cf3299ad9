// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05).
//
// The two expert projections (bloomery issue page, s.2 "Checkpoint facts":
// ungated ReLU^2 experts, width 1856; s.3: ungated up/down parts) are, for
// every expert e and the rows r of its segment in the permuted layout,
//   up:    H[r, f] = relu( sum_h W_up[e][f][h] * X_perm[r][h] )^2
//   down:  Y[r, j] =       sum_f W_down[e][j][f] * H[r][f]
// with X_perm[r] = x[perm_src[r] / K].  Both are computed "swap-AB": a block of
// 128 weight rows of W[e] is the MMA's M side (TMEM lanes) and the expert's
// tokens are its N side (16..256 TMEM columns).  A decode batch has a few
// tokens per expert, so the kernel is a weight stream that the tensor cores
// consume at N = 16; a prefill chunk has ~192 tokens per expert, so every
// weight tile is read from HBM once and used for all of them.
//
// Work unit = (schedule entry {e, row0, nrows}, one 128-row weight block).
// Persistent CTAs (one per SM) walk units u = blockIdx.x + i * gridDim.x.
// Roles (192 threads):
//   warp 0      TMA producer (one thread): per 128-byte K slice the weight
//               tile (one 128-row box, or a 64-row box for the last block of
//               a 1856-row expert) and the expert's rows (128-, 64- and 16-row
//               boxes, largest first), both in the 128-byte swizzle,
//               into an NS-deep smem ring.  Few, large copies per stage: the
//               copy engine's per-request cost, not bytes, is what limits a
//               ring of many small boxes;
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma (K = 16 bf16 or
//               32 e4m3 per instruction) into one of two TMEM accumulators;
//   warps 2..5  epilogue: tcgen05.ld, scale, ReLU^2 (up) and stores; warp w
//               reads TMEM lanes 32*(w%4) .. +31.
// Every wait is bounded; on expiry the block records MOE_ETIMEOUT, drains what
// it issued and returns.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int GG_THREADS = 192;
constexpr int GG_BM = 128;                 // weight rows per unit (MMA M)
constexpr int GG_ROW_BYTES = 128;          // bytes of one operand row per stage (K extent)
constexpr int GG_A_BYTES = GG_BM * GG_ROW_BYTES;   // 16 KB
constexpr int GG_TMEM_COLS = 512;          // two accumulators of up to 256 columns

struct GemmArgs {
    const int4* sched;       // {e, row0, nrows, 0}
    const int* n_sched;      // device count of schedule entries
    int m_blocks;            // ceil(Nout / 128)
    int Nout;                // rows of one expert's weight (F for up, H for down)
    int k_stages;            // ceil(Kdim * elem / 128)
    int n_stages;            // smem ring depth
    int b_stage_bytes;       // bn_max * 128
    void* out;               // [rows][Nout], bf16 (or e4m3 codes for the fp8 up output)
    int64_t out_ld;          // elements
    const float* w_scale;    // [E] (fp8) or null
    float in_scale;          // x_scale (up) or h_scale (down), fp8 only
    float out_scale;         // h_scale for the fp8 up output
    int debug_withhold;      // 1: block 0 withholds its first load
    int e_shared;            // schedule entries with e >= e_shared are chunk e - e_shared of the shared expert
    int shared_cols;         // down: chunk j starts at column j * shared_cols of a {n * F, H, 1} map
                             // (0: chunk j is z = j of a {F, H, n} map)
};

struct GemmMaps {
    CUtensorMap a128;        // weights, 128-row box
    CUtensorMap a64;         // weights, 64-row box
    CUtensorMap b128;        // activations, 128-row box
    CUtensorMap b64;         // activations, 64-row box
    CUtensorMap b16;         // activations, 16-row box
    CUtensorMap s128;        // shared-expert weights, 128-row box: [n * F][H] (up) or 3-D (down, below)
    CUtensorMap s64;         // shared-expert weights, 64-row box
    CUtensorMap r128;        // down projection with a shared expert: the routed bank as 3-D {F, H, E}
    CUtensorMap r64;
};

// SHD: the schedule may name chunks of the shared expert (a separate
// instantiation, so the routed-only kernel carries none of that code).
template <bool FP8, bool UP, bool SHD>
__global__ void __launch_bounds__(GG_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmMaps maps, GemmArgs g, DevCtx ctx) {
    constexpr int KEL = GG_ROW_BYTES / (FP8 ? 1 : 2);   // elements of K per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NS = g.n_stages;
    uint8_t* smA = smem;
    uint8_t* smB = smA + (size_t)NS * GG_A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smB + (size_t)NS * g.b_stage_bytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + NS;
    uint64_t* tfull = bars + 2 * NS;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&maps.a128);
        tma_prefetch_desc(&maps.a64);
        tma_prefetch_desc(&maps.b128);
        tma_prefetch_desc(&maps.b64);
        tma_prefetch_desc(&maps.b16);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), GG_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();   // after the local setup: nothing above reads what an earlier kernel writes

    const int n_units = (*g.n_sched) * g.m_blocks;

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            bool withhold = g.debug_withhold && blockIdx.x == 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int4 sc = g.sched[u / g.m_blocks];
                const int mb = u % g.m_blocks;
                const bool a_full = g.Nout - mb * GG_BM > 64;
                const int n16 = (sc.z + 15) / 16;         // 16-row groups of activations
                const int n128 = n16 / 8, n64 = (n16 % 8) / 4, r16 = n16 % 4;
                const uint32_t bytes = (uint32_t)((a_full ? 128 : 64) * GG_ROW_BYTES + n16 * 16 * GG_ROW_BYTES);
                // the weight box of this unit: one map and one origin for all its K stages
                const CUtensorMap* amap = a_full ? &maps.a128 : &maps.a64;
                int ax0 = 0, ay = sc.x * g.Nout + mb * GG_BM, az = 0;
                if constexpr (SHD) {
                    const bool shd = sc.x >= g.e_shared;   // a chunk of the shared expert
                    const int a_e = shd ? sc.x - g.e_shared : sc.x;
                    if (shd) amap = a_full ? &maps.s128 : &maps.s64;
                    if constexpr (UP) {
                        ay = a_e * g.Nout + mb * GG_BM;   // rows a_e * F + mb * 128 of [n * F][H] or [E * F][H]
                    } else {
                        if (!shd) amap = a_full ? &maps.r128 : &maps.r64;
                        ay = mb * GG_BM;                  // routed: (kx, row, e); shared: (kx, row, j) or
                        az = shd && g.shared_cols ? 0 : a_e;   // (j * F + kx, row, 0)
                        ax0 = shd ? a_e * g.shared_cols : 0;
                    }
                }
                for (int ks = 0; ks < g.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_arrive_expect_tx(fb, bytes);
                    if (withhold) {
                        withhold = false;   // this stage never completes: the consumer's wait expires
                    } else {
                        const int kx = ks * KEL;
                        const uint32_t a_dst = smem_u32(smA + (size_t)stage * GG_A_BYTES);
                        const uint32_t b_dst = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
                        if constexpr (SHD && !UP)
                            tma_load_3d(a_dst, amap, fb, ax0 + kx, ay, az, pol_w);
                        else
                            tma_load_2d(a_dst, amap, fb, kx, ay, pol_w);
                        int row = 0;
                        for (int j = 0; j < n128; ++j, row += 128)
                            tma_load_2d(b_dst + row * GG_ROW_BYTES, &maps.b128, fb, kx, sc.y + row, pol_x);
                        for (int j = 0; j < n64; ++j, row += 64)
                            tma_load_2d(b_dst + row * GG_ROW_BYTES, &maps.b64, fb, kx, sc.y + row, pol_x);
                        for (int j = 0; j < r16; ++j, row += 16)
                            tma_load_2d(b_dst + row * GG_ROW_BYTES, &maps.b16, fb, kx, sc.y + row, pol_x);
                    }
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let loads already in flight land before the block exits
                const uint64_t t0 = globaltimer();
                while (globaltimer() - t0 < 200000ull) __nanosleep(1000);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            bool issued = false;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int4 sc = g.sched[u / g.m_blocks];
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = make_idesc(FP8 ? 0u : 1u, GG_BM, n_mma);
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
                    const uint32_t a_base = smem_u32(smA + (size_t)stage * GG_A_BYTES);
                    const uint32_t b_base = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        mma_ss<FP8>(d_tmem, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32), idesc,
                                    (ks | kk) != 0 ? 1u : 0u);
                    }
                    issued = true;
                    mma_commit(smem_u32(&empty[stage]));
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(smem_u32(&tfull[acc]));
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (!ok && issued) {
                // wait for every MMA issued so far before TMEM is released
                mma_commit(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else {
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
            const int4 sc = g.sched[u / g.m_blocks];
            const int mb = u % g.m_blocks;
            if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, ctx, abort_flag)) break;
            tc_fence_after();
            const int f = mb * GG_BM + q * 32 + lane;
            const bool fvalid = f < g.Nout;
            float scale = 1.0f;
            if constexpr (FP8) scale = __fmul_rn(g.w_scale[sc.x], g.in_scale);
            // E4M3 codes of the ReLU^2 tensor: a * (1 / h_scale), the reciprocal correctly rounded
            const float inv_out = (FP8 && UP) ? __frcp_rn(g.out_scale) : 1.0f;
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
            mbar_arrive(smem_u32(&tempty[acc]));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GG_TMEM_COLS);
    }
}

// ----------------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
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

// 2-D map over a row-major [rows][cols] matrix, box = 128 bytes x box_rows,
// 128-byte swizzle, out-of-range elements read as zero.
static bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, bool fp8, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int es = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * es)};
    cuuint32_t box[2] = {(cuuint32_t)(GG_ROW_BYTES / es), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D bf16 map with dims {d0, d1, d2} (d0 contiguous) and byte strides s1,
// s2 of dims 1 and 2; box = 128 bytes x box_rows x 1, 128-byte swizzle,
// out-of-range elements read as zero.
bool make_map3(CUtensorMap* m, const void* base, int64_t d0, int64_t d1, int64_t d2, int64_t s1,
               int64_t s2, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2};
    cuuint64_t strides[2] = {(cuuint64_t)s1, (cuuint64_t)s2};
    cuuint32_t box[3] = {(cuuint32_t)(GG_ROW_BYTES / 2), (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The column chunks of a row-major bf16 [rows][n * chunk] matrix as {chunk,
// rows, n}: a box never reads into the next chunk.
bool make_map_chunks(CUtensorMap* m, const void* base, int64_t rows, int64_t chunk, int64_t n,
                     int box_rows) {
    return make_map3(m, base, chunk, rows, n, n * chunk * 2, chunk * 2, box_rows);
}

GemmPlan gemm_plan(int64_t T, int K, int E) {
    GemmPlan p;
    const int64_t rows = T * K;
    int64_t per_expert_max = T < rows ? T : rows;   // an expert gets each token at most once
    int bn = (int)((per_expert_max + 15) / 16 * 16);
    // Tile height: when experts average 128 rows or more (a prefill chunk: ~192 each) a
    // 256-row tile holds nearly every expert whole, in four 48 KB stages; when they are sparse
    // (most tiles small, a few hot experts) 224-row tiles give five 44 KB stages and split
    // only the hot experts.  Measured on B200: prefill FFN 558 us at 256 against 580 at 224;
    // the skewed batch 303 us at 224 against 318 at 256.
    const int cap = rows / (E > 0 ? E : 1) >= 128 ? 256 : 224;
    if (bn > cap) bn = cap;
    if (bn < 16) bn = 16;
    p.bn = bn;
    const int stage = GG_A_BYTES + bn * GG_ROW_BYTES;
    int ns = (220 * 1024) / stage;
    if (ns > 8) ns = 8;
    if (ns < 2) ns = 2;
    p.n_stages = ns;
    p.smem_bytes = 1024 + (size_t)ns * stage + (size_t)(2 * ns + 5) * 8 + 16;
    const int64_t nonempty = E < rows ? E : rows;
    p.max_sched = (int)(nonempty + (rows + bn - 1) / bn);
    return p;
}

template <bool FP8, bool UP, bool SHD = false>
static cudaError_t launch_one(const GemmMaps& maps, const GemmArgs& g, int grid, size_t smem, const DevCtx& ctx,
                              cudaStream_t stream) {
    auto kfn = grouped_gemm_kernel<FP8, UP, SHD>;
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch_k(kfn, dim3(grid), dim3(GG_THREADS), smem, stream, maps, g, ctx);
}

// One grouped projection.  W: [E * Nout][Kdim] (bf16 or e4m3), act: [rows][Kdim]
// in the expert layout, out: [rows][Nout].  sched / n_sched: device schedule.
// Ws (n_shared > 0, bf16): the shared expert as n_shared chunks of width F,
// schedule entries E .. E + n_shared - 1 -- the up weight [n_shared * Nout][Kdim]
// (chunk j = rows j * Nout ..), the down weight [Nout][n_shared * Kdim] (chunk j =
// columns j * Kdim ..).
cudaError_t launch_grouped_gemm(bool fp8, bool up, const void* W, int E, int Nout, int Kdim, const void* act,
                                int64_t rows, const int4* sched, const int* n_sched, const GemmPlan& plan,
                                void* out, const float* w_scale, float in_scale, float out_scale, int num_sms,
                                int debug_withhold, const DevCtx& ctx, cudaStream_t stream, const void* Ws,
                                int n_shared) {
    if (rows == 0) return cudaSuccess;
    GemmMaps maps;
    if (!make_map(&maps.a128, W, (int64_t)E * Nout, Kdim, fp8, 128) ||
        !make_map(&maps.a64, W, (int64_t)E * Nout, Kdim, fp8, 64) ||
        !make_map(&maps.b128, act, rows, Kdim, fp8, 128) || !make_map(&maps.b64, act, rows, Kdim, fp8, 64) ||
        !make_map(&maps.b16, act, rows, Kdim, fp8, 16))
        return cudaErrorInvalidValue;
    int shared_cols = 0;
    maps.s128 = maps.r128 = maps.a128;   // read only by the instantiation for a shared expert
    maps.s64 = maps.r64 = maps.a64;
    if (n_shared > 0) {
        if (fp8 || !Ws) return cudaErrorInvalidValue;
        bool ok = up ? make_map(&maps.s128, Ws, (int64_t)n_shared * Nout, Kdim, false, 128) &&
                           make_map(&maps.s64, Ws, (int64_t)n_shared * Nout, Kdim, false, 64)
                     : !shared_map_2d() && make_map_chunks(&maps.s128, Ws, Nout, Kdim, n_shared, 128) &&
                           make_map_chunks(&maps.s64, Ws, Nout, Kdim, n_shared, 64);
        if (!ok && !up) {
            // a driver that refuses the chunked view: the plain [H][n * F] matrix as {n * F, H, 1},
            // chunk j from column j * F (a K tail meets activation columns that read as zero)
            shared_cols = Kdim;
            ok = make_map_chunks(&maps.s128, Ws, Nout, (int64_t)n_shared * Kdim, 1, 128) &&
                 make_map_chunks(&maps.s64, Ws, Nout, (int64_t)n_shared * Kdim, 1, 64);
        }
        // the routed bank [E][H][F] as {F, H, E}: the down kernel then issues one load form
        if (ok && !up)
            ok = make_map3(&maps.r128, W, Kdim, Nout, E, (int64_t)Kdim * 2, (int64_t)Nout * Kdim * 2, 128) &&
                 make_map3(&maps.r64, W, Kdim, Nout, E, (int64_t)Kdim * 2, (int64_t)Nout * Kdim * 2, 64);
        if (!ok) return cudaErrorInvalidValue;
    }
    GemmArgs g;
    g.sched = sched;
    g.n_sched = n_sched;
    g.m_blocks = (Nout + GG_BM - 1) / GG_BM;
    g.Nout = Nout;
    const int es = fp8 ? 1 : 2;
    g.k_stages = (int)(((int64_t)Kdim * es + GG_ROW_BYTES - 1) / GG_ROW_BYTES);
    g.n_stages = plan.n_stages;
    g.b_stage_bytes = plan.bn * GG_ROW_BYTES;
    g.out = out;
    g.out_ld = Nout;
    g.w_scale = w_scale;
    g.in_scale = in_scale;
    g.out_scale = out_scale;
    g.debug_withhold = debug_withhold;
    g.e_shared = n_shared > 0 ? E : 0x7fffffff;
    g.shared_cols = shared_cols;
    const int64_t max_units = (int64_t)plan.max_sched * g.m_blocks;
    const int grid = (int)(max_units < num_sms ? max_units : num_sms);
    if (fp8) {
        return up ? launch_one<true, true>(maps, g, grid, plan.smem_bytes, ctx, stream)
                  : launch_one<true, false>(maps, g, grid, plan.smem_bytes, ctx, stream);
    }
    if (n_shared > 0)   // bf16 only
        return up ? launch_one<false, true, true>(maps, g, grid, plan.smem_bytes, ctx, stream)
                  : launch_one<false, false, true>(maps, g, grid, plan.smem_bytes, ctx, stream);
    return up ? launch_one<false, true>(maps, g, grid, plan.smem_bytes, ctx, stream)
              : launch_one<false, false>(maps, g, grid, plan.smem_bytes, ctx, stream);
}

}  // namespace moe
