// Both expert projections in one persistent launch (bf16 or E4M3 experts, no
// shared expert): the up projection's units, then the down projection's, in
// one list from which the CTAs claim units in order.
//
// The products are those of grouped_gemm.cu (bloomery issue page, s.2
// "Checkpoint facts" and s.3: ungated ReLU^2 experts with up/down parts):
//   up:    H[r, f] = relu( sum_h W_up[e][f][h] * X_perm[r][h] )^2
//   down:  Y[r, j] =       sum_f W_down[e][j][f] * H[r][f]
// with the same swap-AB units, TMA ring, TMEM accumulators and epilogue.
// What changes is the boundary between the two: a down unit of schedule entry
// s reads the rows of H that the up units of s write, so instead of a kernel
// boundary (every down unit waits for every up unit, and the last up wave
// leaves SMs idle), the producer of a down unit waits only for entry s:
//   up epilogue   each of the four epilogue warps stores its rows of H, every
//                 lane fences its stores for the async proxy, the warp
//                 synchronises, and lane 0 adds 1 to done[s] with release
//                 semantics (cumulative over the warp's stores);
//   down producer spins (bounded) on an acquire load of done[s] until it
//                 reaches 4 * m_up, fences the async proxy, then issues the
//                 TMA loads of H.
// Claiming: each CTA's producer takes the next unit of the list from a global
// counter (one relaxed atomic add per unit, issued while the previous unit
// loads) and passes it to the MMA thread and the epilogue warps through a
// small queue in shared memory (FF_UQ slots, each with a full and an empty
// mbarrier).  A CTA that runs ahead simply claims more units, so the CTAs end
// within about one unit of each other (a fixed round-robin left the last CTA
// 16 us behind the median at decode).
// Deadlock freedom: units are claimed in list order, so every up unit is
// claimed, by a running CTA, before any down unit is, and a CTA processes its
// units in claim order; the up units a down unit waits for therefore belong to
// running CTAs that finish them without waiting on anything but their own
// pipeline (no CTA needs to be resident for another to progress).  done[] and
// the claim counter are zeroed by the row gather that precedes this kernel on
// the stream.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int FF_THREADS = 192;
constexpr int FF_BM = 128;
constexpr int FF_ROW_BYTES = 128;
constexpr int FF_A_BYTES = FF_BM * FF_ROW_BYTES;
constexpr int FF_EPI_WARPS = 4;
constexpr int FF_UQ = 4;   // unit queue slots (producer -> MMA and epilogue warps)

// TMEM layout: two accumulators of ACC token columns.  Tiles of up to 256 rows take all 512
// columns and one CTA per SM with a ring of up to 220 KB; tiles of up to 128 rows (decode, and
// sparse batches whose experts average fewer rows) take 256 columns, a ring of up to 100 KB and
// two CTAs per SM, whose two in-order streams of TMA stages keep more bytes landing than one
// deeper ring (decode FFN 354 -> 350 us, skewed T=576 batch 292 -> 283 us).
template <bool SMALL>
struct FfnTmem {
    static constexpr int COLS = SMALL ? 256 : 512;
    static constexpr int ACC = SMALL ? 128 : 256;
    static constexpr int CTAS = SMALL ? 2 : 1;
    static constexpr int RING = SMALL ? 100 * 1024 : 220 * 1024;
};

static_assert(FfnTmem<true>::ACC == kFfnSparseRows, "sparse batches' tiles fit the two-CTA layout");

struct FfnArgs {
    int* claim;             // unit counter (zero at launch; right after done[]): producers claim units
    const int4* sched;      // {e, row0, nrows, 0}
    const int* n_sched;
    int* done;              // [max_sched] up epilogue warps finished per entry (zero at launch)
    int m_up, m_down;       // 128-row blocks of F and of H
    int F, H;
    int k_up, k_down;       // 128-byte K stages of H and of F
    int n_stages;
    int b_stage_bytes;
    void* hb;               // up output [rows][F] (bf16, or E4M3 codes)
    void* y;                // down output [rows][H] bf16
    const float* su;        // [E] E4M3 weight scales (null for bf16)
    const float* sd;
    float x_scale, h_scale;
    int debug_hold;         // 1: the list's first up unit never reports its rows (a wait must expire)
    int e_shared;           // entries with e >= e_shared are chunk e - e_shared of the shared expert (bf16)
    int shared_cols;        // shared down weight through the 2-D fallback: chunk j from column j * F
};

struct FfnMaps {
    CUtensorMap ua128, ua64;          // W_up [E * F][H]
    CUtensorMap ub128, ub64, ub16;    // X_perm [rows][H]
    CUtensorMap da128, da64;          // W_down [E * H][F]
    CUtensorMap db128, db64, db16;    // H [rows][F]
    CUtensorMap us128, us64;          // shared expert's up weight [n * F][H]
    CUtensorMap ds128, ds64;          // shared expert's down weight [H][n * F] as {F, H, n} (or {n F, H, 1})
};

// SHD: the schedule may name chunks of the shared expert (a separate instantiation, so that the
// routed-only kernel's producer keeps its per-stage path: the prefill FFN is bound by its ingest).
template <bool FP8, bool SMALL, bool SHD>
__global__ void __launch_bounds__(FF_THREADS, FfnTmem<SMALL>::CTAS)
    grouped_ffn_kernel(const __grid_constant__ FfnMaps maps, FfnArgs g, DevCtx ctx) {
    using TM = FfnTmem<SMALL>;
    constexpr int KEL = FF_ROW_BYTES / (FP8 ? 1 : 2);   // elements of K per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NS = g.n_stages;
    uint8_t* smA = smem;
    uint8_t* smB = smA + (size_t)NS * FF_A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smB + (size_t)NS * g.b_stage_bytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + NS;
    uint64_t* tfull = bars + 2 * NS;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;
    // the epilogue warps' turn-around tiles: 16 x 32 16-bit values each, 16-byte aligned
    uint16_t* tbuf = reinterpret_cast<uint16_t*>((reinterpret_cast<uintptr_t>(tmem_holder + 1) + 15) &
                                                 ~static_cast<uintptr_t>(15));
    // the unit queue: the units this block claimed, in claim order
    uint64_t* uq_full = reinterpret_cast<uint64_t*>(tbuf + FF_EPI_WARPS * 16 * 32);
    uint64_t* uq_empty = uq_full + FF_UQ;
    volatile int* uq = reinterpret_cast<volatile int*>(uq_empty + FF_UQ);

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
        for (int q = 0; q < FF_UQ; ++q) {
            mbar_init(smem_u32(&uq_full[q]), 1);
            mbar_init(smem_u32(&uq_empty[q]), 1 + FF_EPI_WARPS);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), TM::COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();

    const int n_sched = *g.n_sched;
    const int n_up = n_sched * g.m_up;
    const int n_units = n_up + n_sched * g.m_down;
    const int up_target = FF_EPI_WARPS * g.m_up;   // reports of one entry's up units

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int qs = 0;
            uint32_t qph = 0;
            int claim = atomicAdd(g.claim, 1);
            while (ok) {
                // publish the claimed unit (or the end) to the MMA and epilogue warps
                const int u = claim < n_units ? claim : -1;
                if (!mbar_wait(smem_u32(&uq_empty[qs]), qph ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                uq[qs] = u;
                mbar_arrive(smem_u32(&uq_full[qs]));
                if (++qs == FF_UQ) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (u < 0) break;
                claim = atomicAdd(g.claim, 1);   // the next unit, claimed while this one loads
                const bool up = u < n_up;
                const int v = up ? u : u - n_up;
                const int m_blocks = up ? g.m_up : g.m_down;
                const int s_idx = v / m_blocks, mb = v % m_blocks;
                const int4 sc = g.sched[s_idx];
                const int Nout = up ? g.F : g.H;
                const int k_stages = up ? g.k_up : g.k_down;
                const bool a_full = Nout - mb * FF_BM > 64;
                const int n16 = (sc.z + 15) / 16;
                const int n128 = n16 / 8, n64 = (n16 % 8) / 4, r16 = n16 % 4;
                const uint32_t bytes = (uint32_t)((a_full ? 128 : 64) * FF_ROW_BYTES + n16 * 16 * FF_ROW_BYTES);
                const CUtensorMap* amap = up ? (a_full ? &maps.ua128 : &maps.ua64) : (a_full ? &maps.da128 : &maps.da64);
                const CUtensorMap* b128 = up ? &maps.ub128 : &maps.db128;
                const CUtensorMap* b64 = up ? &maps.ub64 : &maps.db64;
                const CUtensorMap* b16 = up ? &maps.ub16 : &maps.db16;
                int ay = sc.x * Nout + mb * FF_BM;
                // a chunk j of the shared expert: its up weight's rows j * F + ..., or its down
                // weight's columns j * F + ... (a 3-D load: (kx, row, j) or (j * F + kx, row, 0))
                const bool shd = SHD && sc.x >= g.e_shared;
                int sx0 = 0, sz = 0;
                if (shd) {
                    const int j = sc.x - g.e_shared;
                    if (up) {
                        amap = a_full ? &maps.us128 : &maps.us64;
                        ay = j * Nout + mb * FF_BM;
                    } else {
                        amap = a_full ? &maps.ds128 : &maps.ds64;
                        ay = mb * FF_BM;
                        sx0 = g.shared_cols ? j * g.shared_cols : 0;
                        sz = g.shared_cols ? 0 : j;
                    }
                }
                if (!up) {
                    // the rows of H this unit reads are written by the up units of its entry
                    if (!wait_count(g.done + s_idx, up_target, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();
                }
                for (int ks = 0; ks < k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_arrive_expect_tx(fb, bytes);
                    const int kx = ks * KEL;
                    const uint32_t a_dst = smem_u32(smA + (size_t)stage * FF_A_BYTES);
                    const uint32_t b_dst = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
                    if (SHD && shd && !up)
                        tma_load_3d(a_dst, amap, fb, sx0 + kx, ay, sz, pol_w);
                    else
                        tma_load_2d(a_dst, amap, fb, kx, ay, pol_w);
                    int row = 0;
                    for (int j = 0; j < n128; ++j, row += 128)
                        tma_load_2d(b_dst + row * FF_ROW_BYTES, b128, fb, kx, sc.y + row, pol_x);
                    for (int j = 0; j < n64; ++j, row += 64)
                        tma_load_2d(b_dst + row * FF_ROW_BYTES, b64, fb, kx, sc.y + row, pol_x);
                    for (int j = 0; j < r16; ++j, row += 16)
                        tma_load_2d(b_dst + row * FF_ROW_BYTES, b16, fb, kx, sc.y + row, pol_x);
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
            bool ok = true, issued = false;
            int qs = 0;
            uint32_t qph = 0;
            while (ok) {
                if (!mbar_wait(smem_u32(&uq_full[qs]), qph, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                const int u = uq[qs];
                mbar_arrive(smem_u32(&uq_empty[qs]));
                if (++qs == FF_UQ) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (u < 0) break;
                const bool up = u < n_up;
                const int v = up ? u : u - n_up;
                const int4 sc = g.sched[v / (up ? g.m_up : g.m_down)];
                const int k_stages = up ? g.k_up : g.k_down;
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = make_idesc(FP8 ? 0u : 1u, FF_BM, n_mma);
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TM::ACC);
                for (int ks = 0; ks < k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&full[stage]), phase, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smA + (size_t)stage * FF_A_BYTES);
                    const uint32_t b_base = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss<FP8>(d_tmem, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32), idesc,
                                    (ks | kk) != 0 ? 1u : 0u);
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
        // Epilogue: a warp reads 32 weight rows (features) x 16 token columns from TMEM, one
        // feature per lane, rounds them to their stored type and turns the tile around
        // through shared memory, so that each lane holds 16 consecutive features of one token
        // and stores them as 32 (bf16) or 16 (E4M3) contiguous bytes.
        const int q = warp & 3;   // TMEM lane quadrant of this warp
        uint16_t* tb = tbuf + (warp - 2) * (16 * 32);   // 16 rows x 32 bf16 (or E4M3 codes in the low byte)
        const int tj = lane & 15, th = lane >> 4;       // after the turn: token column, feature half
        int acc = 0;
        uint32_t acc_phase = 0;
        const float inv_h = (FP8) ? __frcp_rn(g.h_scale) : 1.0f;
        int qs = 0;
        uint32_t qph = 0;
        while (true) {
            if (!mbar_wait_warp(smem_u32(&uq_full[qs]), qph, ctx, abort_flag)) break;
            const int u = uq[qs];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&uq_empty[qs]));
            if (++qs == FF_UQ) {
                qs = 0;
                qph ^= 1u;
            }
            if (u < 0) break;
            const bool up = u < n_up;
            const int v = up ? u : u - n_up;
            const int m_blocks = up ? g.m_up : g.m_down;
            const int s_idx = v / m_blocks, mb = v % m_blocks;
            const int4 sc = g.sched[s_idx];
            const int Nout = up ? g.F : g.H;
            if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, ctx, abort_flag)) break;
            tc_fence_after();
            const int f16 = mb * FF_BM + q * 32 + th * 16;   // first of this lane's 16 features
            float scale = 1.0f;
            if constexpr (FP8) scale = up ? __fmul_rn(g.su[sc.x], g.x_scale) : __fmul_rn(g.sd[sc.x], g.h_scale);
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TM::ACC);
            const int nchunks = (sc.z + 15) / 16;
            for (int c = 0; c < nchunks; ++c) {
                uint32_t vv[16];
                tmem_ld16(t_row + (uint32_t)(c * 16), vv);
#pragma unroll
                for (int j = 0; j < 16; j += 2) {
                    // token columns j and j + 1 of this lane's feature, converted as a pair
                    float z0 = __uint_as_float(vv[j]), z1 = __uint_as_float(vv[j + 1]);
                    if constexpr (FP8) {
                        z0 = __fmul_rn(z0, scale);
                        z1 = __fmul_rn(z1, scale);
                    }
                    if (up) {
                        z0 = z0 > 0.0f ? __fmul_rn(z0, z0) : 0.0f;
                        z1 = z1 > 0.0f ? __fmul_rn(z1, z1) : 0.0f;
                    }
                    uint32_t pair;
                    if (up && FP8) {
                        pair = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(z0, inv_h), __fmul_rn(z1, inv_h)),
                                                        __NV_SATFINITE, __NV_E4M3);
                        pair = (pair & 0xFFu) | ((pair & 0xFF00u) << 8);   // one code per 16-bit slot
                    } else {
                        const __nv_bfloat162 p2 = __floats2bfloat162_rn(z0, z1);
                        pair = *reinterpret_cast<const uint32_t*>(&p2);
                    }
                    // row j, feature `lane`: 16-byte chunk (lane / 8) xor (j mod 4)
                    tb[j * 32 + ((((lane >> 3) ^ (j & 3))) << 3) + (lane & 7)] = (uint16_t)(pair & 0xFFFFu);
                    tb[(j + 1) * 32 + ((((lane >> 3) ^ ((j + 1) & 3))) << 3) + (lane & 7)] = (uint16_t)(pair >> 16);
                }
                __syncwarp();
                const uint4 c0 = *reinterpret_cast<const uint4*>(tb + tj * 32 + (((2 * th) ^ (tj & 3)) << 3));
                const uint4 c1 = *reinterpret_cast<const uint4*>(tb + tj * 32 + (((2 * th + 1) ^ (tj & 3)) << 3));
                __syncwarp();
                const int r = c * 16 + tj;
                if (r < sc.z && f16 < Nout) {
                    const int64_t row = sc.y + r;
                    if (up && FP8) {
                        // 16 codes, one per 16-bit slot: keep the low bytes
                        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                        uint32_t p4[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            p4[i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x6420);
                        *reinterpret_cast<uint4*>(static_cast<uint8_t*>(g.hb) + row * g.F + f16) =
                            make_uint4(p4[0], p4[1], p4[2], p4[3]);
                    } else {
                        uint4* d4 = reinterpret_cast<uint4*>(up ? static_cast<uint16_t*>(g.hb) + row * g.F + f16
                                                                : static_cast<uint16_t*>(g.y) + row * g.H + f16);
                        d4[0] = c0;
                        d4[1] = c1;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));
            if (up) {
                // this warp's rows of H are complete: every lane orders its stores for the async
                // proxy (the TMA loads of H), the warp barrier orders them before lane 0's release
                fence_proxy_async_global();
                __syncwarp();
                const bool hold = g.debug_hold && u == 0;
                if (lane == 0 && !hold) red_release_add(g.done + s_idx, 1);
            }
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
        tmem_dealloc(tmem_base, TM::COLS);
    }
}

typedef CUresult (*EncodeTiledFnF)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnF encode_fn_ffn() {
    static EncodeTiledFnF fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFnF>(p);
    }
    return fn;
}

// 2-D map over a row-major [rows][cols] matrix, box = 128 bytes x box_rows, 128-byte swizzle.
bool map_ffn(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, bool fp8, int box_rows) {
    EncodeTiledFnF fn = encode_fn_ffn();
    if (!fn) return false;
    const int es = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * es)};
    cuuint32_t box[2] = {(cuuint32_t)(FF_ROW_BYTES / es), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Both projections of the grouped FFN in one launch.  xp [rows][H] and hb [rows][F]
// (bf16, or E4M3 codes), y [rows][H] bf16; done: max_sched + 1 ints (the per-entry counters, then
// the unit claim counter), zero before the launch.
cudaError_t launch_grouped_ffn(bool fp8, const void* w_up, const void* w_down, int E, int F, int H, const void* xp,
                               void* hb, void* y, int64_t rows, const int4* sched, const int* n_sched, int* done,
                               const GemmPlan& plan, const float* su, const float* sd, float x_scale, float h_scale,
                               int num_sms, int debug_hold, const DevCtx& ctx, cudaStream_t stream,
                               const void* w_up_s, const void* w_down_s, int n_shared) {
    if (rows == 0) return cudaSuccess;
    FfnMaps maps;
    if (!map_ffn(&maps.ua128, w_up, (int64_t)E * F, H, fp8, 128) || !map_ffn(&maps.ua64, w_up, (int64_t)E * F, H, fp8, 64) ||
        !map_ffn(&maps.ub128, xp, rows, H, fp8, 128) || !map_ffn(&maps.ub64, xp, rows, H, fp8, 64) ||
        !map_ffn(&maps.ub16, xp, rows, H, fp8, 16) || !map_ffn(&maps.da128, w_down, (int64_t)E * H, F, fp8, 128) ||
        !map_ffn(&maps.da64, w_down, (int64_t)E * H, F, fp8, 64) || !map_ffn(&maps.db128, hb, rows, F, fp8, 128) ||
        !map_ffn(&maps.db64, hb, rows, F, fp8, 64) || !map_ffn(&maps.db16, hb, rows, F, fp8, 16))
        return cudaErrorInvalidValue;
    // the shared expert (bf16 only): n_shared chunks of width F, schedule entries E .. E + n_shared - 1
    int shared_cols = 0;
    maps.us128 = maps.ua128;   // read only by units of shared-expert entries
    maps.us64 = maps.ua64;
    maps.ds128 = maps.ds64 = maps.da128;
    if (n_shared > 0) {
        if (fp8 || !w_up_s || !w_down_s) return cudaErrorInvalidValue;
        if (!map_ffn(&maps.us128, w_up_s, (int64_t)n_shared * F, H, false, 128) ||
            !map_ffn(&maps.us64, w_up_s, (int64_t)n_shared * F, H, false, 64))
            return cudaErrorInvalidValue;
        bool ok = !shared_map_2d() && make_map_chunks(&maps.ds128, w_down_s, H, F, n_shared, 128) &&
                  make_map_chunks(&maps.ds64, w_down_s, H, F, n_shared, 64);
        if (!ok) {
            // the plain [H][n * F] matrix as {n * F, H, 1}, chunk j from column j * F (a K tail meets
            // activation columns that read as zero)
            shared_cols = F;
            ok = make_map_chunks(&maps.ds128, w_down_s, H, (int64_t)n_shared * F, 1, 128) &&
                 make_map_chunks(&maps.ds64, w_down_s, H, (int64_t)n_shared * F, 1, 64);
        }
        if (!ok) return cudaErrorInvalidValue;
    }
    FfnArgs g;
    g.e_shared = n_shared > 0 ? E : 0x7fffffff;
    g.shared_cols = shared_cols;
    g.sched = sched;
    g.n_sched = n_sched;
    g.done = done;
    g.claim = done + plan.max_sched;
    g.m_up = (F + FF_BM - 1) / FF_BM;
    g.m_down = (H + FF_BM - 1) / FF_BM;
    g.F = F;
    g.H = H;
    const int es = fp8 ? 1 : 2;
    g.k_up = (int)(((int64_t)H * es + FF_ROW_BYTES - 1) / FF_ROW_BYTES);
    g.k_down = (int)(((int64_t)F * es + FF_ROW_BYTES - 1) / FF_ROW_BYTES);
    if (plan.bn > FfnTmem<false>::ACC) return cudaErrorInvalidValue;
    const bool small = plan.bn <= FfnTmem<true>::ACC;
    // ring depth for this launch's layout: as many stages as fit in its budget, 2 to 8
    const int stage_bytes = FF_A_BYTES + plan.bn * FF_ROW_BYTES;
    int ns = (small ? FfnTmem<true>::RING : FfnTmem<false>::RING) / stage_bytes;
    if (ns > 8) ns = 8;
    if (ns < 2) ns = 2;
    g.n_stages = ns;
    g.b_stage_bytes = plan.bn * FF_ROW_BYTES;
    g.hb = hb;
    g.y = y;
    g.su = su;
    g.sd = sd;
    g.x_scale = x_scale;
    g.h_scale = h_scale;
    g.debug_hold = debug_hold;
    const int64_t max_units = (int64_t)plan.max_sched * (g.m_up + g.m_down);
    const int64_t slots = (int64_t)num_sms * (small ? FfnTmem<true>::CTAS : FfnTmem<false>::CTAS);
    const int grid = (int)(max_units < slots ? max_units : slots);
    const bool shd = n_shared > 0;   // bf16 only
    auto kfn = shd ? (small ? grouped_ffn_kernel<false, true, true> : grouped_ffn_kernel<false, false, true>)
               : small ? (fp8 ? grouped_ffn_kernel<true, true, false> : grouped_ffn_kernel<false, true, false>)
                       : (fp8 ? grouped_ffn_kernel<true, false, false> : grouped_ffn_kernel<false, false, false>);
    // ring, its barriers (full, empty, two tfull, two tempty, drain), the abort flag and TMEM
    // holder, the epilogue's turn-around tiles and the unit queue
    const size_t smem = 1024 + (size_t)ns * stage_bytes + (size_t)(2 * ns + 5) * 8 + 16 + 16 +
                        (size_t)FF_EPI_WARPS * 16 * 32 * sizeof(uint16_t) + 2 * FF_UQ * sizeof(uint64_t) +
                        FF_UQ * sizeof(int);
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch_k(kfn, dim3(grid), dim3(FF_THREADS), smem, stream, maps, g, ctx);
}

}  // namespace moe
