// FP8_B128 W8A8 grouped expert GEMMs (bloomery issue page, s.3 "Kernel
// dispatch" and the FP8 release: FP8_B128 scales, the 64-value tail of
// K = 1856, physical K 1920).  The weights are E4M3 codes with one fp32
// scale per block of 128 values along K of each row (K padded with zero codes
// to Kp = 128 * ceil(K / 128)); the activations are E4M3 codes with one static
// scale per tensor.  For a weight row f and a token row r,
//   z[r, f] = s_act * sum_b s_w[f, b] * sum_{k in block b} q_w[f, k] q_act[r, k],
// followed by ReLU^2 and the E4M3 requantisation of H (up) or the bf16 output
// (down), as in the scalar-scale path.
//
// Same swap-AB orientation, schedule and TMA ring as the bf16 / E4M3 kernel:
// a 128-row weight block is the MMA's M side, the expert's token rows (at most
// 128 per schedule entry here) its N side.  A 128-byte K stage of E4M3 values
// is exactly one scale block, so every stage's product goes to its own TMEM
// partial (one of four slots of 64 or 128 columns): the MMA overwrites the slot with
// the block's sum, and the epilogue warps, which hold the running fp32 sums
// of their weight row in registers, add s_w[f, b] times the partial and free
// the slot.  Roles (192 threads): warp 0 TMA producer, warp 1 MMA, warps 2..5
// the partial sums and the epilogue.  Every wait is bounded.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int GB_THREADS = 192;
constexpr int GB_BM = 128;                  // weight rows per unit
constexpr int GB_ROW = 128;                 // bytes = E4M3 values of one K stage = one scale block
constexpr int GB_A_BYTES = GB_BM * GB_ROW;  // 16 KB
constexpr int GB_NP = 4;                    // TMEM partial slots of BN columns
// BN: token rows per schedule entry at most, 64 or 128 (a template parameter: the
// running sums are BN registers per thread); TMEM holds GB_NP slots of BN columns.

struct B128Maps {
    CUtensorMap a128;   // weight codes [E * Nout][Kp], 128-row box
    CUtensorMap a64;    // 64-row box
    CUtensorMap b64;    // activation codes [rows][K], 64-row box
    CUtensorMap b16;    // 16-row box
};

struct B128Args {
    const int4* sched;     // {e, row0, nrows, 0}, nrows <= BN
    const int* n_sched;
    int m_blocks;          // ceil(Nout / 128)
    int Nout;
    int k_stages;          // Kp / 128 = scale blocks per weight row
    int n_stages;          // smem ring depth
    int b_stage_bytes;     // bn * 128
    void* out;             // up: e4m3 codes [rows][Nout]; down: bf16 [rows][Nout]
    int64_t out_ld;
    const float* w_scale;  // [E][Nout][k_stages]
    float in_scale;        // x_scale (up) or h_scale (down)
    float out_scale;       // h_scale (up)
    int debug_withhold;
};

// The epilogue warps' part of one K stage: add s_w[f, block] times the stage's partial (its first
// nch 16-column chunks at t_row) to the running fp32 sums of this lane's weight row.
template <int BN>
__device__ __forceinline__ void b128_add_block(float (&acc)[BN], uint32_t t_row, int nch, float sw) {
#pragma unroll
    for (int c = 0; c < BN / 16; ++c) {
        if (c < nch) {
            uint32_t v[16];
            tmem_ld16(t_row + (uint32_t)(c * 16), v);
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[c * 16 + j] = __fmaf_rn(sw, __uint_as_float(v[j]), acc[c * 16 + j]);
        }
    }
}

// After a unit's last block: this lane's feature f for the tile's token rows r < nrows (row0 + r):
// times the activation scale, then ReLU^2 and the E4M3 code of H / s_h (up, into h [.][ld]) or
// the bf16 Y (down, into y [.][ld]).
template <int BN>
__device__ __forceinline__ void b128_store_unit(const float (&acc)[BN], int nch, int nrows, int64_t row0, int f,
                                                bool up, float in_scale, float inv_h, uint8_t* h,
                                                __nv_bfloat16* y, int64_t ld) {
#pragma unroll
    for (int c = 0; c < BN / 16; ++c) {
        if (c >= nch) break;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int r = c * 16 + j;
            if (r < nrows) {
                const float z = __fmul_rn(acc[r], in_scale);
                const int64_t o = (row0 + r) * ld + f;
                if (up) {
                    const float a = z > 0.0f ? __fmul_rn(z, z) : 0.0f;
                    h[o] = (uint8_t)__nv_cvt_float_to_fp8(__fmul_rn(a, inv_h), __NV_SATFINITE, __NV_E4M3);
                } else {
                    y[o] = __float2bfloat16_rn(z);
                }
            }
        }
    }
}

template <bool UP, int BN>
__global__ void __launch_bounds__(GB_THREADS, 1)
    grouped_gemm_b128_kernel(const __grid_constant__ B128Maps maps, B128Args g, DevCtx ctx) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NS = g.n_stages;
    uint8_t* smA = smem;
    uint8_t* smB = smA + (size_t)NS * GB_A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smB + (size_t)NS * g.b_stage_bytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + NS;
    uint64_t* pfull = bars + 2 * NS;
    uint64_t* pempty = pfull + GB_NP;
    uint64_t* drain = pempty + GB_NP;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int p = 0; p < GB_NP; ++p) {
            mbar_init(smem_u32(&pfull[p]), 1);
            mbar_init(smem_u32(&pempty[p]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&maps.a128);
        tma_prefetch_desc(&maps.a64);
        tma_prefetch_desc(&maps.b64);
        tma_prefetch_desc(&maps.b16);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), GB_NP * BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();

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
                const bool a_full = g.Nout - mb * GB_BM > 64;
                const int n16 = (sc.z + 15) / 16;   // <= 4
                const int n64 = n16 / 4, r16 = n16 % 4;
                const uint32_t bytes = (uint32_t)((a_full ? 128 : 64) * GB_ROW + n16 * 16 * GB_ROW);
                const int a_y = sc.x * g.Nout + mb * GB_BM;
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
                        const int kx = ks * GB_ROW;
                        const uint32_t a_dst = smem_u32(smA + (size_t)stage * GB_A_BYTES);
                        const uint32_t b_dst = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
                        tma_load_2d(a_dst, a_full ? &maps.a128 : &maps.a64, fb, kx, a_y, pol_w);
                        int row = 0;
                        for (int j = 0; j < n64; ++j, row += 64)
                            tma_load_2d(b_dst + row * GB_ROW, &maps.b64, fb, kx, sc.y + row, pol_x);
                        for (int j = 0; j < r16; ++j, row += 16)
                            tma_load_2d(b_dst + row * GB_ROW, &maps.b16, fb, kx, sc.y + row, pol_x);
                    }
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
        if (lane == 0) {
            int stage = 0, ps = 0;
            uint32_t phase = 0, pph = 0;
            bool ok = true, issued = false;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int4 sc = g.sched[u / g.m_blocks];
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = make_idesc(0u, GB_BM, n_mma);
                for (int ks = 0; ks < g.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&full[stage]), phase, ctx, abort_flag) ||
                        !mbar_wait(smem_u32(&pempty[ps]), pph ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(ps * BN);
                    const uint32_t a_base = smem_u32(smA + (size_t)stage * GB_A_BYTES);
                    const uint32_t b_base = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // 4 x K = 32: the block's sum, the slot overwritten first
                        mma_ss<true>(d_tmem, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32), idesc,
                                     kk != 0 ? 1u : 0u);
                    issued = true;
                    mma_commit(smem_u32(&empty[stage]));
                    mma_commit(smem_u32(&pfull[ps]));
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++ps == GB_NP) {
                        ps = 0;
                        pph ^= 1u;
                    }
                }
            }
            if (!ok && issued) {
                mma_commit(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else {
        const int q = warp & 3;   // TMEM lane quadrant of this warp
        int ps = 0;
        uint32_t pph = 0;
        bool ok = true;
        const float inv_out = UP ? __frcp_rn(g.out_scale) : 1.0f;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            const int4 sc = g.sched[u / g.m_blocks];
            const int mb = u % g.m_blocks;
            const int f = mb * GB_BM + q * 32 + lane;
            const bool fvalid = f < g.Nout;
            const int nch = (sc.z + 15) / 16;   // warp-uniform, <= 4
            const float* wrow = g.w_scale + ((int64_t)sc.x * g.Nout + (fvalid ? f : 0)) * g.k_stages;
            float acc[BN];
#pragma unroll
            for (int i = 0; i < BN; ++i) acc[i] = 0.0f;
            for (int ks = 0; ks < g.k_stages; ++ks) {
                if (!mbar_wait_warp(smem_u32(&pfull[ps]), pph, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(ps * BN);
                b128_add_block<BN>(acc, t_row, nch, wrow[ks]);
                tc_fence_before();
                mbar_arrive(smem_u32(&pempty[ps]));
                if (++ps == GB_NP) {
                    ps = 0;
                    pph ^= 1u;
                }
            }
            if (!ok) break;
            if (fvalid)
                b128_store_unit<BN>(acc, nch, sc.z, sc.y, f, UP, g.in_scale, inv_out, static_cast<uint8_t*>(g.out),
                                    static_cast<__nv_bfloat16*>(g.out), g.out_ld);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GB_NP * BN);
    }
}

// ----------------------------------------------------------------------------- one-launch FFN

// Both FP8_B128 projections in one persistent launch, as the bf16 one-launch FFN
// (grouped_ffn.cu) does it: every up unit (schedule entry x 128-row block of F), then every
// down unit (entry x block of H), claimed in that order from a global counter by each CTA's
// producer and passed to the MMA thread and the epilogue warps through a small queue in shared
// memory.  An up unit's epilogue warps store their features of H, fence them for the async
// proxy and each add 1 to done[entry] with release semantics; the producer of a down unit
// waits (bounded) until done[entry] reaches 4 x (blocks of F) before it loads the entry's H.
// Tiles of up to 64 rows (TMEM: 4 partial slots of 64 columns, 256 in all) run two CTAs per SM
// with a 100 KB ring each.
constexpr int FB_UQ = 4;   // unit queue slots
constexpr int FB_BN = 64;  // token rows per schedule entry at most
constexpr int FB_RING = 100 * 1024;
static_assert(FB_BN == kB128OneLaunchTileRows, "one-launch FP8_B128 tile rows");

struct B128FfnArgs {
    int* claim;              // unit counter (zero at launch; right after done[])
    int* done;               // [max_sched] up epilogue warps finished per entry (zero at launch)
    const int4* sched;
    const int* n_sched;
    int m_up, m_down;        // 128-row blocks of F and of H
    int F, H;
    int k_up, k_down;        // scale blocks (K stages) of H and of F
    int n_stages;
    int b_stage_bytes;
    const float* su;         // [E][F][k_up]
    const float* sd;         // [E][H][k_down]
    float x_scale, h_scale;
    uint8_t* hb;             // H codes [rows][F]
    void* y;                 // bf16 [rows][H]
    int debug_hold;          // 1: the list's first up unit never reports its rows (a wait must expire)
};

struct B128FfnMaps {
    B128Maps up, down;
};

template <int BN>
__global__ void __launch_bounds__(GB_THREADS, 2)
    grouped_ffn_b128_kernel(const __grid_constant__ B128FfnMaps maps, B128FfnArgs g, DevCtx ctx) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NS = g.n_stages;
    uint8_t* smA = smem;
    uint8_t* smB = smA + (size_t)NS * GB_A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smB + (size_t)NS * g.b_stage_bytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + NS;
    uint64_t* pfull = bars + 2 * NS;
    uint64_t* pempty = pfull + GB_NP;
    uint64_t* drain = pempty + GB_NP;
    uint64_t* uq_full = drain + 1;
    uint64_t* uq_empty = uq_full + FB_UQ;
    volatile int* uq = reinterpret_cast<volatile int*>(uq_empty + FB_UQ);
    volatile int* abort_flag = uq + FB_UQ;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(const_cast<int*>(abort_flag + 1));

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int p = 0; p < GB_NP; ++p) {
            mbar_init(smem_u32(&pfull[p]), 1);
            mbar_init(smem_u32(&pempty[p]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        for (int q = 0; q < FB_UQ; ++q) {
            mbar_init(smem_u32(&uq_full[q]), 1);
            mbar_init(smem_u32(&uq_empty[q]), 1 + 4);   // the MMA thread and the 4 epilogue warps
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), GB_NP * BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();

    const int n_sched = *g.n_sched;
    const int n_up = n_sched * g.m_up;
    const int n_units = n_up + n_sched * g.m_down;
    const int up_target = 4 * g.m_up;   // reports of one entry's up units

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
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
                const int u = claim < n_units ? claim : -1;
                if (!mbar_wait(smem_u32(&uq_empty[qs]), qph ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                uq[qs] = u;
                mbar_arrive(smem_u32(&uq_full[qs]));
                if (++qs == FB_UQ) {
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
                const B128Maps& mp = up ? maps.up : maps.down;
                const bool a_full = Nout - mb * GB_BM > 64;
                const int n16 = (sc.z + 15) / 16;
                const int n64 = n16 / 4, r16 = n16 % 4;
                const uint32_t bytes = (uint32_t)((a_full ? 128 : 64) * GB_ROW + n16 * 16 * GB_ROW);
                const int a_y = sc.x * Nout + mb * GB_BM;
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
                    const int kx = ks * GB_ROW;
                    const uint32_t a_dst = smem_u32(smA + (size_t)stage * GB_A_BYTES);
                    const uint32_t b_dst = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
                    tma_load_2d(a_dst, a_full ? &mp.a128 : &mp.a64, fb, kx, a_y, pol_w);
                    int row = 0;
                    for (int j = 0; j < n64; ++j, row += 64)
                        tma_load_2d(b_dst + row * GB_ROW, &mp.b64, fb, kx, sc.y + row, pol_x);
                    for (int j = 0; j < r16; ++j, row += 16)
                        tma_load_2d(b_dst + row * GB_ROW, &mp.b16, fb, kx, sc.y + row, pol_x);
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
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            int stage = 0, ps = 0;
            uint32_t phase = 0, pph = 0;
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
                if (++qs == FB_UQ) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (u < 0) break;
                const bool up = u < n_up;
                const int v = up ? u : u - n_up;
                const int4 sc = g.sched[v / (up ? g.m_up : g.m_down)];
                const int k_stages = up ? g.k_up : g.k_down;
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = make_idesc(0u, GB_BM, n_mma);
                for (int ks = 0; ks < k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&full[stage]), phase, ctx, abort_flag) ||
                        !mbar_wait(smem_u32(&pempty[ps]), pph ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(ps * BN);
                    const uint32_t a_base = smem_u32(smA + (size_t)stage * GB_A_BYTES);
                    const uint32_t b_base = smem_u32(smB + (size_t)stage * g.b_stage_bytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // 4 x K = 32: the block's sum, the slot overwritten first
                        mma_ss<true>(d_tmem, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32), idesc,
                                     kk != 0 ? 1u : 0u);
                    issued = true;
                    mma_commit(smem_u32(&empty[stage]));
                    mma_commit(smem_u32(&pfull[ps]));
                    if (++stage == NS) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++ps == GB_NP) {
                        ps = 0;
                        pph ^= 1u;
                    }
                }
            }
            if (!ok && issued) {
                mma_commit(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else {
        // ---------------------------------------------------------------- block sums and epilogue
        const int q = warp & 3;   // TMEM lane quadrant of this warp
        int ps = 0;
        uint32_t pph = 0;
        bool ok = true;
        int qs = 0;
        uint32_t qph = 0;
        const float inv_h = __frcp_rn(g.h_scale);
        while (ok) {
            if (!mbar_wait_warp(smem_u32(&uq_full[qs]), qph, ctx, abort_flag)) break;
            const int u = uq[qs];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&uq_empty[qs]));
            if (++qs == FB_UQ) {
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
            const int k_stages = up ? g.k_up : g.k_down;
            const int f = mb * GB_BM + q * 32 + lane;
            const bool fvalid = f < Nout;
            const int nch = (sc.z + 15) / 16;   // warp-uniform, <= BN / 16
            const float* wrow = (up ? g.su : g.sd) + ((int64_t)sc.x * Nout + (fvalid ? f : 0)) * k_stages;
            const float in_scale = up ? g.x_scale : g.h_scale;
            float acc[BN];
#pragma unroll
            for (int i = 0; i < BN; ++i) acc[i] = 0.0f;
            for (int ks = 0; ks < k_stages; ++ks) {
                if (!mbar_wait_warp(smem_u32(&pfull[ps]), pph, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(ps * BN);
                b128_add_block<BN>(acc, t_row, nch, wrow[ks]);
                tc_fence_before();
                mbar_arrive(smem_u32(&pempty[ps]));
                if (++ps == GB_NP) {
                    ps = 0;
                    pph ^= 1u;
                }
            }
            if (!ok) break;
            if (fvalid)
                b128_store_unit<BN>(acc, nch, sc.z, sc.y, f, up, in_scale, inv_h, g.hb, static_cast<__nv_bfloat16*>(g.y),
                                    up ? g.F : g.H);
            if (up) {
                // this warp's features of H are complete: every lane orders its stores for the async
                // proxy (the TMA loads of H), the warp barrier orders them before lane 0's release
                fence_proxy_async_global();
                __syncwarp();
                const bool hold = g.debug_hold && u == 0;
                if (lane == 0 && !hold) red_release_add(g.done + s_idx, 1);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, GB_NP * BN);
    }
}

// One warp per (row, block of 128): scale amax / 448 (1 for a zero block),
// codes e4m3(fl32(w / scale)) nearest-even and saturating, zero past K.
__global__ void quantize_fp8_b128_kernel(const uint16_t* __restrict__ src, int64_t rows, int K, int Kp,
                                         uint8_t* __restrict__ codes, float* __restrict__ scales) {
    const int nb = Kp / 128;
    const int lane = threadIdx.x % 32;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t item = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; item < rows * nb;
         item += warps) {
        const int64_t r = item / nb;
        const int k0 = (int)(item % nb) * 128 + lane * 4;
        float v[4];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int k = k0 + i;
            v[i] = k < K ? __uint_as_float((uint32_t)src[r * K + k] << 16) : 0.0f;
            amax = fmaxf(amax, fabsf(v[i]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t c = k0 + i < K ? (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(v[i], s), __NV_SATFINITE,
                                                                             __NV_E4M3)
                                          : 0u;
            packed |= c << (8 * i);
        }
        *reinterpret_cast<uint32_t*>(codes + r * Kp + k0) = packed;
        if (lane == 0) scales[item] = s;
    }
}

// ----------------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFnB)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFnB encode_fn_b128() {
    static EncodeTiledFnB fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFnB>(p);
    }
    return fn;
}

// 2-D map over a row-major u8 [rows][cols] matrix, box 128 bytes x box_rows, 128-byte swizzle.
static bool make_map_u8_b128(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFnB fn = encode_fn_b128();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {(cuuint32_t)GB_ROW, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int b128_kp(int K) { return (K + 127) / 128 * 128; }

// One FP8_B128 projection.  W: codes [E * Nout][Kp], w_scale [E][Nout][Kp / 128];
// act: E4M3 codes [rows][Kdim] in the expert layout; out [rows][Nout] (e4m3 codes
// for the up projection, bf16 for the down).  bn <= 128 (the schedule's tile): the
// kernel's running sums are 64 registers per thread up to 64 rows, 128 beyond.
cudaError_t launch_grouped_gemm_b128(bool up, const uint8_t* W, const float* w_scale, int E, int Nout, int Kdim,
                                     const uint8_t* act, int64_t rows, const int4* sched, const int* n_sched, int bn,
                                     int max_sched, void* out, float in_scale, float out_scale, int num_sms,
                                     int debug_withhold, const DevCtx& ctx, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    if (bn < 16 || bn > kB128MaxTileRows || bn % 16 != 0) return cudaErrorInvalidValue;
    const int Kp = b128_kp(Kdim);
    B128Maps maps;
    if (!make_map_u8_b128(&maps.a128, W, (int64_t)E * Nout, Kp, 128) ||
        !make_map_u8_b128(&maps.a64, W, (int64_t)E * Nout, Kp, 64) ||
        !make_map_u8_b128(&maps.b64, act, rows, Kdim, 64) || !make_map_u8_b128(&maps.b16, act, rows, Kdim, 16))
        return cudaErrorInvalidValue;
    B128Args g;
    g.sched = sched;
    g.n_sched = n_sched;
    g.m_blocks = (Nout + GB_BM - 1) / GB_BM;
    g.Nout = Nout;
    g.k_stages = Kp / GB_ROW;
    g.b_stage_bytes = bn * GB_ROW;
    const int stage = GB_A_BYTES + g.b_stage_bytes;
    int ns = (200 * 1024) / stage;
    if (ns > 8) ns = 8;
    if (ns < 2) ns = 2;
    g.n_stages = ns;
    g.out = out;
    g.out_ld = Nout;
    g.w_scale = w_scale;
    g.in_scale = in_scale;
    g.out_scale = out_scale;
    g.debug_withhold = debug_withhold;
    const size_t smem = 1024 + (size_t)ns * stage + (size_t)(2 * ns + 2 * GB_NP + 1) * 8 + 16;
    const int64_t max_units = (int64_t)max_sched * g.m_blocks;
    const int grid = (int)(max_units < num_sms ? max_units : num_sms);
    auto kfn = bn > 64 ? (up ? grouped_gemm_b128_kernel<true, 128> : grouped_gemm_b128_kernel<false, 128>)
                       : (up ? grouped_gemm_b128_kernel<true, 64> : grouped_gemm_b128_kernel<false, 64>);
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch_k(kfn, dim3(grid), dim3(GB_THREADS), smem, stream, maps, g, ctx);
}

// Both FP8_B128 projections in one launch.  W_up codes [E*F][Kp(H)] with scales su
// [E][F][Kp(H)/128], W_down codes [E*H][Kp(F)] with sd [E][H][Kp(F)/128]; xp: E4M3 codes of the
// permuted rows [rows][H]; hb: H's E4M3 codes [rows][F]; y: bf16 [rows][H].  done: max_sched + 1
// ints (the per-entry counters, then the unit claim counter), zero before the launch.
cudaError_t launch_grouped_ffn_b128(const uint8_t* w_up, const float* su, const uint8_t* w_down, const float* sd,
                                    int E, int F, int H, const uint8_t* xp, uint8_t* hb, void* y, int64_t rows,
                                    const int4* sched, const int* n_sched, int bn, int max_sched, int* done,
                                    float x_scale, float h_scale, int num_sms, int debug_hold, const DevCtx& ctx,
                                    cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    if (bn < 16 || bn > FB_BN || bn % 16 != 0) return cudaErrorInvalidValue;
    const int Kh = b128_kp(H), Kf = b128_kp(F);
    B128FfnMaps maps;
    if (!make_map_u8_b128(&maps.up.a128, w_up, (int64_t)E * F, Kh, 128) ||
        !make_map_u8_b128(&maps.up.a64, w_up, (int64_t)E * F, Kh, 64) ||
        !make_map_u8_b128(&maps.up.b64, xp, rows, H, 64) || !make_map_u8_b128(&maps.up.b16, xp, rows, H, 16) ||
        !make_map_u8_b128(&maps.down.a128, w_down, (int64_t)E * H, Kf, 128) ||
        !make_map_u8_b128(&maps.down.a64, w_down, (int64_t)E * H, Kf, 64) ||
        !make_map_u8_b128(&maps.down.b64, hb, rows, F, 64) || !make_map_u8_b128(&maps.down.b16, hb, rows, F, 16))
        return cudaErrorInvalidValue;
    B128FfnArgs g;
    g.done = done;
    g.claim = done + max_sched;
    g.sched = sched;
    g.n_sched = n_sched;
    g.m_up = (F + GB_BM - 1) / GB_BM;
    g.m_down = (H + GB_BM - 1) / GB_BM;
    g.F = F;
    g.H = H;
    g.k_up = Kh / GB_ROW;
    g.k_down = Kf / GB_ROW;
    g.b_stage_bytes = bn * GB_ROW;
    const int stage = GB_A_BYTES + g.b_stage_bytes;
    int ns = FB_RING / stage;
    if (ns > 8) ns = 8;
    if (ns < 2) ns = 2;
    g.n_stages = ns;
    g.su = su;
    g.sd = sd;
    g.x_scale = x_scale;
    g.h_scale = h_scale;
    g.hb = hb;
    g.y = y;
    g.debug_hold = debug_hold;
    // ring, barriers (full, empty, 4 pfull, 4 pempty, drain, the queue's full and empty), the
    // queue, the abort flag and the TMEM holder
    const size_t smem = 1024 + (size_t)ns * stage + (size_t)(2 * ns + 2 * GB_NP + 1 + 2 * FB_UQ) * 8 +
                        FB_UQ * sizeof(int) + 8 + 16;
    const int64_t max_units = (int64_t)max_sched * (g.m_up + g.m_down);
    const int64_t slots = (int64_t)num_sms * 2;   // two CTAs per SM
    const int grid = (int)(max_units < slots ? max_units : slots);
    auto kfn = grouped_ffn_b128_kernel<FB_BN>;
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch_k(kfn, dim3(grid), dim3(GB_THREADS), smem, stream, maps, g, ctx);
}

cudaError_t launch_quantize_fp8_b128(int64_t rows, int K, const uint16_t* src, uint8_t* codes, float* scales,
                                     int num_sms, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    const int Kp = b128_kp(K);
    const int64_t items = rows * (Kp / 128);
    int64_t blocks = (items + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    quantize_fp8_b128_kernel<<<(unsigned)blocks, 256, 0, stream>>>(src, rows, K, Kp, codes, scales);
    return cudaGetLastError();
}

}  // namespace moe
