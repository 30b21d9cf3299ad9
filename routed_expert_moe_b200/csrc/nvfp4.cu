// NVFP4 W4A4 experts (bloomery issue page, s.2 "Checkpoint facts": the NVFP4
// release runs the experts W4A4; the format is NVIDIA's NVFP4): E2M1 codes,
// one E4M3 scale per block of 16 elements along the contraction dimension,
// one fp32 scale per tensor.
//
//   s_t   = amax / 2688 for a weight tensor (6 x 448), a static value for the
//           activations x and H;
//   S_b   = e4m3(fl32(fl32(amax_b / 6) / s_t)),  e_b = fl32(dec(S_b) * s_t);
//   q     = e2m1(fl32(x / e_b)) (nearest, ties to even, saturating at 6), 0 if e_b = 0.
//
// Layouts: codes [rows][K/2] bytes (element 2i in the low nibble), block
// scales [rows][KSP] bytes with KSP = K/16 rounded up to 16 (the padding is
// zero), tensor scales fp32.
//
// The grouped GEMM (swap-AB like the bf16 kernel: 128 weight rows are the
// MMA's M side, the expert's token rows its N side) streams the packed codes
// and block scales with TMA, 256 K values per stage, and four converter
// warps dequantise them into fp16 tiles in shared memory: every product
// e2m1 x e4m3 is exact in fp16 (at most 5 significant bits, magnitudes 2^-10
// .. 2688), so the tensor cores (kind::f16, fp32 accumulate) see exactly the
// dequantised block values; the two tensor scales multiply the accumulator
// in the epilogue.  The up projection's epilogue quantises ReLU^2 to NVFP4
// in blocks of 16 features (16 TMEM lanes: a half warp) for the down
// projection.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

// ----------------------------------------------------------------------------- element helpers

// Two fp32 values to one byte of E2M1 codes (lo in the low nibble), nearest-even, saturating.
__device__ __forceinline__ uint32_t e2m1_pack(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t e4m3_code(float v) {
    return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    return __half2float(__half(h));
}

// x / s rounded to nearest from y = RN(1/s), with Markstein's one-FMA
// correction (P. Markstein, IBM J. Res. Dev. 34(1), 1990); zeros and
// non-finite quotients are returned as they are.  The tests compare the codes
// this gives with those of a correctly rounded division.
__device__ __forceinline__ float nv_div(float x, float s, float y) {
    const float q = __fmul_rn(x, y);
    if (q == 0.0f || !isfinite(q)) return q;
    const float r = __fmaf_rn(-q, s, x);
    return __fmaf_rn(r, y, q);
}

// One block of 16 fp32 values: scale code and 8 bytes of packed codes.
__device__ __forceinline__ uint32_t nvfp4_block(const float (&v)[16], float s_t, uint32_t (&packed)[2]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t sc = e4m3_code(__fdiv_rn(__fdiv_rn(amax, 6.0f), s_t));
    const float e = __fmul_rn(e4m3_value(sc), s_t);
    packed[0] = packed[1] = 0u;
    if (e != 0.0f) {
        const float y = __frcp_rn(e);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t b = e2m1_pack(nv_div(v[2 * i], e, y), nv_div(v[2 * i + 1], e, y));
            packed[i / 4] |= b << (8 * (i % 4));
        }
    }
    return sc;
}

__device__ __forceinline__ void bf16x16(const uint4& a, const uint4& b, float (&v)[16]) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// ----------------------------------------------------------------------------- quantisers

__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const uint16_t* __restrict__ src, int64_t elems,
                                                         unsigned int* __restrict__ amax_bits) {
    pdl_enter();
    const uint16_t* p = src + (int64_t)blockIdx.y * elems;
    uint32_t m = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < elems; i += stride)
        m = max(m, ((uint32_t)p[i] << 16) & 0x7FFFFFFFu);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(&amax_bits[blockIdx.y], m);
}

__global__ void nvfp4_tensor_scale_kernel(float* scales, int64_t n) {
    pdl_enter();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float amax = __uint_as_float(reinterpret_cast<unsigned int*>(scales)[i]);
    scales[i] = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// One thread per (tensor, row, block slot of the padded scale row).
__global__ void __launch_bounds__(256) nvfp4_quantize_kernel(const uint16_t* __restrict__ src, int64_t n_tensors,
                                                             int64_t rows, int K, const float* __restrict__ tscale,
                                                             uint8_t* __restrict__ codes, uint8_t* __restrict__ bscale) {
    pdl_enter();
    const int nb = K / 16, ksp = (nb + 15) / 16 * 16;
    const int64_t total = n_tensors * rows * ksp;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int b = (int)(i % ksp);
        const int64_t row = i / ksp;           // tensor * rows + r
        if (b >= nb) {
            bscale[row * ksp + b] = 0;
            continue;
        }
        const float s_t = tscale[row / rows];
        const uint4* p = reinterpret_cast<const uint4*>(src + row * K + 16 * b);
        float v[16];
        bf16x16(p[0], p[1], v);
        uint32_t packed[2];
        bscale[row * ksp + b] = (uint8_t)nvfp4_block(v, s_t, packed);
        *reinterpret_cast<uint2*>(codes + row * (K / 2) + 8 * b) = make_uint2(packed[0], packed[1]);
    }
}

// Activation rows: out row r = x[perm_src[r] / K] (or row r when perm_src is null),
// quantised with the static tensor scale s_t.  One warp per row, a lane per block.
__global__ void __launch_bounds__(256) nvfp4_gather_kernel(const uint16_t* __restrict__ x,
                                                           const int32_t* __restrict__ perm_src, int64_t rows,
                                                           int K, int64_t T, int H, float s_t,
                                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ bscale,
                                                           DevCtx ctx) {
    pdl_enter();
    const int lane = threadIdx.x % 32;
    const int nb = H / 16, ksp = (nb + 15) / 16 * 16;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
        int64_t t = r;
        if (perm_src) {
            const int32_t src = perm_src[r];
            t = src / K;
            if (src < 0 || t >= T) {
                if (lane == 0) record_error(ctx.err, MOE_EINDEX);
                continue;
            }
        }
        const uint4* xr = reinterpret_cast<const uint4*>(x + t * H);
        for (int b = lane; b < ksp; b += 32) {
            if (b >= nb) {
                bscale[r * ksp + b] = 0;
                continue;
            }
            float v[16];
            bf16x16(xr[2 * b], xr[2 * b + 1], v);
            uint32_t packed[2];
            bscale[r * ksp + b] = (uint8_t)nvfp4_block(v, s_t, packed);
            *reinterpret_cast<uint2*>(codes + r * (H / 2) + 8 * b) = make_uint2(packed[0], packed[1]);
        }
    }
}

// ----------------------------------------------------------------------------- grouped GEMM

constexpr int FG_THREADS = 320;            // 10 warps
constexpr int FG_BM = 128;                 // weight rows per unit
constexpr int FG_KR = 256;                 // K values per raw (packed) stage
constexpr int FG_KF = 64;                  // K values per fp16 stage (128-byte rows)
constexpr int FG_A_RAW = FG_BM * FG_KR / 2;   // 16 KB of codes
constexpr int FG_A_SC = FG_BM * 16;           // 2 KB of block scales (16 blocks x 128 rows)
constexpr int FG_A_F16 = FG_BM * 128;         // 16 KB
constexpr int FG_TMEM_COLS = 512;

struct Fp4Args {
    const int4* sched;
    const int* n_sched;
    int m_blocks;
    int Nout;
    int Kdim;
    int k_raw;               // ceil(K / 256)
    int k_f16;               // ceil(K / 64)
    int nr, nf;              // ring depths
    int bn;                  // max rows per schedule entry
    const float* w_tscale;   // [E]
    float in_tscale;         // x (up) or H (down) tensor scale
    float out_tscale;        // H tensor scale (up)
    void* out;               // up: H codes [rows][F/2]; down: bf16 [rows][H]
    uint8_t* out_scale;      // up: H block scales [rows][FSP]
    int debug_withhold;
};

struct Fp4Maps {
    CUtensorMap a128, a64;       // weight codes, 128-byte boxes of 128 / 64 rows (SW128)
    CUtensorMap as128, as64;     // weight block scales, 16-byte boxes of 128 / 64 rows
    CUtensorMap b128, b64, b16;  // activation codes (SW128)
    CUtensorMap bs128, bs64, bs16;   // activation block scales
};

__device__ __forceinline__ void e2m1x8_to_f16(uint32_t packed, uint32_t (&out)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3]) : "r"(packed));
}

__device__ __forceinline__ uint32_t e4m3_pair_f16(uint32_t code) {
    uint32_t r;
    const uint16_t two = (uint16_t)(code * 0x0101u);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
    return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// One row of one fp16 stage: 64 values (32 code bytes at chunks 2*sub, 2*sub+1 of a
// 128-byte-swizzled raw row; 4 scale bytes) -> 128 bytes into a 128-byte-swizzled fp16 row.
// Scales of blocks at or beyond nb read as zero.
__device__ __forceinline__ void convert_row(const uint8_t* raw_row, const uint8_t* sc_row, uint8_t* f16_row, int row,
                                            int sub, int kb0, int nb) {
    const int sw = row & 7;
    const uint4 c0 = *reinterpret_cast<const uint4*>(raw_row + 16 * ((2 * sub) ^ sw));
    const uint4 c1 = *reinterpret_cast<const uint4*>(raw_row + 16 * ((2 * sub + 1) ^ sw));
    const uint32_t scw = *reinterpret_cast<const uint32_t*>(sc_row + 4 * sub);
    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
        uint32_t sc = (scw >> (8 * blk)) & 0xFFu;
        if (kb0 + blk >= nb) sc = 0;
        const uint32_t s2 = e4m3_pair_f16(sc);
        uint32_t h[8];
        uint32_t t[4];
        e2m1x8_to_f16(words[2 * blk], t);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = hmul2(t[i], s2);
        e2m1x8_to_f16(words[2 * blk + 1], t);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[4 + i] = hmul2(t[i], s2);
        *reinterpret_cast<uint4*>(f16_row + 16 * ((2 * blk) ^ sw)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(f16_row + 16 * ((2 * blk + 1) ^ sw)) = make_uint4(h[4], h[5], h[6], h[7]);
    }
}

template <bool UP>
__global__ void __launch_bounds__(FG_THREADS, 1)
    grouped_gemm_fp4_kernel(const __grid_constant__ Fp4Maps maps, Fp4Args g, DevCtx ctx) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NR = g.nr, NF = g.nf;
    const int b_raw = g.bn * 128, b_sc = g.bn * 16, b_f16 = g.bn * 128;
    // codes first, then scales; every stage starts on a 1024-byte boundary (128-byte swizzle atoms)
    const int raw_bytes = (FG_A_RAW + b_raw + FG_A_SC + b_sc + 1023) & ~1023;
    const int f16_bytes = FG_A_F16 + b_f16;
    uint8_t* raw = smem;
    uint8_t* f16 = raw + (size_t)NR * raw_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(f16 + (size_t)NF * f16_bytes);
    uint64_t* raw_full = bars;
    uint64_t* raw_empty = raw_full + NR;
    uint64_t* f16_full = raw_empty + NR;
    uint64_t* f16_empty = f16_full + NF;
    uint64_t* tfull = f16_empty + NF;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NR; ++s) {
            mbar_init(smem_u32(&raw_full[s]), 1);
            mbar_init(smem_u32(&raw_empty[s]), 128);   // every converter thread
        }
        for (int s = 0; s < NF; ++s) {
            mbar_init(smem_u32(&f16_full[s]), 128);
            mbar_init(smem_u32(&f16_empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), FG_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();

    const int n_units = (*g.n_sched) * g.m_blocks;
    const int nbk = g.Kdim / 16;   // valid blocks along K

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
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
                const bool a_full = g.Nout - mb * FG_BM > 64;
                const int n16 = (sc.z + 15) / 16;
                const int n128 = n16 / 8, n64 = (n16 % 8) / 4, r16 = n16 % 4;
                const int arows = a_full ? 128 : 64;
                const uint32_t bytes = (uint32_t)(arows * 128 + arows * 16 + n16 * 16 * 128 + n16 * 16 * 16);
                const int a_y = sc.x * g.Nout + mb * FG_BM;
                for (int kr = 0; kr < g.k_raw; ++kr) {
                    if (!mbar_wait(smem_u32(&raw_empty[stage]), phase ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&raw_full[stage]);
                    mbar_arrive_expect_tx(fb, bytes);
                    if (withhold) {
                        withhold = false;   // this stage never completes: the consumers' waits expire
                    } else {
                        uint8_t* st = raw + (size_t)stage * raw_bytes;
                        const uint32_t a_c = smem_u32(st), b_c = smem_u32(st + FG_A_RAW);
                        const uint32_t a_s = smem_u32(st + FG_A_RAW + b_raw), b_s = smem_u32(st + FG_A_RAW + b_raw + FG_A_SC);
                        tma_load_2d(a_c, a_full ? &maps.a128 : &maps.a64, fb, kr * 128, a_y, pol_w);
                        tma_load_2d(a_s, a_full ? &maps.as128 : &maps.as64, fb, kr * 16, a_y, pol_w);
                        int row = 0;
                        for (int j = 0; j < n128; ++j, row += 128) {
                            tma_load_2d(b_c + row * 128, &maps.b128, fb, kr * 128, sc.y + row, pol_x);
                            tma_load_2d(b_s + row * 16, &maps.bs128, fb, kr * 16, sc.y + row, pol_x);
                        }
                        for (int j = 0; j < n64; ++j, row += 64) {
                            tma_load_2d(b_c + row * 128, &maps.b64, fb, kr * 128, sc.y + row, pol_x);
                            tma_load_2d(b_s + row * 16, &maps.bs64, fb, kr * 16, sc.y + row, pol_x);
                        }
                        for (int j = 0; j < r16; ++j, row += 16) {
                            tma_load_2d(b_c + row * 128, &maps.b16, fb, kr * 128, sc.y + row, pol_x);
                            tma_load_2d(b_s + row * 16, &maps.bs16, fb, kr * 16, sc.y + row, pol_x);
                        }
                    }
                    if (++stage == NR) {
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
    } else if (warp >= 6) {
        // ---------------------------------------------------------------- converters
        // The 128 converter threads dequantise the four fp16 stages of every raw stage in order:
        // thread i converts weight row i and the unit's token rows i, i + 128, ...  All of them
        // take the fp16 buffers in the same order and each arrives once per use, so a buffer's
        // full / empty phases advance one use at a time.
        const int i = threadIdx.x - 192;
        int rs = 0, fs = 0;
        uint32_t rph = 0, fph = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            const int4 sc = g.sched[u / g.m_blocks];
            const int mb = u % g.m_blocks;
            const bool a_full = g.Nout - mb * FG_BM > 64;
            const int nrows = ((sc.z + 15) / 16) * 16;
            for (int kr = 0; kr < g.k_raw && ok; ++kr) {
                if (!mbar_wait(smem_u32(&raw_full[rs]), rph, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint8_t* st = raw + (size_t)rs * raw_bytes;
                const uint8_t* a_c = st;
                const uint8_t* b_c = st + FG_A_RAW;
                const uint8_t* a_s = st + FG_A_RAW + b_raw;
                const uint8_t* b_s = a_s + FG_A_SC;
                for (int sub = 0; sub < 4; ++sub) {
                    const int kf = kr * 4 + sub;
                    if (kf >= g.k_f16) break;
                    if (!mbar_wait(smem_u32(&f16_empty[fs]), fph ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* fa = f16 + (size_t)fs * f16_bytes;
                    uint8_t* fbt = fa + FG_A_F16;
                    const int kb0 = kr * 16 + sub * 4;
                    if (a_full || i < 64)
                        convert_row(a_c + i * 128, a_s + i * 16, fa + i * 128, i, sub, kb0, nbk);
                    else
#pragma unroll
                        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(fa + i * 128 + 16 * c) = make_uint4(0, 0, 0, 0);
                    for (int j = i; j < nrows; j += 128)
                        convert_row(b_c + j * 128, b_s + j * 16, fbt + j * 128, j, sub, kb0, nbk);
                    // this thread's fp16 writes become visible to the tensor cores
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive(smem_u32(&f16_full[fs]));
                    if (++fs == NF) {
                        fs = 0;
                        fph ^= 1u;
                    }
                }
                if (!ok) break;
                mbar_arrive(smem_u32(&raw_empty[rs]));
                if (++rs == NR) {
                    rs = 0;
                    rph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            int fs = 0;
            uint32_t fph = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, issued = false;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int4 sc = g.sched[u / g.m_blocks];
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = make_idesc(0u, FG_BM, n_mma);   // fp16 A and B, fp32 accumulate
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
                for (int kf = 0; kf < g.k_f16; ++kf) {
                    if (!mbar_wait(smem_u32(&f16_full[fs]), fph, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(f16 + (size_t)fs * f16_bytes);
                    const uint32_t b_base = a_base + FG_A_F16;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss<false>(d_tmem, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32), idesc,
                                      (kf | kk) != 0 ? 1u : 0u);
                    issued = true;
                    mma_commit(smem_u32(&f16_empty[fs]));
                    if (++fs == NF) {
                        fs = 0;
                        fph ^= 1u;
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
                mma_commit(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2..5)
        const int q = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        const int fsp = (g.Nout / 16 + 15) / 16 * 16;   // padded block-scale row of the H tensor (up)
        for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
            const int4 sc = g.sched[u / g.m_blocks];
            const int mb = u % g.m_blocks;
            if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, ctx, abort_flag)) break;
            tc_fence_after();
            const int f = mb * FG_BM + q * 32 + lane;
            const bool fvalid = f < g.Nout;
            const float scale = __fmul_rn(g.w_tscale[sc.x], g.in_tscale);
            const float r6 = __frcp_rn(6.0f), rts = __frcp_rn(g.out_tscale);   // quotients via nv_div
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
            const int nchunks = (sc.z + 15) / 16;
            for (int c = 0; c < nchunks; ++c) {
                uint32_t v[16];
                tmem_ld16(t_row + (uint32_t)(c * 16), v);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = c * 16 + j;
                    const float z = __fmul_rn(__uint_as_float(v[j]), scale);
                    if constexpr (UP) {
                        // H = relu(z)^2 in blocks of 16 features (this half warp), quantised with s_h
                        const float a = z > 0.0f ? __fmul_rn(z, z) : 0.0f;
                        float amax = a;
#pragma unroll
                        for (int off = 8; off > 0; off >>= 1)
                            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
                        const uint32_t scode = e4m3_code(nv_div(nv_div(amax, 6.0f, r6), g.out_tscale, rts));
                        const float e = __fmul_rn(e4m3_value(scode), g.out_tscale);
                        const float qv = e != 0.0f ? nv_div(a, e, __frcp_rn(e)) : 0.0f;
                        const float qn = __shfl_down_sync(0xffffffffu, qv, 1);   // the odd neighbour
                        if (r < sc.z && fvalid) {
                            const int64_t row = sc.y + r;
                            if ((lane & 1) == 0)
                                static_cast<uint8_t*>(g.out)[row * (g.Nout / 2) + f / 2] =
                                    e != 0.0f ? (uint8_t)e2m1_pack(qv, qn) : (uint8_t)0;
                            if ((lane & 15) == 0) g.out_scale[row * fsp + f / 16] = (uint8_t)scode;
                        }
                    } else {
                        if (r < sc.z && fvalid)
                            static_cast<__nv_bfloat16*>(g.out)[(int64_t)(sc.y + r) * g.Nout + f] =
                                __float2bfloat16_rn(z);
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
        tmem_dealloc(tmem_base, FG_TMEM_COLS);
    }
}

// ----------------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn4)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn4 encode_fn4() {
    static EncodeTiledFn4 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn4>(p);
    }
    return fn;
}

// 2-D byte map over [rows][cols] with row stride `stride` bytes, box box_cols x box_rows.
static bool make_map_u8(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t stride, int box_cols,
                        int box_rows, bool sw128) {
    EncodeTiledFn4 fn = encode_fn4();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)stride};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Fp4Plan {
    int bn, nr, nf;
    size_t smem_bytes;
};

static int ksp_of(int K) { return (K / 16 + 15) / 16 * 16; }

Fp4Plan fp4_plan(int bn) {
    Fp4Plan p;
    p.bn = bn;
    const int raw = (FG_A_RAW + bn * 128 + FG_A_SC + bn * 16 + 1023) & ~1023;
    const int f16 = FG_A_F16 + bn * 128;
    // fp16 buffers: two for the wide tiles of large batches, five when the tiles are small
    const int nf = bn > 64 ? 2 : 5;
    int nr = (220 * 1024 - nf * f16) / raw;
    if (nr > 8) nr = 8;
    if (nr < 2) nr = 2;
    p.nr = nr;
    p.nf = nf;
    p.smem_bytes = 1024 + (size_t)nr * raw + (size_t)nf * f16 + (size_t)(2 * nr + 2 * nf + 5) * 8 + 16;
    return p;
}

size_t nvfp4_scale_row_bytes(int K) { return (size_t)ksp_of(K); }

template <bool UP>
static cudaError_t launch_fp4(const Fp4Maps& maps, const Fp4Args& g, int grid, size_t smem, cudaStream_t stream,
                              const DevCtx& ctx) {
    auto kfn = grouped_gemm_fp4_kernel<UP>;
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch_k(kfn, dim3(grid), dim3(FG_THREADS), smem, stream, maps, g, ctx);
}

// One grouped projection on NVFP4 operands.  W codes [E*Nout][K/2], W scales
// [E*Nout][KSP]; activation codes [rows][K/2], scales [rows][KSP].
// up: out = H codes [rows][Nout/2], out_scale = H block scales [rows][ksp(Nout)].
// down: out = bf16 [rows][Nout].
cudaError_t launch_grouped_gemm_fp4(bool up, const uint8_t* w_codes, const uint8_t* w_scales, const float* w_tscale,
                                    int E, int Nout, int Kdim, const uint8_t* a_codes, const uint8_t* a_scales,
                                    float in_tscale, float out_tscale, int64_t rows, const int4* sched,
                                    const int* n_sched, int bn, int max_sched, void* out, uint8_t* out_scale,
                                    int num_sms, int debug_withhold, const DevCtx& ctx, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    const int ksp = ksp_of(Kdim);
    const int64_t wrows = (int64_t)E * Nout;
    Fp4Maps maps;
    if (!make_map_u8(&maps.a128, w_codes, wrows, Kdim / 2, Kdim / 2, 128, 128, true) ||
        !make_map_u8(&maps.a64, w_codes, wrows, Kdim / 2, Kdim / 2, 128, 64, true) ||
        !make_map_u8(&maps.as128, w_scales, wrows, ksp, ksp, 16, 128, false) ||
        !make_map_u8(&maps.as64, w_scales, wrows, ksp, ksp, 16, 64, false) ||
        !make_map_u8(&maps.b128, a_codes, rows, Kdim / 2, Kdim / 2, 128, 128, true) ||
        !make_map_u8(&maps.b64, a_codes, rows, Kdim / 2, Kdim / 2, 128, 64, true) ||
        !make_map_u8(&maps.b16, a_codes, rows, Kdim / 2, Kdim / 2, 128, 16, true) ||
        !make_map_u8(&maps.bs128, a_scales, rows, ksp, ksp, 16, 128, false) ||
        !make_map_u8(&maps.bs64, a_scales, rows, ksp, ksp, 16, 64, false) ||
        !make_map_u8(&maps.bs16, a_scales, rows, ksp, ksp, 16, 16, false))
        return cudaErrorInvalidValue;
    const Fp4Plan plan = fp4_plan(bn);
    Fp4Args g;
    g.sched = sched;
    g.n_sched = n_sched;
    g.m_blocks = (Nout + FG_BM - 1) / FG_BM;
    g.Nout = Nout;
    g.Kdim = Kdim;
    g.k_raw = (Kdim + FG_KR - 1) / FG_KR;
    g.k_f16 = (Kdim + FG_KF - 1) / FG_KF;
    g.nr = plan.nr;
    g.nf = plan.nf;
    g.bn = bn;
    g.w_tscale = w_tscale;
    g.in_tscale = in_tscale;
    g.out_tscale = out_tscale;
    g.out = out;
    g.out_scale = out_scale;
    g.debug_withhold = debug_withhold;
    const int64_t max_units = (int64_t)max_sched * g.m_blocks;
    const int grid = (int)(max_units < num_sms ? max_units : num_sms);
    return up ? launch_fp4<true>(maps, g, grid, plan.smem_bytes, stream, ctx)
              : launch_fp4<false>(maps, g, grid, plan.smem_bytes, stream, ctx);
}

cudaError_t launch_quantize_nvfp4(int64_t n_tensors, int64_t rows, int K, const uint16_t* src, uint8_t* codes,
                                  uint8_t* bscale, float* tscale, int num_sms, cudaStream_t stream) {
    if (n_tensors == 0 || rows == 0) return cudaSuccess;
    cudaError_t err = cudaMemsetAsync(tscale, 0, (size_t)n_tensors * sizeof(float), stream);
    if (err != cudaSuccess) return err;
    const int64_t elems = rows * K;
    int64_t bx = (elems + 255) / 256;
    const int64_t cap = (n_tensors >= num_sms) ? 4 : (int64_t)num_sms * 8 / n_tensors + 1;
    if (bx > cap) bx = cap;
    for (int64_t t0 = 0; t0 < n_tensors; t0 += 65535) {
        const int64_t nt = n_tensors - t0 < 65535 ? n_tensors - t0 : 65535;
        err = launch_k(nvfp4_amax_kernel, dim3((unsigned)bx, (unsigned)nt), dim3(256), 0, stream, src + t0 * elems,
                       elems, reinterpret_cast<unsigned int*>(tscale) + t0);
        if (err != cudaSuccess) return err;
    }
    err = launch_k(nvfp4_tensor_scale_kernel, dim3((unsigned)((n_tensors + 255) / 256)), dim3(256), 0, stream, tscale,
                   n_tensors);
    if (err != cudaSuccess) return err;
    const int64_t items = n_tensors * rows * ksp_of(K);
    int64_t blocks = (items + 255) / 256;
    if (blocks > (int64_t)num_sms * 16) blocks = (int64_t)num_sms * 16;
    return launch_k(nvfp4_quantize_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, src, n_tensors, rows, K,
                    (const float*)tscale, codes, bscale);
}

cudaError_t launch_gather_nvfp4(const uint16_t* x, const int32_t* perm_src, int64_t rows, int K, int64_t T, int H,
                                float s_t, uint8_t* codes, uint8_t* bscale, int num_sms, const DevCtx& ctx,
                                cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    int64_t blocks = (rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    return launch_k(nvfp4_gather_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, x, perm_src, rows, K, T, H, s_t,
                    codes, bscale, ctx);
}

}  // namespace moe
