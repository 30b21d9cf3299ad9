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
                                                           int* zero, int64_t n_zero, DevCtx ctx) {
    pdl_enter();
    // counters of the kernel that follows (the one-launch NVFP4 FFN), zero before it starts
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_zero; i += (int64_t)gridDim.x * blockDim.x)
        zero[i] = 0;
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

// The tensor cores multiply NVFP4 operands directly: tcgen05.mma
// kind::mxf4nvf4 with block scaling (scale_vec::4X: one E4M3 scale per 16
// values along K, four per row per instruction of K = 64).  Each MMA reads its
// scale factors from TMEM; tcgen05.cp copies them there from 512-byte atoms in
// shared memory.  An atom holds the four scales of one K block of 64 for 128
// rows, row r = r0 + 32 * r1 at byte 16 * r0 + 4 * r1 (+ the scale index
// 0..3); the copy (32x128b.warpx4) replicates its 32 x 16 bytes into the four
// TMEM lane quadrants, so that the MMA finds row r's scales in lane r,
// column r / 32 of the atom's four columns (B: the same layout over its N
// rows, one atom per 128 rows).  The TMA brings the scales in row-major, 16
// bytes per row per stage, and four "scale" warps rearrange them into atoms.
//
// Roles (320 threads):
//   warp 0      TMA producer: per stage of 256 K values the weight block's
//               codes (128 rows x 128 bytes, 128-byte swizzle) and scales
//               (128 x 16 bytes), the token rows' codes and scales;
//   warp 1      TMEM allocator; one lane copies each stage's atoms to TMEM and
//               issues the four block-scaled MMAs into one of two accumulators;
//   warps 2..5  epilogue: tensor scales, ReLU^2 and the NVFP4 quantisation of
//               H (up) or the bf16 store (down); warp w reads lanes 32*(w%4)..
//               and turns each 32 x 16 tile around in shared memory so that a
//               lane holds one 16-feature block of one token;
//   warps 6..9  scale warps: thread i writes row i's (and row i + 128's)
//               scales into the stage's atoms, zero for rows a tile lacks.
constexpr int FG_THREADS = 320;
constexpr int FG_BM = 128;                    // weight rows per unit (MMA M)
constexpr int FG_KR = 256;                    // K values per stage (128 code bytes per row)
constexpr int FG_A_CODES = FG_BM * 128;       // 16 KB
constexpr int FG_A_SC = FG_BM * 16;           // 2 KB
constexpr int FG_ATOM = 512;                  // scales of one K block of 64 for 128 rows
// TMEM layout: two accumulators of ACC token columns, then the A scales (4 K blocks x 4 columns)
// and the B scales (4 K blocks x 8 columns, two atoms).  Tiles of up to 224 token rows take all
// 512 columns and one CTA per SM; tiles of up to 64 rows (decode) take 256 columns and two CTAs
// per SM, so that one CTA's stage hand-offs (TMA, the scale warps' transposition, barrier waits)
// overlap the other's scale copies and MMAs (the up projection at decode: 139 -> 86 us).
template <bool SMALL>
struct Fp4Tmem {
    static constexpr int COLS = SMALL ? 256 : 512;
    static constexpr int ACC = SMALL ? 64 : 224;
    static constexpr int SFA = 2 * ACC;
    static constexpr int SFB = SFA + 16;
    static constexpr int CTAS = SMALL ? 2 : 1;        // CTAs per SM
    static constexpr int RING = SMALL ? 100 * 1024 : 216 * 1024;
    static_assert(SFB + 32 <= COLS, "TMEM columns");
};
constexpr int FG_BN_MAX = Fp4Tmem<false>::ACC;          // token rows per schedule entry
constexpr int FG_BN_SMALL = Fp4Tmem<true>::ACC;         // at most this many: two CTAs per SM
static_assert(FG_BN_MAX == kFp4MaxTileRows, "NVFP4 tile rows");

struct Fp4Args {
    const int4* sched;
    const int* n_sched;
    int m_blocks;
    int Nout;
    int Kdim;
    int k_stages;            // ceil(K / 256)
    int ns;                  // ring depth
    int bn;                  // max rows per schedule entry (<= the layout's ACC)
    int stage_bytes;
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

// Byte offsets inside one ring stage (codes first: their regions start on 1024-byte boundaries).
struct Fp4Stage {
    int b_codes, a_sc, b_sc, a_atoms, b_atoms, nbat, bytes;
    __host__ __device__ explicit Fp4Stage(int bn) {
        nbat = bn > 128 ? 2 : 1;
        b_codes = FG_A_CODES;
        a_sc = b_codes + bn * 128;
        b_sc = a_sc + FG_A_SC;
        a_atoms = (b_sc + bn * 16 + 127) & ~127;
        b_atoms = a_atoms + 4 * FG_ATOM;
        bytes = (b_atoms + 4 * nbat * FG_ATOM + 1023) & ~1023;
    }
};

// No-swizzle K-major descriptor of one 512-byte scale atom (32 rows of 16 bytes:
// core matrices of 8 rows, 128 bytes apart), the source of tcgen05.cp.
__device__ __forceinline__ uint64_t atom_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(128u >> 4) << 16;
    d |= (uint64_t)(128u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    return d;
}

__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint64_t desc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// Instruction descriptor of the block-scaled MMA: E2M1 A and B (K-major), UE4M3 scales,
// fp32 accumulate, M x N.
__host__ __device__ __forceinline__ uint32_t fp4_idesc(int M, int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                        uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
}

// One stage's scale atoms, by thread i of the 128 scale threads: weight row i's 16 scales (four
// per K block of 64) and token rows i and i + 128, written where tcgen05.cp expects them; rows
// past the tile's rows (arows weight rows, nrows token rows) get zero scales, and scales of blocks
// past K (nbk blocks in all) read as zero whatever the padding bytes hold (the H tensor's padding
// is never written), so that 0 codes times them stay 0.
__device__ __forceinline__ void fp4_stage_atoms(uint8_t* st, const Fp4Stage& L, int i, int arows, int nrows,
                                                int nbk, int ks) {
    const int valid = min(16, max(0, nbk - ks * 16));
    uint4 km;
    km.x = valid >= 4 ? 0xFFFFFFFFu : (valid <= 0 ? 0u : (0xFFFFFFFFu >> (8 * (4 - valid))));
    km.y = valid >= 8 ? 0xFFFFFFFFu : (valid <= 4 ? 0u : (0xFFFFFFFFu >> (8 * (8 - valid))));
    km.z = valid >= 12 ? 0xFFFFFFFFu : (valid <= 8 ? 0u : (0xFFFFFFFFu >> (8 * (12 - valid))));
    km.w = valid >= 16 ? 0xFFFFFFFFu : (valid <= 12 ? 0u : (0xFFFFFFFFu >> (8 * (16 - valid))));
    {
        uint4 v = i < arows ? *reinterpret_cast<const uint4*>(st + L.a_sc + 16 * i) : make_uint4(0u, 0u, 0u, 0u);
        v.x &= km.x;
        v.y &= km.y;
        v.z &= km.z;
        v.w &= km.w;
        uint8_t* at = st + L.a_atoms + 16 * (i % 32) + 4 * (i / 32);
        *reinterpret_cast<uint32_t*>(at) = v.x;
        *reinterpret_cast<uint32_t*>(at + FG_ATOM) = v.y;
        *reinterpret_cast<uint32_t*>(at + 2 * FG_ATOM) = v.z;
        *reinterpret_cast<uint32_t*>(at + 3 * FG_ATOM) = v.w;
    }
    for (int n = i; n < L.nbat * 128; n += 128) {
        uint4 v = n < nrows ? *reinterpret_cast<const uint4*>(st + L.b_sc + 16 * n) : make_uint4(0u, 0u, 0u, 0u);
        v.x &= km.x;
        v.y &= km.y;
        v.z &= km.z;
        v.w &= km.w;
        uint8_t* at = st + L.b_atoms + (n / 128) * FG_ATOM + 16 * (n % 32) + 4 * ((n / 32) % 4);
        const int kstep = L.nbat * FG_ATOM;
        *reinterpret_cast<uint32_t*>(at) = v.x;
        *reinterpret_cast<uint32_t*>(at + kstep) = v.y;
        *reinterpret_cast<uint32_t*>(at + 2 * kstep) = v.z;
        *reinterpret_cast<uint32_t*>(at + 3 * kstep) = v.w;
    }
}

// One stage's scale copies and block-scaled MMAs (nk of K = 64) into d_tmem: the A atoms to
// columns sfa + 4 kk, the B atoms to sfb + 8 kk (+ 4 for a second atom); the first MMA of a
// unit (ks == 0) overwrites the accumulator.
__device__ __forceinline__ void fp4_stage_mma(uint32_t st, const Fp4Stage& L, int nk, uint32_t sfa, uint32_t sfb,
                                              uint32_t d_tmem, uint32_t idesc, int ks) {
    for (int kk = 0; kk < nk; ++kk) {
        tmem_cp_atom(sfa + 4 * kk, atom_desc(st + L.a_atoms + kk * FG_ATOM));
        for (int j = 0; j < L.nbat; ++j)
            tmem_cp_atom(sfb + 8 * kk + 4 * j, atom_desc(st + L.b_atoms + (kk * L.nbat + j) * FG_ATOM));
    }
    for (int kk = 0; kk < nk; ++kk)
        mma_fp4(d_tmem, sw128_desc(st + kk * 32), sw128_desc(st + L.b_codes + kk * 32), idesc, sfa + 4 * kk,
                sfb + 8 * kk, (ks | kk) != 0 ? 1u : 0u);
}

// One chunk of a unit's epilogue: the 16 token columns at t_col of this warp's 32 TMEM lanes
// (features), times `scale`, squared after the ReLU for the up projection, turned around in
// the warp's shared tile tb so that lane (tj + 16 th) holds features f16 .. f16 + 15 of token
// row tj; then, if `store`, the up projection quantises them as one NVFP4 block of H (static
// tensor scale s_h: E4M3 block scale code, E2M1 codes) and the down projection stores bf16 Y.
__device__ __forceinline__ void fp4_epilogue_chunk(uint32_t t_col, float* tb, int lane, bool up, float scale,
                                                   bool store, int64_t row, int f16, int n_out, uint8_t* hc,
                                                   uint8_t* hs, int fsp, __nv_bfloat16* y, float s_h, float r6,
                                                   float rts) {
    const int tj = lane & 15, th = lane >> 4;
    uint32_t v[16];
    tmem_ld16(t_col, v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float z = __fmul_rn(__uint_as_float(v[j]), scale);
        if (up) z = z > 0.0f ? __fmul_rn(z, z) : 0.0f;   // H = relu(z)^2
        tb[j * 32 + (((lane >> 2) ^ (j & 7)) << 2) + (lane & 3)] = z;
    }
    __syncwarp();
    float a[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 t4 = *reinterpret_cast<const float4*>(tb + tj * 32 + (((4 * th + k) ^ (tj & 7)) << 2));
        a[4 * k] = t4.x;
        a[4 * k + 1] = t4.y;
        a[4 * k + 2] = t4.z;
        a[4 * k + 3] = t4.w;
    }
    __syncwarp();
    if (!store) return;
    if (up) {
        // one block of 16 features, quantised with the static tensor scale s_h
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, a[i]);
        const uint32_t scode = e4m3_code(nv_div(nv_div(amax, 6.0f, r6), s_h, rts));
        const float e = __fmul_rn(e4m3_value(scode), s_h);
        uint32_t packed[2] = {0u, 0u};
        if (e != 0.0f) {
            const float yv = __frcp_rn(e);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                packed[i / 4] |= e2m1_pack(nv_div(a[2 * i], e, yv), nv_div(a[2 * i + 1], e, yv)) << (8 * (i % 4));
        }
        *reinterpret_cast<uint2*>(hc + row * (n_out / 2) + f16 / 2) = make_uint2(packed[0], packed[1]);
        hs[row * fsp + f16 / 16] = (uint8_t)scode;
    } else {
        uint32_t w8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const __nv_bfloat162 p2 = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
            w8[i] = *reinterpret_cast<const uint32_t*>(&p2);
        }
        uint4* d4 = reinterpret_cast<uint4*>(y + row * n_out + f16);
        d4[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
        d4[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
    }
}

template <bool UP, bool SMALL>
__global__ void __launch_bounds__(FG_THREADS, Fp4Tmem<SMALL>::CTAS)
    grouped_gemm_fp4_kernel(const __grid_constant__ Fp4Maps maps, Fp4Args g, DevCtx ctx) {
    using TM = Fp4Tmem<SMALL>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NS = g.ns;
    const Fp4Stage L(g.bn);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)NS * L.bytes);
    uint64_t* full = bars;             // the stage's TMA bytes have landed
    uint64_t* sfready = full + NS;     // its scale atoms are written (128 scale threads)
    uint64_t* empty = sfready + NS;    // its MMAs are complete
    uint64_t* tfull = empty + NS;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;
    float* tbuf = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(tmem_holder + 1) + 15) &
                                           ~static_cast<uintptr_t>(15));   // 4 x (16 x 32) fp32

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&sfready[s]), 128);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), TM::COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();

    const int n_units = (*g.n_sched) * g.m_blocks;

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
                const uint32_t bytes = (uint32_t)(arows * (128 + 16) + n16 * 16 * (128 + 16));
                const int a_y = sc.x * g.Nout + mb * FG_BM;
                for (int ks = 0; ks < g.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_arrive_expect_tx(fb, bytes);
                    if (withhold) {
                        withhold = false;   // this stage never completes: the consumers' waits expire
                    } else {
                        const uint32_t st = smem_u32(smem + (size_t)stage * L.bytes);
                        const uint32_t b_c = st + L.b_codes, a_s = st + L.a_sc, b_s = st + L.b_sc;
                        tma_load_2d(st, a_full ? &maps.a128 : &maps.a64, fb, ks * 128, a_y, pol_w);
                        tma_load_2d(a_s, a_full ? &maps.as128 : &maps.as64, fb, ks * 16, a_y, pol_w);
                        int row = 0;
                        for (int j = 0; j < n128; ++j, row += 128) {
                            tma_load_2d(b_c + row * 128, &maps.b128, fb, ks * 128, sc.y + row, pol_x);
                            tma_load_2d(b_s + row * 16, &maps.bs128, fb, ks * 16, sc.y + row, pol_x);
                        }
                        for (int j = 0; j < n64; ++j, row += 64) {
                            tma_load_2d(b_c + row * 128, &maps.b64, fb, ks * 128, sc.y + row, pol_x);
                            tma_load_2d(b_s + row * 16, &maps.bs64, fb, ks * 16, sc.y + row, pol_x);
                        }
                        for (int j = 0; j < r16; ++j, row += 16) {
                            tma_load_2d(b_c + row * 128, &maps.b16, fb, ks * 128, sc.y + row, pol_x);
                            tma_load_2d(b_s + row * 16, &maps.bs16, fb, ks * 16, sc.y + row, pol_x);
                        }
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
    } else if (warp >= 6) {
        // ---------------------------------------------------------------- scale warps
        // Thread i moves weight row i's 16 scales (four per K block) and token rows i and
        // i + 128 into the stage's atoms; rows past the tile's rows get zero scales, so
        // their (unstored) products are zero rather than whatever the smem held.
        const int i = threadIdx.x - 192;
        const int nbk = g.Kdim / 16;   // scale blocks along K; the rest of a padded scale row is masked
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
            const int4 sc = g.sched[u / g.m_blocks];
            const int mb = u % g.m_blocks;
            const int arows = g.Nout - mb * FG_BM > 64 ? 128 : 64;
            const int nrows = (sc.z + 15) / 16 * 16;
            for (int ks = 0; ks < g.k_stages; ++ks) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + (size_t)stage * L.bytes;
                fp4_stage_atoms(st, L, i, arows, nrows, nbk, ks);
                // the atoms become visible to the tensor cores' copies
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(smem_u32(&sfready[stage]));
                if (++stage == NS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, issued = false;
            const uint32_t sfa = tmem_base + TM::SFA, sfb = tmem_base + TM::SFB;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int4 sc = g.sched[u / g.m_blocks];
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = fp4_idesc(FG_BM, n_mma);
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TM::ACC);
                for (int ks = 0; ks < g.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&sfready[stage]), phase, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + (size_t)stage * L.bytes);
                    const int left = g.Kdim - ks * FG_KR;                 // K values of this stage
                    const int nk = left >= FG_KR ? 4 : (left + 63) / 64;   // MMAs of K = 64
                    fp4_stage_mma(st, L, nk, sfa, sfb, d_tmem, idesc, ks);
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
                mma_commit(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2..5)
        // A warp reads 32 weight rows (features) x 16 token columns from TMEM, one feature per
        // lane, and turns the tile around through shared memory: each lane then holds 16
        // consecutive features of one token -- exactly one NVFP4 block of H (up), or 32 bytes
        // of bf16 Y (down) -- so the block amax needs no shuffles, the block's scale and its
        // reciprocal are computed once, and the stores are 8- or 32-byte vectors.
        const int q = warp & 3;
        float* tb = tbuf + (warp - 2) * (16 * 32);
        const int tj = lane & 15, th = lane >> 4;
        int acc = 0;
        uint32_t acc_phase = 0;
        const int fsp = (g.Nout / 16 + 15) / 16 * 16;   // padded block-scale row of the H tensor (up)
        const float r6 = __frcp_rn(6.0f), rts = __frcp_rn(g.out_tscale);   // quotients via nv_div
        for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
            const int4 sc = g.sched[u / g.m_blocks];
            const int mb = u % g.m_blocks;
            if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, ctx, abort_flag)) break;
            tc_fence_after();
            const int f16 = mb * FG_BM + q * 32 + th * 16;   // first feature of this lane's block
            const float scale = __fmul_rn(g.w_tscale[sc.x], g.in_tscale);
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TM::ACC);
            const int nchunks = (sc.z + 15) / 16;
            for (int c = 0; c < nchunks; ++c) {
                const int r = c * 16 + tj;
                fp4_epilogue_chunk(t_row + (uint32_t)(c * 16), tb, lane, UP, scale, r < sc.z && f16 < g.Nout,
                                   sc.y + r, f16, g.Nout, static_cast<uint8_t*>(g.out), g.out_scale, fsp,
                                   static_cast<__nv_bfloat16*>(g.out), g.out_tscale, r6, rts);
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
        tmem_dealloc(tmem_base, TM::COLS);
    }
}

// ----------------------------------------------------------------------------- one-launch FFN

// Both NVFP4 projections in one persistent launch, as the bf16 one-launch FFN (grouped_ffn.cu)
// does it: every up unit (schedule entry x 128-row block of F), then every down unit (entry x
// block of H), claimed in that order from a global counter by each CTA's producer and passed to
// the MMA thread, the scale warps and the epilogue warps through a small queue in shared
// memory.  An up unit's epilogue warps store their rows of H (codes and block scales), fence
// them for the async proxy and each add 1 to done[entry] with release semantics; the producer
// of a down unit waits (bounded) until done[entry] reaches 4 x (blocks of F) before it loads
// the entry's H.  Units are claimed in list order and processed in claim order, so every up
// unit a down unit waits for belongs to a running CTA that needs nothing else to finish it.
constexpr int FF4_UQ = 4;   // unit queue slots

struct Fp4FfnArgs {
    int* claim;              // unit counter (zero at launch; right after done[])
    int* done;               // [max_sched] up epilogue warps finished per entry (zero at launch)
    const int4* sched;
    const int* n_sched;
    int m_up, m_down;        // 128-row blocks of F and of H
    int F, H;
    int k_up, k_down;        // 256-value K stages of H and of F
    int ns;                  // ring depth
    int bn;                  // max rows per schedule entry (<= the layout's ACC)
    const float* wu_tscale;  // [E]
    const float* wd_tscale;  // [E]
    float x_tscale, h_tscale;
    uint8_t* hb;             // H codes [rows][F/2]
    uint8_t* hb_block;       // H block scales [rows][ksp(F)]
    void* y;                 // bf16 [rows][H]
    int debug_hold;          // 1: the list's first up unit never reports its rows (a wait must expire)
};

struct Fp4FfnMaps {
    Fp4Maps up, down;
};

struct Fp4Unit {
    bool up;
    int s, mb;               // schedule entry, 128-row block of the projection's outputs
    int Nout, Kdim, k_stages;
};

__device__ __forceinline__ Fp4Unit fp4_unit(const Fp4FfnArgs& g, int u, int n_up) {
    Fp4Unit r;
    r.up = u < n_up;
    const int v = r.up ? u : u - n_up;
    const int m = r.up ? g.m_up : g.m_down;
    r.s = v / m;
    r.mb = v % m;
    r.Nout = r.up ? g.F : g.H;
    r.Kdim = r.up ? g.H : g.F;
    r.k_stages = r.up ? g.k_up : g.k_down;
    return r;
}

template <bool SMALL>
__global__ void __launch_bounds__(FG_THREADS, Fp4Tmem<SMALL>::CTAS)
    grouped_ffn_fp4_kernel(const __grid_constant__ Fp4FfnMaps maps, Fp4FfnArgs g, DevCtx ctx) {
    using TM = Fp4Tmem<SMALL>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int NS = g.ns;
    const Fp4Stage L(g.bn);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)NS * L.bytes);
    uint64_t* full = bars;
    uint64_t* sfready = full + NS;
    uint64_t* empty = sfready + NS;
    uint64_t* tfull = empty + NS;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;
    float* tbuf = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(tmem_holder + 1) + 15) &
                                           ~static_cast<uintptr_t>(15));   // 4 x (16 x 32) fp32
    // the unit queue: the units this block claimed, in claim order
    uint64_t* uq_full = reinterpret_cast<uint64_t*>(tbuf + 4 * 16 * 32);
    uint64_t* uq_empty = uq_full + FF4_UQ;
    volatile int* uq = reinterpret_cast<volatile int*>(uq_empty + FF4_UQ);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&sfready[s]), 128);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        for (int q = 0; q < FF4_UQ; ++q) {
            mbar_init(smem_u32(&uq_full[q]), 1);
            mbar_init(smem_u32(&uq_empty[q]), 1 + 4 + 4);   // the MMA thread, 4 epilogue and 4 scale warps
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
                if (++qs == FF4_UQ) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (u < 0) break;
                claim = atomicAdd(g.claim, 1);   // the next unit, claimed while this one loads
                const Fp4Unit un = fp4_unit(g, u, n_up);
                const Fp4Maps& mp = un.up ? maps.up : maps.down;
                const int4 sc = g.sched[un.s];
                const bool a_full = un.Nout - un.mb * FG_BM > 64;
                const int n16 = (sc.z + 15) / 16;
                const int n128 = n16 / 8, n64 = (n16 % 8) / 4, r16 = n16 % 4;
                const int arows = a_full ? 128 : 64;
                const uint32_t bytes = (uint32_t)(arows * (128 + 16) + n16 * 16 * (128 + 16));
                const int a_y = sc.x * un.Nout + un.mb * FG_BM;
                if (!un.up) {
                    // the rows of H this unit reads are written by the up units of its entry
                    if (!wait_count(g.done + un.s, up_target, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();
                }
                for (int ks = 0; ks < un.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_arrive_expect_tx(fb, bytes);
                    const uint32_t st = smem_u32(smem + (size_t)stage * L.bytes);
                    const uint32_t b_c = st + L.b_codes, a_s = st + L.a_sc, b_s = st + L.b_sc;
                    tma_load_2d(st, a_full ? &mp.a128 : &mp.a64, fb, ks * 128, a_y, pol_w);
                    tma_load_2d(a_s, a_full ? &mp.as128 : &mp.as64, fb, ks * 16, a_y, pol_w);
                    int row = 0;
                    for (int j = 0; j < n128; ++j, row += 128) {
                        tma_load_2d(b_c + row * 128, &mp.b128, fb, ks * 128, sc.y + row, pol_x);
                        tma_load_2d(b_s + row * 16, &mp.bs128, fb, ks * 16, sc.y + row, pol_x);
                    }
                    for (int j = 0; j < n64; ++j, row += 64) {
                        tma_load_2d(b_c + row * 128, &mp.b64, fb, ks * 128, sc.y + row, pol_x);
                        tma_load_2d(b_s + row * 16, &mp.bs64, fb, ks * 16, sc.y + row, pol_x);
                    }
                    for (int j = 0; j < r16; ++j, row += 16) {
                        tma_load_2d(b_c + row * 128, &mp.b16, fb, ks * 128, sc.y + row, pol_x);
                        tma_load_2d(b_s + row * 16, &mp.bs16, fb, ks * 16, sc.y + row, pol_x);
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
    } else if (warp >= 6) {
        // ---------------------------------------------------------------- scale warps
        // Thread i moves weight row i's 16 scales (four per K block) and token rows i and
        // i + 128 into the stage's atoms; rows past the tile's rows get zero scales.
        const int i = threadIdx.x - 192;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int qs = 0;
        uint32_t qph = 0;
        // Every lane waits on the barrier itself (it then sees the TMA's bytes) and the warp
        // votes, so that a lane that gave up alone cannot split its warp's control flow.
        auto wait_all = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, ctx, abort_flag)) != 0;
        };
        while (ok) {
            if (!wait_all(smem_u32(&uq_full[qs]), qph)) break;
            const int u = uq[qs];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&uq_empty[qs]));
            if (++qs == FF4_UQ) {
                qs = 0;
                qph ^= 1u;
            }
            if (u < 0) break;
            const Fp4Unit un = fp4_unit(g, u, n_up);
            const int4 sc = g.sched[un.s];
            const int arows = un.Nout - un.mb * FG_BM > 64 ? 128 : 64;
            const int nrows = (sc.z + 15) / 16 * 16;
            const int nbk = un.Kdim / 16;   // scale blocks along K; the rest of a padded scale row is masked
            for (int ks = 0; ks < un.k_stages; ++ks) {
                if (!wait_all(smem_u32(&full[stage]), phase)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + (size_t)stage * L.bytes;
                fp4_stage_atoms(st, L, i, arows, nrows, nbk, ks);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(smem_u32(&sfready[stage]));
                if (++stage == NS) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true, issued = false;
            int qs = 0;
            uint32_t qph = 0;
            const uint32_t sfa = tmem_base + TM::SFA, sfb = tmem_base + TM::SFB;
            while (ok) {
                if (!mbar_wait(smem_u32(&uq_full[qs]), qph, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                const int u = uq[qs];
                mbar_arrive(smem_u32(&uq_empty[qs]));
                if (++qs == FF4_UQ) {
                    qs = 0;
                    qph ^= 1u;
                }
                if (u < 0) break;
                const Fp4Unit un = fp4_unit(g, u, n_up);
                const int4 sc = g.sched[un.s];
                const int n_mma = max(16, (sc.z + 15) & ~15);
                const uint32_t idesc = fp4_idesc(FG_BM, n_mma);
                if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TM::ACC);
                for (int ks = 0; ks < un.k_stages; ++ks) {
                    if (!mbar_wait(smem_u32(&sfready[stage]), phase, ctx, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + (size_t)stage * L.bytes);
                    const int left = un.Kdim - ks * FG_KR;
                    const int nk = left >= FG_KR ? 4 : (left + 63) / 64;
                    fp4_stage_mma(st, L, nk, sfa, sfb, d_tmem, idesc, ks);
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
                mma_commit(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2..5)
        // As in grouped_gemm_fp4_kernel: a warp reads 32 features x 16 token columns from TMEM
        // and turns the tile around in shared memory, so that a lane holds one 16-feature block
        // of one token.  Up units quantise H to NVFP4 and report their rows; down units store Y.
        const int q = warp & 3;
        float* tb = tbuf + (warp - 2) * (16 * 32);
        const int tj = lane & 15, th = lane >> 4;
        int acc = 0;
        uint32_t acc_phase = 0;
        int qs = 0;
        uint32_t qph = 0;
        const int fsp = (g.F / 16 + 15) / 16 * 16;   // padded block-scale row of the H tensor
        const float r6 = __frcp_rn(6.0f), rts = __frcp_rn(g.h_tscale);   // quotients via nv_div
        while (true) {
            if (!mbar_wait_warp(smem_u32(&uq_full[qs]), qph, ctx, abort_flag)) break;
            const int u = uq[qs];
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&uq_empty[qs]));
            if (++qs == FF4_UQ) {
                qs = 0;
                qph ^= 1u;
            }
            if (u < 0) break;
            const Fp4Unit un = fp4_unit(g, u, n_up);
            const int4 sc = g.sched[un.s];
            if (!mbar_wait_warp(smem_u32(&tfull[acc]), acc_phase, ctx, abort_flag)) break;
            tc_fence_after();
            const int f16 = un.mb * FG_BM + q * 32 + th * 16;   // first feature of this lane's block
            const float scale = un.up ? __fmul_rn(g.wu_tscale[sc.x], g.x_tscale)
                                      : __fmul_rn(g.wd_tscale[sc.x], g.h_tscale);
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TM::ACC);
            const int nchunks = (sc.z + 15) / 16;
            for (int c = 0; c < nchunks; ++c) {
                const int r = c * 16 + tj;
                fp4_epilogue_chunk(t_row + (uint32_t)(c * 16), tb, lane, un.up, scale, r < sc.z && f16 < un.Nout,
                                   sc.y + r, f16, un.Nout, g.hb, g.hb_block, fsp, static_cast<__nv_bfloat16*>(g.y),
                                   g.h_tscale, r6, rts);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));
            if (un.up) {
                // this warp's rows of H are complete: every lane orders its stores for the async
                // proxy (the TMA loads of H), the warp barrier orders them before lane 0's release
                fence_proxy_async_global();
                __syncwarp();
                const bool hold = g.debug_hold && u == 0;
                if (lane == 0 && !hold) red_release_add(g.done + un.s, 1);
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

static int ksp_of(int K) { return (K / 16 + 15) / 16 * 16; }

// The maps of one projection: weight codes [E*Nout][K/2] and block scales [E*Nout][KSP(K)],
// activation codes [rows][K/2] and block scales [rows][KSP(K)].
static bool make_fp4_maps(Fp4Maps* m, const uint8_t* w_codes, const uint8_t* w_scales, int E, int Nout, int Kdim,
                          const uint8_t* a_codes, const uint8_t* a_scales, int64_t rows) {
    const int ksp = ksp_of(Kdim);
    const int64_t wrows = (int64_t)E * Nout;
    return make_map_u8(&m->a128, w_codes, wrows, Kdim / 2, Kdim / 2, 128, 128, true) &&
           make_map_u8(&m->a64, w_codes, wrows, Kdim / 2, Kdim / 2, 128, 64, true) &&
           make_map_u8(&m->as128, w_scales, wrows, ksp, ksp, 16, 128, false) &&
           make_map_u8(&m->as64, w_scales, wrows, ksp, ksp, 16, 64, false) &&
           make_map_u8(&m->b128, a_codes, rows, Kdim / 2, Kdim / 2, 128, 128, true) &&
           make_map_u8(&m->b64, a_codes, rows, Kdim / 2, Kdim / 2, 128, 64, true) &&
           make_map_u8(&m->b16, a_codes, rows, Kdim / 2, Kdim / 2, 128, 16, true) &&
           make_map_u8(&m->bs128, a_scales, rows, ksp, ksp, 16, 128, false) &&
           make_map_u8(&m->bs64, a_scales, rows, ksp, ksp, 16, 64, false) &&
           make_map_u8(&m->bs16, a_scales, rows, ksp, ksp, 16, 16, false);
}

// Ring depth of the NVFP4 kernel for entries of up to bn token rows: as many stages as fit in
// the layout's ring budget (216 KB, or 100 KB with two CTAs per SM), at most 8; then the
// barriers and the epilogue's 8 KB turn-around tiles.
static int fp4_stages(int bn, bool small, size_t* smem) {
    const Fp4Stage L(bn);
    int ns = (small ? Fp4Tmem<true>::RING : Fp4Tmem<false>::RING) / L.bytes;
    if (ns > 8) ns = 8;
    if (ns < 2) ns = 2;
    *smem = 1024 + (size_t)ns * L.bytes + (size_t)(3 * ns + 5) * 8 + 32 + 4 * 16 * 32 * sizeof(float);
    return ns;
}

size_t nvfp4_scale_row_bytes(int K) { return (size_t)ksp_of(K); }

template <bool UP, bool SMALL>
static cudaError_t launch_fp4(const Fp4Maps& maps, const Fp4Args& g, int grid, size_t smem, cudaStream_t stream,
                              const DevCtx& ctx) {
    auto kfn = grouped_gemm_fp4_kernel<UP, SMALL>;
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
    Fp4Maps maps;
    if (!make_fp4_maps(&maps, w_codes, w_scales, E, Nout, Kdim, a_codes, a_scales, rows))
        return cudaErrorInvalidValue;
    if (bn > FG_BN_MAX) return cudaErrorInvalidValue;
    const bool small = bn <= FG_BN_SMALL;
    size_t smem = 0;
    Fp4Args g;
    g.ns = fp4_stages(bn, small, &smem);
    g.stage_bytes = Fp4Stage(bn).bytes;
    g.sched = sched;
    g.n_sched = n_sched;
    g.m_blocks = (Nout + FG_BM - 1) / FG_BM;
    g.Nout = Nout;
    g.Kdim = Kdim;
    g.k_stages = (Kdim + FG_KR - 1) / FG_KR;
    g.bn = bn;
    g.w_tscale = w_tscale;
    g.in_tscale = in_tscale;
    g.out_tscale = out_tscale;
    g.out = out;
    g.out_scale = out_scale;
    g.debug_withhold = debug_withhold;
    const int64_t max_units = (int64_t)max_sched * g.m_blocks;
    const int64_t slots = (int64_t)num_sms * (small ? Fp4Tmem<true>::CTAS : Fp4Tmem<false>::CTAS);
    const int grid = (int)(max_units < slots ? max_units : slots);
    if (small)
        return up ? launch_fp4<true, true>(maps, g, grid, smem, stream, ctx)
                  : launch_fp4<false, true>(maps, g, grid, smem, stream, ctx);
    return up ? launch_fp4<true, false>(maps, g, grid, smem, stream, ctx)
              : launch_fp4<false, false>(maps, g, grid, smem, stream, ctx);
}

// Both NVFP4 projections in one launch.  done: max_sched + 1 ints (the per-entry counters, then
// the unit claim counter), zero before the launch.  The H codes and block scales go to hb and
// hb_block; Y (bf16 [rows][H]) to y.
cudaError_t launch_grouped_ffn_fp4(const uint8_t* wu_codes, const uint8_t* wu_scales, const float* wu_tscale,
                                   const uint8_t* wd_codes, const uint8_t* wd_scales, const float* wd_tscale, int E,
                                   int F, int H, const uint8_t* x_codes, const uint8_t* x_scales, float x_tscale,
                                   float h_tscale, uint8_t* hb, uint8_t* hb_block, void* y, int64_t rows,
                                   const int4* sched, const int* n_sched, int bn, int max_sched, int* done,
                                   int num_sms, int debug_hold, const DevCtx& ctx, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    Fp4FfnMaps maps;
    if (!make_fp4_maps(&maps.up, wu_codes, wu_scales, E, F, H, x_codes, x_scales, rows) ||
        !make_fp4_maps(&maps.down, wd_codes, wd_scales, E, H, F, hb, hb_block, rows))
        return cudaErrorInvalidValue;
    if (bn > FG_BN_MAX) return cudaErrorInvalidValue;
    const bool small = bn <= FG_BN_SMALL;
    size_t smem = 0;
    Fp4FfnArgs g;
    g.ns = fp4_stages(bn, small, &smem);
    smem += 16 + 2 * FF4_UQ * sizeof(uint64_t) + FF4_UQ * sizeof(int);   // the unit queue (after the tiles)
    g.bn = bn;
    g.done = done;
    g.claim = done + max_sched;
    g.sched = sched;
    g.n_sched = n_sched;
    g.m_up = (F + FG_BM - 1) / FG_BM;
    g.m_down = (H + FG_BM - 1) / FG_BM;
    g.F = F;
    g.H = H;
    g.k_up = (H + FG_KR - 1) / FG_KR;
    g.k_down = (F + FG_KR - 1) / FG_KR;
    g.wu_tscale = wu_tscale;
    g.wd_tscale = wd_tscale;
    g.x_tscale = x_tscale;
    g.h_tscale = h_tscale;
    g.hb = hb;
    g.hb_block = hb_block;
    g.y = y;
    g.debug_hold = debug_hold;
    const int64_t max_units = (int64_t)max_sched * (g.m_up + g.m_down);
    const int64_t slots = (int64_t)num_sms * (small ? Fp4Tmem<true>::CTAS : Fp4Tmem<false>::CTAS);
    const int grid = (int)(max_units < slots ? max_units : slots);
    auto kfn = small ? grouped_ffn_fp4_kernel<true> : grouped_ffn_fp4_kernel<false>;
    cudaError_t err = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    return launch_k(kfn, dim3(grid), dim3(FG_THREADS), smem, stream, maps, g, ctx);
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
                                cudaStream_t stream, int* zero, int64_t n_zero) {
    if (rows == 0) return cudaSuccess;
    int64_t blocks = (rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    return launch_k(nvfp4_gather_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, x, perm_src, rows, K, T, H, s_t,
                    codes, bscale, zero, n_zero, ctx);
}

}  // namespace moe
