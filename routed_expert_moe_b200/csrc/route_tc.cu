// Router on the tensor cores: the logits x Wr^T of a batch as exact integer
// products of fixed-point slices, ranked with a rigorous bound.
//
// The method (bloomery issue page, s.2 "Checkpoint facts": top-6 routing over
// 128 experts; audio.cpp model page, "CPU weight offload": the router and the
// routing-weight formulas) ranks the logits l = x . w_e (+ b_e).  The ranking
// is defined on the fixed-point sum of the exact bf16 products (route.cu);
// this path reaches the same ranking through integer tensor-core products:
//
//   1. router_quant_kernel writes every row v (a token row of x or an expert
//      row of Wr) as integers X_i = rint(v_i 2^q), with q chosen so that
//      |X_i| < 2^22, split into three int8 slices X = 2^16 h + 2^8 m + l
//      (h in [-64, 64], m and l in [-128, 127]), and records q and
//      S = sum_i |X_i|.
//   2. router_mma_kernel multiplies the slices with tcgen05.mma kind::i8
//      (exact int32 accumulation), the nine slice products grouped by their
//      weight into five accumulators A_s (s = 32, 24, 16, 8, 0 bits), one CTA
//      per (32-token tile, range of K), and stores the int32 partials.
//   3. router_select_kernel (one warp per token) adds the partials of the K
//      ranges (exact integer sums) and forms l~ = 2^-(qx+qw) sum_s 2^s A_s,
//      which is sum_i x~_i w~_i of the rounded rows to within the fp64
//      rounding of the last additions.  Since |x_i - x~_i| <= 2^-(qx+1),
//        |l - l~| <= 2^-(qx+qw) (Sx / 2 + Sw / 2 + H / 4),
//      a bound computed from integers.  Each token is ranked with that bound
//      (route_select.cuh): if every gap among the K+1 best exceeds twice the
//      bound the order is certified, else the candidates get their exact
//      fixed-point logits.  As in the other router kernels, a certified
//      token's weights come from its approximate logits l~ (here within about
//      2^-21 of the row scales' product).
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "route_select.cuh"

namespace moe {

namespace {

constexpr int RC_THREADS = 192;   // warp 0 TMA, warp 1 MMA, warps 2-5 TMEM read-out
constexpr int RC_NT = 32;         // tokens per CTA (the MMA's N)
constexpr int RC_ME = 128;        // expert rows per tile (the MMA's M; E <= 128)
constexpr int RC_KB = 128;        // K bytes (int8 values) per stage: one 128-byte swizzled row
constexpr int RC_STAGES = 3;
constexpr int RC_SL = 3;          // int8 slices per row
constexpr int RC_A_BYTES = RC_ME * RC_KB;   // one slice of the expert tile
constexpr int RC_B_BYTES = RC_NT * RC_KB;   // one slice of the token tile
constexpr int RC_STAGE_BYTES = RC_SL * (RC_A_BYTES + RC_B_BYTES);
constexpr int RC_NACC = 5;                  // accumulators by slice weight: 2^32, 2^24, 2^16, 2^8, 1
constexpr int RC_TMEM_COLS = 256;           // RC_NACC x RC_NT columns, rounded up to a power of two
constexpr int RQ_B = 4;                     // 16-byte loads in flight per lane in router_quant_kernel

struct RouterQuantArgs {
    const uint16_t* x;    // [T][H] bf16
    const uint16_t* wr;   // [E][H] bf16
    int64_t T;
    int H, E;
    int8_t* sl;           // [RC_SL][T + E][H]: slices h, m, l; token rows, then expert rows
    int* q;               // [T + E]
    long long* S;         // [T + E]
};

// One warp per row.  The largest biased exponent e1 of the row's values gives
// |v| < 2^(e1 - 126), so q = 148 - e1 keeps |X| = |rint(v 2^q)| < 2^22 (a value
// m8 2^(e - 134), m8 its 8-bit significand, becomes m8 2^(e - e1 + 14), rounded
// to nearest even).
__global__ void __launch_bounds__(256) router_quant_kernel(RouterQuantArgs a, DevCtx ctx) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int nv = a.H / 8;
    const int64_t rows = a.T + a.E;
    for (int64_t r = (int64_t)blockIdx.x * 8 + threadIdx.x / 32; r < rows; r += (int64_t)gridDim.x * 8) {
        const uint4* src = reinterpret_cast<const uint4*>(r < a.T ? a.x + r * a.H : a.wr + (r - a.T) * a.H);
        const size_t plane = (size_t)rows * a.H;
        // X = rint(v 2^q): v (bf16, exact in fp32) times 2^q in two exact power-of-two steps
        // (q may exceed fp32's exponent range), rounded to nearest even by the conversion; a
        // product below 2^-149 would round to X = 0 anyway
        auto emit = [&](const uint4& f, int v, float s1, float s2, long long& S) {
            const uint32_t u[4] = {f.x, f.y, f.z, f.w};
            int X[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                X[2 * j] = __float2int_rn(__fmul_rn(__fmul_rn(__uint_as_float(u[j] << 16), s1), s2));
                X[2 * j + 1] = __float2int_rn(__fmul_rn(__fmul_rn(__uint_as_float(u[j] & 0xFFFF0000u), s1), s2));
            }
            int sa = 0;   // |X| < 2^22: eight of them fit an int
            uint32_t ph[2] = {0u, 0u}, pm[2] = {0u, 0u}, pl[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                sa += abs(X[j]);
                // X = 2^16 h + 2^8 m + l with l, m in [-128, 127]: l is X's low byte as a signed value
                const int lo = (int)(int8_t)(X[j] & 0xFF);
                const int X1 = (X[j] - lo) >> 8;
                const int mi = (int)(int8_t)(X1 & 0xFF);
                const int hi = (X1 - mi) >> 8;
                ph[j >> 2] |= (uint32_t)(hi & 0xFF) << ((j & 3) * 8);
                pm[j >> 2] |= (uint32_t)(mi & 0xFF) << ((j & 3) * 8);
                pl[j >> 2] |= (uint32_t)(lo & 0xFF) << ((j & 3) * 8);
            }
            S += sa;
            int8_t* d = a.sl + r * a.H + 8 * v;
            *reinterpret_cast<uint2*>(d) = make_uint2(ph[0], ph[1]);
            *reinterpret_cast<uint2*>(d + plane) = make_uint2(pm[0], pm[1]);
            *reinterpret_cast<uint2*>(d + 2 * plane) = make_uint2(pl[0], pl[1]);
        };
        auto emax_of = [](const uint4& f) {
            const uint32_t u[4] = {f.x, f.y, f.z, f.w};
            uint32_t m = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) m = max(m, max((u[j] >> 7) & 0xFFu, (u[j] >> 23) & 0xFFu));
            return m;
        };
        uint32_t emax = 0;
        long long S = 0;
        int e1;
        for (int v0 = lane; v0 < nv; v0 += 32 * RQ_B) {
            uint4 f[RQ_B];   // RQ_B loads in flight per lane
#pragma unroll
            for (int b = 0; b < RQ_B; ++b) f[b] = v0 + 32 * b < nv ? src[v0 + 32 * b] : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int b = 0; b < RQ_B; ++b) emax = max(emax, emax_of(f[b]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, off));
        e1 = emax > 0 ? (int)emax : 1;
        const int q = 148 - e1;                      // in [-106, 147]
        const int qa = q > 100 ? 100 : q;
        const float s1 = __uint_as_float((uint32_t)(127 + qa) << 23), s2 = __uint_as_float((uint32_t)(127 + q - qa) << 23);
        for (int v0 = lane; v0 < nv; v0 += 32 * RQ_B) {
            uint4 f[RQ_B];
#pragma unroll
            for (int b = 0; b < RQ_B; ++b) f[b] = v0 + 32 * b < nv ? src[v0 + 32 * b] : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int b = 0; b < RQ_B; ++b)
                if (v0 + 32 * b < nv) emit(f[b], v0 + 32 * b, s1, s2, S);
        }
        if (emax == 0xFFu && lane == 0) record_error(ctx.err, MOE_ERANGE);   // an infinity or NaN
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) S += __shfl_xor_sync(0xffffffffu, S, off);
        if (lane == 0) {
            a.q[r] = q;
            a.S[r] = S;
        }
    }
}

struct RouterTcMaps {
    CUtensorMap x[RC_SL];   // token slices [T][H], box 128 B x RC_NT rows
    CUtensorMap w[RC_SL];   // expert slices [E][H], box 128 B x RC_ME rows
};

struct RouterMmaArgs {
    int64_t T;
    int E;
    int n_k;              // K stages: ceil(H / 128)
    int splits;           // CTAs per token tile, each over its own range of K stages
    int* part;            // [splits][RC_NACC][T][E] int32 partial accumulators
};

__device__ __forceinline__ double pow2i(int k) {   // 2^k, -1022 <= k <= 1023
    return __longlong_as_double((long long)(1023 + k) << 52);
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// Warp-wide bounded wait on phase 0 of `bar` that polls every half microsecond (the
// read-out warps wait out the whole pipeline; frequent polls would take issue slots and
// shared-memory cycles from the TMA and MMA threads).
__device__ __forceinline__ bool wait_sleeping(uint32_t bar, const DevCtx& ctx, volatile int* abort) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(bar, 0)) {
            __nanosleep(500);
            if (*abort) {
                ok = 0;
                break;
            }
            if (globaltimer() - t0 > ctx.timeout_ns) {
                record_error(ctx.err, MOE_ETIMEOUT);
                *abort = 1;
                ok = 0;
                break;
            }
        }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// One CTA per (token tile of RC_NT, split of the K stages).  Warp 0 (one lane)
// streams the split's K stages of the expert and token slices (TMA, 128-byte
// swizzle) through an RC_STAGES ring; warp 1 (one lane) issues 36 MMAs per
// stage (M = 128 experts, N = RC_NT tokens, K = 32 each) into five TMEM
// accumulators; warps 2-5 store them as the split's int32 partials.
__global__ void __launch_bounds__(RC_THREADS, 1)
    router_mma_kernel(const __grid_constant__ RouterTcMaps maps, RouterMmaArgs a, DevCtx ctx) {
    extern __shared__ uint8_t rc_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rc_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + RC_STAGES * RC_STAGE_BYTES);
    uint64_t* empty = full + RC_STAGES;
    uint64_t* done = empty + RC_STAGES;
    uint64_t* drain = done + 1;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 1);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1) + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int tile = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
    const int64_t t0 = (int64_t)tile * RC_NT;
    const int k_begin = (int)((int64_t)split * a.n_k / a.splits), k_end = (int)((int64_t)(split + 1) * a.n_k / a.splits);
    if (threadIdx.x == 0) {
        for (int s = 0; s < RC_STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        mbar_init(smem_u32(done), 1);
        mbar_init(smem_u32(drain), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_holder), RC_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_enter();

    if (warp == 0) {
        if (lane == 0) {
            for (int j = 0; j < RC_SL; ++j) {
                tma_prefetch_desc(&maps.w[j]);
                tma_prefetch_desc(&maps.x[j]);
            }
            const uint64_t pol_w = l2_policy_evict_last();    // the expert slices: read by every CTA
            const uint64_t pol_x = l2_policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int ks = k_begin; ks < k_end; ++ks) {
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = smem_u32(&full[stage]);
                mbar_arrive_expect_tx(fb, RC_STAGE_BYTES);
                const uint32_t base = smem_u32(ring + (size_t)stage * RC_STAGE_BYTES);
                const int kx = ks * RC_KB;
#pragma unroll
                for (int j = 0; j < RC_SL; ++j) {
                    tma_load_2d(base + j * RC_A_BYTES, &maps.w[j], fb, kx, 0, pol_w);
                    tma_load_2d(base + RC_SL * RC_A_BYTES + j * RC_B_BYTES, &maps.x[j], fb, kx, (int)t0, pol_x);
                }
                if (++stage == RC_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                // let loads already in flight land before the block exits
                const uint64_t tw = globaltimer();
                while (globaltimer() - tw < 200000ull) __nanosleep(1000);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // D[e][t] int32, A = expert slices (K-major), B = token slices (K-major), signed x signed
            const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(RC_NT >> 3) << 17) |
                                   ((uint32_t)(RC_ME >> 4) << 24);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int ks = k_begin; ks < k_end; ++ks) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, ctx, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t base = smem_u32(ring + (size_t)stage * RC_STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = (ks > k_begin || kk > 0) ? 1u : 0u;
                    uint64_t da[RC_SL], db[RC_SL];
#pragma unroll
                    for (int j = 0; j < RC_SL; ++j) {
                        da[j] = sw128_desc(base + j * RC_A_BYTES + kk * 32);
                        db[j] = sw128_desc(base + RC_SL * RC_A_BYTES + j * RC_B_BYTES + kk * 32);
                    }
                    // slice i of the expert times slice j of the token weighs 2^(8 (4 - i - j)):
                    // accumulator i + j, started by its first product in this order
#pragma unroll
                    for (int i = 0; i < RC_SL; ++i)
#pragma unroll
                        for (int j = 0; j < RC_SL; ++j) {
                            const bool starts = i + j < RC_SL ? i == 0 : j == RC_SL - 1;
                            mma_i8(tmem_base + (uint32_t)((i + j) * RC_NT), da[i], db[j], idesc, starts ? acc : 1u);
                        }
                }
                issued = true;
                mma_commit(smem_u32(&empty[stage]));
                if (++stage == RC_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) {
                mma_commit(smem_u32(done));
            } else if (issued) {
                // wait for every MMA issued so far before TMEM is released
                mma_commit(smem_u32(drain));
                mbar_wait_drain(smem_u32(drain), 0, ctx.timeout_ns);
            }
        }
    } else if (wait_sleeping(smem_u32(done), ctx, abort_flag)) {
        tc_fence_after();
        const int qd = warp & 3;   // TMEM lane quadrant of this warp: experts 32 qd ..
        const int e = qd * 32 + lane;
        const uint32_t tq = tmem_base + ((uint32_t)(qd * 32) << 16);
        const int64_t TE = a.T * a.E;
        int* out = a.part + (int64_t)split * RC_NACC * TE;
#pragma unroll
        for (int s = 0; s < RC_NACC; ++s) {
#pragma unroll
            for (int h = 0; h < RC_NT / 16; ++h) {
                uint32_t r[16];
                tmem_ld16(tq + (uint32_t)(s * RC_NT + h * 16), r);
                if (e < a.E) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int64_t t = t0 + h * 16 + j;
                        if (t < a.T) out[(int64_t)s * TE + t * a.E + e] = (int)r[j];
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, RC_TMEM_COLS);
    }
}

struct RouterSelectArgs {
    const uint16_t* x;
    const uint16_t* wr;
    const float* bias;    // [E] or null
    int64_t T;
    int H, E, K, splits;
    const int* part;      // [splits][RC_NACC][T][E]
    const int* q;         // [T + E]
    const long long* S;   // [T + E]
    int32_t* idx;         // [T][K]
    float* w;             // [T][K]
};

constexpr int RS_TOK = 8;   // tokens (warps) per block of router_select_kernel

// One warp per token: the token's l~ from the split partials (Horner over the
// accumulator weights, exact integer sums), its bound, the certified ranking;
// the block's open candidates get their exact logits together; then each
// warp finishes its token.
__global__ void __launch_bounds__(RS_TOK * 32) router_select_kernel(RouterSelectArgs a, DevCtx ctx) {
    pdl_enter();
    __shared__ uint8_t c_tok[RS_TOK * RC_ME];
    __shared__ uint16_t c_e[RS_TOK * RC_ME];
    __shared__ long long c_val[RS_TOK * RC_ME];
    __shared__ double Ls[RS_TOK][RC_ME];
    __shared__ int s_oe[RS_TOK][TK_MAXK];
    __shared__ double s_ol[RS_TOK][TK_MAXK];
    __shared__ double cst[3];
    __shared__ int n_cand;
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    const int64_t t_base = (int64_t)blockIdx.x * RS_TOK;
    const int64_t t = t_base + warp;
    const bool active = t < a.T;
    const int E = a.E, H = a.H;
    if (threadIdx.x == 0) n_cand = 0;
    if (warp == 0) {
        // the experts' bound constants: max_e 2^-qw, max_e 2^-qw Sw, max_e |b_e|
        double aw = 0.0, bw = 0.0, bm = 0.0;
        for (int e = lane; e < E; e += 32) {
            const double p = pow2i(-a.q[a.T + e]);
            aw = fmax(aw, p);
            bw = fmax(bw, p * (double)a.S[a.T + e]);
            if (a.bias) bm = fmax(bm, fabs((double)a.bias[e]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            aw = fmax(aw, __shfl_xor_sync(0xffffffffu, aw, off));
            bw = fmax(bw, __shfl_xor_sync(0xffffffffu, bw, off));
            bm = fmax(bm, __shfl_xor_sync(0xffffffffu, bm, off));
        }
        if (lane == 0) {
            cst[0] = aw;
            cst[1] = bw;
            cst[2] = bm;
        }
    }
    int qx = 0;
    long long sx = 0;
    if (active) {
        qx = a.q[t];
        sx = a.S[t];
        const int64_t TE = a.T * (int64_t)E;
        for (int e = lane; e < E; e += 32) {
            int acc[RC_NACC];
#pragma unroll
            for (int s = 0; s < RC_NACC; ++s) acc[s] = 0;
            const int* pp = a.part + t * E + e;
            for (int sp0 = 0; sp0 < a.splits; sp0 += 4) {
                int v[4][RC_NACC];   // the loads of up to four splits in flight
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int s = 0; s < RC_NACC; ++s)
                        v[k][s] = sp0 + k < a.splits ? pp[((int64_t)(sp0 + k) * RC_NACC + s) * TE] : 0;
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int s = 0; s < RC_NACC; ++s) acc[s] += v[k][s];
            }
            double v = 0.0;   // Horner over the weights 2^32 .. 1
#pragma unroll
            for (int s = 0; s < RC_NACC; ++s) v = v * 256.0 + (double)acc[s];
            Ls[warp][e] = v * pow2i(-(qx + a.q[a.T + e]));
        }
    }
    __syncthreads();
    bool certified = true;
    if (active) {
        const double aw = cst[0], bw = cst[1], bm = cst[2];
        const double px = pow2i(-qx);
        // |l~ - l| <= 2^-qx (Sx/2 + H/4) max_e 2^-qw + 2^-qx max_e(2^-qw Sw) / 2; (1 + 2^-48) covers
        // this expression's own roundings
        const double eps = px * (((double)sx * 0.5 + (double)H * 0.25) * aw + bw * 0.5) * (1.0 + 0x1p-48);
        const double lmax = px * (double)sx * aw * 0x1p22;   // >= sum_i |x~_i w~_i| (|W| < 2^22)
        if ((lmax + eps >= 0x1p22 || bm >= 0x1p21) && lane == 0) record_error(ctx.err, MOE_ERANGE);
        // the Horner steps' partial sums stay below sum_i (|X_i| + 2^17)(|W_i| + 2^17) (a slice
        // decomposition exceeds |X| by at most 2^17), which lbig bounds in logit units
        const double lbig = px * aw * ((double)sx + (double)H * 0x1p17) * 0x1p23;
        // + the fixed-point definition's roundings, the four Horner steps' and l~ + b's fp64 roundings
        const double eps_star = eps + (double)(H + 1) * 0x1p-41 + (lbig + bm + 1.0) * 0x1p-50;
        certified = rank_certified_eps(Ls[warp], eps_star, a.bias, E, a.K, lane, warp, s_oe[warp], s_ol[warp],
                                       c_tok, c_e, &n_cand);
    }
    __syncthreads();
    const int nc = n_cand;
    exact_candidates(nc, c_tok, c_e, c_val, t_base, a.x, a.wr, H, a.bias, warp, RS_TOK, lane);
    __syncthreads();
    if (!active) return;
    finish_token(certified, warp, t, nc, c_tok, c_e, c_val, a.K, s_oe[warp], s_ol[warp], lane, a.idx, a.w);
}

typedef CUresult (*EncodeTiledFnR)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnR encode_fn_router() {
    static EncodeTiledFnR fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFnR>(p);
    }
    return fn;
}

// [rows][cols] int8 slices, box 128 bytes x box_rows, 128-byte swizzle; rows past the end read as zero.
bool map_slices(CUtensorMap* m, const int8_t* base, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFnR fn = encode_fn_router();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {(cuuint32_t)RC_KB, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t a256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

// Splits of the K stages per token tile: about one CTA per SM (at most 160 CTAs, 8 splits).
static_assert(RC_NACC * RC_NT <= RC_TMEM_COLS, "accumulators exceed the TMEM allocation");
int route_tc_splits(int64_t T, int H, int num_sms) {
    const int64_t tiles = (T + RC_NT - 1) / RC_NT;
    const int n_k = (H + RC_KB - 1) / RC_KB;
    int64_t sp = (num_sms < 160 ? num_sms : 160) / (tiles > 0 ? tiles : 1);
    if (sp > 8) sp = 8;   // more splits add partials to write and read back for little gain
    if (sp > n_k) sp = n_k;
    return sp < 1 ? 1 : (int)sp;
}

size_t route_tc_scratch_bytes(int64_t T, int H, int E) {
    const size_t rows = (size_t)(T + E);
    // splits x tiles <= min(8 tiles, max(tiles, 160)) (route_tc_splits): the partials of that many tiles
    const int64_t tiles = (T + RC_NT - 1) / RC_NT;
    const int64_t most = tiles > 160 ? tiles : 160;
    const size_t ptok = (size_t)RC_NT * (size_t)(8 * tiles < most ? 8 * tiles : most);
    return a256(RC_SL * rows * (size_t)H) + a256(rows * sizeof(int)) + a256(rows * sizeof(long long)) +
           a256(ptok * RC_NACC * (size_t)E * sizeof(int));
}

cudaError_t launch_route_tc(const uint16_t* x, const uint16_t* wr, const float* bias, int64_t T, int H, int E,
                            int K, int32_t* idx, float* w, void* scratch, int num_sms, const DevCtx& ctx,
                            cudaStream_t stream, void (*between)(cudaStream_t)) {
    if (T == 0) return cudaSuccess;
    // H <= 32768 keeps each accumulator (at most three slice products of |.| <= H 2^14) in int32
    if (E > RC_ME || K > TK_MAXK || H % 16 != 0 || H > 32768 || T + RC_NT > ((int64_t)1 << 31))
        return cudaErrorInvalidValue;
    const size_t rows = (size_t)(T + E);
    uint8_t* b = static_cast<uint8_t*>(scratch);
    int8_t* sl = reinterpret_cast<int8_t*>(b);
    size_t off = a256(RC_SL * rows * H);
    int* q = reinterpret_cast<int*>(b + off);
    off += a256(rows * sizeof(int));
    long long* S = reinterpret_cast<long long*>(b + off);
    off += a256(rows * sizeof(long long));
    int* part = reinterpret_cast<int*>(b + off);

    RouterQuantArgs qa{x, wr, T, H, E, sl, q, S};
    const int64_t qblocks = ((int64_t)rows + 7) / 8;
    cudaError_t err = launch_k(router_quant_kernel, dim3((unsigned)(qblocks < 4096 ? qblocks : 4096)), dim3(256), 0,
                               stream, qa, ctx);
    if (err != cudaSuccess) return err;
    if (between) between(stream);

    RouterTcMaps maps;
    for (int j = 0; j < RC_SL; ++j) {
        const int8_t* p = sl + (size_t)j * rows * H;
        if (!map_slices(&maps.x[j], p, T, H, RC_NT) || !map_slices(&maps.w[j], p + (size_t)T * H, E, H, RC_ME))
            return cudaErrorInvalidValue;
    }
    const int splits = route_tc_splits(T, H, num_sms);
    const int64_t tiles = (T + RC_NT - 1) / RC_NT;
    RouterMmaArgs ma{T, E, (H + RC_KB - 1) / RC_KB, splits, part};
    const size_t smem = 1024 + (size_t)RC_STAGES * RC_STAGE_BYTES + 2 * RC_STAGES * 8 + 16 + 16;
    err = cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    err = launch_k(router_mma_kernel, dim3((unsigned)(tiles * splits)), dim3(RC_THREADS), smem, stream, maps, ma, ctx);
    if (err != cudaSuccess) return err;

    RouterSelectArgs sa{x, wr, bias, T, H, E, K, splits, part, q, S, idx, w};
    return launch_k(router_select_kernel, dim3((unsigned)((T + RS_TOK - 1) / RS_TOK)), dim3(RS_TOK * 32), 0, stream,
                    sa, ctx);
}

}  // namespace moe
