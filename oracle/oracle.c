/*
 * ORACLE — test infrastructure only.
 *
 * A plain, slow, obviously correct CPU statement of the routed
 * mixture-of-experts layer, in fp64 (IEEE double) unless a step names
 * another precision.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file's library; the product path never
 * does, and this file shares no code, header or table with the CUDA path.
 *
 * Sources (web pages, cited by title and section):
 *  [B] bloomery issue "Nemotron 3.5 Transcribe from safetensors on x86 cards
 *      and DGX Spark", section 2 "Checkpoint facts": hidden width 2688, top-6
 *      routing over 128 experts, ungated ReLU^2 experts of width 1856, 23 MoE
 *      layers; "FP8 uses scalar-scale E4M3 W8A8".  Section 3 "Existing owners
 *      and gaps": experts have ungated up/down parts (no gate stack).
 *  [A] audio.cpp "nemotron_transcribe" model page, section "CPU weight
 *      offload": offloading changes neither the router, the expert activation
 *      nor the routing-weight formulas, only the rounding of the grouped
 *      expert matrix products; section "Q4_K, Q3_K and Q2_K expert profiles":
 *      zero-padding the routed banks' input columns, with matching zero
 *      activations, leaves outputs, routing and normalisation unchanged.
 *  The gating function, renormalisation and tie rule are not on the pages;
 *  the workload statement fixes them: softmax over the logits, top-k
 *  renormalised, ties to the lower expert index.
 *
 * Readings where the pages are silent (each is stated where it is used):
 *  - logits are summed in fixed point (see oracle_router_logits_fx);
 *  - no routed scaling factor, no expert biases, no capacity limit;
 *  - weight banks are [out][in] (the input index contiguous);
 *  - FP8 E4M3 is the OCP "fn" format with saturation to +-448.
 *
 * Parity status: every function here is pinned by CPU tests against brute
 * force, closed forms, invariants or a library routine; see tests/.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Exact widening of a bf16 bit pattern. */
static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float bf16_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* float -> bf16, round to nearest even (the usual definition on bit patterns). */
static uint16_t float_to_bf16(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

#define FX_SHIFT 40 /* fixed-point resolution of the router logits: 2^-40 */

/*
 * Router logits.  [B] s.2 (top-6 over 128 experts); the router is a linear
 * map of the token's hidden state, l_e = sum_h x_h * Wr[e,h] (+ b_e).
 *
 * Reading: the sum is taken in fixed point.  Each product of two bf16 values
 * is exact in double; it is scaled by 2^40 and rounded to the nearest
 * integer (ties to even), and the integers are added exactly in int64.  The
 * result is within H * 2^-41 of the real-valued sum, and, being an exact
 * integer sum, does not depend on the order of the additions, so any two
 * implementations that follow this reading rank the experts identically.
 * The bias (fp32) is rounded to the same grid and added.
 * L[t*E + e] receives the logit in units of 2^-40.
 */
void oracle_router_logits_fx(int64_t T, int64_t H, int64_t E, const uint16_t* x,
                             const uint16_t* wr, const float* bias, int64_t* L) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            int64_t acc = 0;
            for (int64_t h = 0; h < H; ++h) {
                double p = bf16_to_double(x[t * H + h]) * bf16_to_double(wr[e * H + h]);
                acc += llrint(ldexp(p, FX_SHIFT));
            }
            if (bias) acc += llrint(ldexp((double)bias[e], FX_SHIFT));
            L[t * E + e] = acc;
        }
    }
}

/*
 * Top-K selection and routing weights.  [B] s.2 (top-6); [A] "CPU weight
 * offload" (routing-weight formula); the workload statement: softmax over the
 * logits, keep the K largest, renormalise over them; ties go to the lower
 * expert index.
 *
 * Selection: K rounds, each taking the largest remaining logit, the lower
 * index winning a tie.  idx[t*K + k] is therefore ordered by descending
 * logit, then ascending index.
 * Weights: w_k = p_k / sum_{j in S} p_j with p = softmax(l), which equals
 * exp(l_k - m) / sum_{j in S} exp(l_j - m) for any m; m = the largest logit.
 */
void oracle_topk(int64_t T, int64_t E, int64_t K, const int64_t* L, int32_t* idx, double* w) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const int64_t* l = L + t * E;
        unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
        for (int64_t k = 0; k < K; ++k) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: lower index keeps ties */
            }
            taken[best] = 1;
            idx[t * K + k] = (int32_t)best;
        }
        free(taken);
        double m = ldexp((double)l[idx[t * K]], -FX_SHIFT);
        double z = 0.0;
        for (int64_t k = 0; k < K; ++k) z += exp(ldexp((double)l[idx[t * K + k]], -FX_SHIFT) - m);
        for (int64_t k = 0; k < K; ++k)
            w[t * K + k] = exp(ldexp((double)l[idx[t * K + k]], -FX_SHIFT) - m) / z;
    }
}

/*
 * Token permutation into expert-contiguous rows: the grouping that the
 * grouped expert matrix products of [A] "CPU weight offload" work on.
 * A stable counting sort of the flat assignments i = t*K + k by expert:
 *   counts[e]  = #{i : idx[i] == e}
 *   offsets    = exclusive prefix sum of counts (E+1 entries)
 *   perm_src[offsets[e] + rank] = i   (rank = order of i among expert e's)
 *   inv_row[i] = the row r with perm_src[r] == i
 */
void oracle_permute(int64_t T, int64_t K, int64_t E, const int32_t* idx, int32_t* counts,
                    int32_t* offsets, int32_t* perm_src, int32_t* inv_row) {
    int64_t n = T * K;
    for (int64_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n; ++i) counts[idx[i]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    for (int64_t i = 0; i < n; ++i) {
        int32_t e = idx[i];
        int32_t r = offsets[e] + fill[e]++;
        perm_src[r] = (int32_t)i;
        inv_row[i] = r;
    }
    free(fill);
}

/*
 * One ungated ReLU^2 expert on one row.  [B] s.2 ("ungated ReLU^2", width F)
 * and s.3 (ungated up/down parts):
 *   z_f = sum_h Wup[f,h] x_h,   a_f = max(z_f, 0)^2,   y_j = sum_f Wdown[j,f] a_f
 * wu is [F][H], wd is [H][F] (bf16 bits), x and y are double.
 */
void oracle_expert_bf16(int64_t H, int64_t F, const uint16_t* wu, const uint16_t* wd,
                        const double* x, double* y) {
    double* a = (double*)malloc((size_t)F * sizeof(double));
    for (int64_t f = 0; f < F; ++f) {
        double z = 0.0;
        for (int64_t h = 0; h < H; ++h) z += bf16_to_double(wu[f * H + h]) * x[h];
        a[f] = z > 0.0 ? z * z : 0.0;
    }
    for (int64_t j = 0; j < H; ++j) {
        double s = 0.0;
        for (int64_t f = 0; f < F; ++f) s += bf16_to_double(wd[j * F + f]) * a[f];
        y[j] = s;
    }
    free(a);
}

/*
 * Expert outputs for R rows: y[r] = expert_{ex[r]}(xrow[r]).  The banks are
 * given for a set of experts; slot[e] is expert e's index into them (-1: not
 * supplied).  Returns 0, or -1 if a row names an expert that is not supplied.
 */
int oracle_expert_rows_bf16(int64_t R, int64_t H, int64_t F, const double* xrow, const int32_t* ex,
                            const uint16_t* wup, const uint16_t* wdown, const int32_t* slot,
                            double* y) {
    for (int64_t r = 0; r < R; ++r)
        if (slot[ex[r]] < 0) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        int64_t s = slot[ex[r]];
        oracle_expert_bf16(H, F, wup + s * F * H, wdown + s * H * F, xrow + r * H, y + r * H);
    }
    return 0;
}

/*
 * Weighted combine.  out[t] = residual[t] + sum_{k=0..K-1} w[t,k] * y[t,k],
 * the sum taken in the order k = 0..K-1 (descending routing logit).
 * residual (bf16 bits) may be NULL.
 */
void oracle_combine(int64_t T, int64_t K, int64_t H, const double* y, const double* w,
                    const uint16_t* residual, double* out) {
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += w[t * K + k] * y[(t * K + k) * H + h];
            out[t * H + h] = residual ? bf16_to_double(residual[t * H + h]) + s : s;
        }
}

/*
 * Shared expert.  [B] section 4 "Placement on card, host RAM and NVMe" lists
 * the model's shared experts among what stays on the card: besides the
 * routed experts, the MoE block has an expert that every token passes
 * through.  The pages give neither its width nor how its output joins the
 * routed sum.  Reading: the same ungated ReLU^2 FFN as a routed expert, of
 * width Fs, added with weight 1 (no gate):
 *   y_s[t] = W_down_s relu(W_up_s x_t)^2,  W_up_s [Fs][H], W_down_s [H][Fs],
 *   out[t] = (residual[t] +) sum_k w[t,k] y[t,k] + y_s[t].
 * This function gives y_s for T rows of x (fp64 values of bf16 inputs).
 */
void oracle_shared_expert_bf16(int64_t T, int64_t H, int64_t Fs, const double* x, const uint16_t* wu,
                               const uint16_t* wd, double* y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) oracle_expert_bf16(H, Fs, wu, wd, x + t * H, y + t * H);
}

/* ----------------------------------------------------------------------- */
/* FP8 E4M3 W8A8 with scalar scales.  [B] s.2: "FP8 uses scalar-scale E4M3  */
/* W8A8".  Reading: OCP FP8 E4M3 ("fn": no infinities, one NaN code per     */
/* sign, largest finite 448), round to nearest even, saturating: any finite  */
/* magnitude above 448, and infinity, maps to +-448.                          */
/* ----------------------------------------------------------------------- */

uint8_t oracle_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    int code;
    if (a < 0x1p-6) {
        /* subnormal range: multiples of 2^-9; 8 * 2^-9 is the smallest normal, code 8 */
        code = (int)nearbyint(a * 512.0);
    } else {
        int e = ilogb(a);                       /* floor(log2 a), a normal double */
        double frac = ldexp(a, -e) - 1.0;       /* in [0, 1), exact */
        int m = (int)nearbyint(frac * 8.0);
        if (m == 8) { m = 0; e += 1; }
        code = ((e + 7) << 3) | m;
        if (code > 0x7E) code = 0x7E;
    }
    return sign | (uint8_t)code;
}

float oracle_e4m3_decode(uint8_t q) {
    int s = q >> 7, e = (q >> 3) & 0xF, m = q & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/*
 * Per-tensor weight quantisation: s = amax|W| / 448 (fp32 division),
 * q = e4m3(fl32(W / s)).  An all-zero tensor takes s = 1.
 */
float oracle_quantize_tensor_fp8(int64_t n, const uint16_t* w, uint8_t* q) {
    float amax = 0.0f;
#pragma omp parallel for reduction(max : amax) schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(bf16_to_float(w[i]));
        if (a > amax) amax = a;
    }
    float s = amax > 0.0f ? amax / 448.0f : 1.0f;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        float t = bf16_to_float(w[i]) / s;
        q[i] = oracle_e4m3_encode(t);
    }
    return s;
}

/* Activation quantisation with a given static scale: q = e4m3(fl32(x / s)). */
void oracle_quantize_act_fp8(int64_t n, const uint16_t* x, float s, uint8_t* q) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(bf16_to_float(x[i]) / s);
}

/*
 * One W8A8 expert on one quantised row.
 *   z_f = s_u * s_x * sum_h dec(qu[f,h]) dec(qx[h])
 *   a_f = max(z_f, 0)^2
 *   qa_f = e4m3(fl32(fl32(a_f) / s_h))            (the H tensor's static scale)
 *   y_j = s_d * s_h * sum_f dec(qd[j,f]) dec(qa_f)
 */
void oracle_expert_fp8(int64_t H, int64_t F, const uint8_t* qu, float su, const uint8_t* qd,
                       float sd, const uint8_t* qx, float sx, float sh, double* y) {
    double* a = (double*)malloc((size_t)F * sizeof(double));
    for (int64_t f = 0; f < F; ++f) {
        double z = 0.0;
        for (int64_t h = 0; h < H; ++h)
            z += (double)oracle_e4m3_decode(qu[f * H + h]) * (double)oracle_e4m3_decode(qx[h]);
        z *= (double)su * (double)sx;
        double act = z > 0.0 ? z * z : 0.0;
        float t = (float)act / sh;
        a[f] = (double)oracle_e4m3_decode(oracle_e4m3_encode(t));
    }
    for (int64_t j = 0; j < H; ++j) {
        double s = 0.0;
        for (int64_t f = 0; f < F; ++f) s += (double)oracle_e4m3_decode(qd[j * F + f]) * a[f];
        y[j] = s * (double)sd * (double)sh;
    }
    free(a);
}

int oracle_expert_rows_fp8(int64_t R, int64_t H, int64_t F, const uint8_t* qxrow, const int32_t* ex,
                           const uint8_t* qup, const float* sup, const uint8_t* qdown,
                           const float* sdown, const int32_t* slot, float sx, float sh, double* y) {
    for (int64_t r = 0; r < R; ++r)
        if (slot[ex[r]] < 0) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        int64_t s = slot[ex[r]];
        oracle_expert_fp8(H, F, qup + s * F * H, sup[s], qdown + s * H * F, sdown[s],
                          qxrow + r * H, sx, sh, y + r * H);
    }
    return 0;
}

/* ----------------------------------------------------------------------- */
/* FP8_B128.  [B] s.3 ("Kernel dispatch") and the FP8 release notes: the    */
/* FP8 matrix normaliser maps scalar scales to FP8_B128, and the 64-value  */
/* tail of K = 1856 remains (physical K 1920).  Reading: E4M3 codes with   */
/* one fp32 scale per block of 128 consecutive values along K of each row; */
/* K is padded with zero codes to Kp = 128 * ceil(K / 128), and a block's  */
/* scale is amax / 448 over its real values (1 for an all-zero block).  A   */
/* scalar scale s maps to FP8_B128 as every block scale = s, codes kept.   */
/* Activations keep the release's W8A8 rule: static scalar scales for x    */
/* and H, their codes zero-padded to Kp like the weights'.                  */
/* ----------------------------------------------------------------------- */

int64_t oracle_b128_kp(int64_t K) { return (K + 127) / 128 * 128; }

/* W [rows][K] bf16 -> codes [rows][Kp] (zero past K), scales [rows][Kp / 128]. */
void oracle_quantize_fp8_b128(int64_t rows, int64_t K, const uint16_t* w, uint8_t* q, float* s) {
    const int64_t Kp = oracle_b128_kp(K), nb = Kp / 128;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const int64_t k0 = b * 128, k1 = k0 + 128 < K ? k0 + 128 : K;
            float amax = 0.0f;
            for (int64_t k = k0; k < k1; ++k) {
                float a = fabsf(bf16_to_float(w[r * K + k]));
                if (a > amax) amax = a;
            }
            const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
            s[r * nb + b] = sc;
            for (int64_t k = k0; k < k0 + 128; ++k)
                q[r * Kp + k] = k < K ? oracle_e4m3_encode(bf16_to_float(w[r * K + k]) / sc) : 0;
        }
    }
}

/* sum over the blocks of one row: sum_b s[b] * sum_{k in b} dec(qw[k]) * v[k], v of length Kp */
static double b128_dot(int64_t Kp, const uint8_t* qw, const float* s, const double* v) {
    double tot = 0.0;
    for (int64_t b = 0; b < Kp / 128; ++b) {
        double part = 0.0;
        for (int64_t k = b * 128; k < b * 128 + 128; ++k) part += (double)oracle_e4m3_decode(qw[k]) * v[k];
        tot += (double)s[b] * part;
    }
    return tot;
}

/*
 * One W8A8 expert with FP8_B128 weights on one quantised row.
 *   qx [Hp]: e4m3(fl32(x / s_x)), zero past H
 *   z_f  = s_x * sum_b su[f,b] * sum_{h in b} dec(qu[f,h]) dec(qx[h])
 *   a_f  = max(z_f, 0)^2,  qa_f = e4m3(fl32(fl32(a_f) / s_h)), zero past F
 *   y_j  = s_h * sum_b sd[j,b] * sum_{f in b} dec(qd[j,f]) dec(qa_f)
 * qu [F][Hp] with su [F][Hp/128]; qd [H][Fp] with sd [H][Fp/128].
 */
void oracle_expert_fp8_b128(int64_t H, int64_t F, const uint8_t* qu, const float* su, const uint8_t* qd,
                            const float* sd, const uint8_t* qx, float sx, float sh, double* y) {
    const int64_t Hp = oracle_b128_kp(H), Fp = oracle_b128_kp(F);
    double* xd = (double*)malloc((size_t)Hp * sizeof(double));
    double* a = (double*)calloc((size_t)Fp, sizeof(double));
    for (int64_t h = 0; h < Hp; ++h) xd[h] = (double)oracle_e4m3_decode(qx[h]);
    for (int64_t f = 0; f < F; ++f) {
        double z = (double)sx * b128_dot(Hp, qu + f * Hp, su + f * (Hp / 128), xd);
        double act = z > 0.0 ? z * z : 0.0;
        a[f] = (double)oracle_e4m3_decode(oracle_e4m3_encode((float)act / sh));
    }
    for (int64_t j = 0; j < H; ++j) y[j] = (double)sh * b128_dot(Fp, qd + j * Fp, sd + j * (Fp / 128), a);
    free(xd);
    free(a);
}

int oracle_expert_rows_fp8_b128(int64_t R, int64_t H, int64_t F, const uint8_t* qxrow, const int32_t* ex,
                                const uint8_t* qup, const float* sup, const uint8_t* qdown, const float* sdown,
                                const int32_t* slot, float sx, float sh, double* y) {
    const int64_t Hp = oracle_b128_kp(H), Fp = oracle_b128_kp(F);
    for (int64_t r = 0; r < R; ++r)
        if (slot[ex[r]] < 0) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        int64_t e = slot[ex[r]];
        oracle_expert_fp8_b128(H, F, qup + e * F * Hp, sup + e * F * (Hp / 128), qdown + e * H * Fp,
                               sdown + e * H * (Fp / 128), qxrow + r * Hp, sx, sh, y + r * H);
    }
    return 0;
}

/* ----------------------------------------------------------------------- */
/* NVFP4 W4A4.  [B] s.2: the NVFP4 release runs the experts "W4A4".  The    */
/* pages name the format without defining it; reading: NVIDIA's published  */
/* NVFP4 -- E2M1 elements (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), one      */
/* E4M3 scale per block of 16 consecutive elements along the contraction    */
/* dimension, and one fp32 scale per tensor.  Quantisation (reading, the    */
/* plainest recipe for that format):                                        */
/*   s_t = amax|X| / 2688 (6 x 448; 1 for an all-zero tensor), or a static  */
/*         calibrated value for activations;                                 */
/*   per block b: S_b = e4m3(fl32(fl32(amax_b / 6) / s_t));                  */
/*   e_b = fl32(dec(S_b) * s_t);  q = e2m1(fl32(x / e_b)), or 0 if e_b == 0;  */
/*   E2M1 rounding: to nearest, ties to the even code, saturating at +-6.    */
/* Dequantised value: dec(q) * dec(S_b) * s_t (exact in fp64).               */
/* Codes are packed two per byte, element 2i in the low nibble.              */
/* ----------------------------------------------------------------------- */

static const double kE2m1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

uint8_t oracle_e2m1_encode(float v) {
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs((double)v);
    if (isnan(v)) return 0;
    if (a >= 6.0) return sign | 7;
    /* walk the grid: the first point whose upper midpoint lies above a, ties to the even code */
    int c = 0;
    while (c < 7) {
        double mid = 0.5 * (kE2m1Mag[c] + kE2m1Mag[c + 1]);
        if (a < mid) break;
        if (a == mid) {
            if (c % 2 == 1) c += 1;   /* the upper neighbour has the even code */
            break;
        }
        c += 1;
    }
    return sign | (uint8_t)c;
}

float oracle_e2m1_decode(uint8_t q) {
    double v = kE2m1Mag[q & 7];
    return (float)((q & 8) ? -v : v);
}

/* One block: scale code and 16 element codes (unpacked), from fp32 values and the tensor scale. */
static uint8_t nvfp4_block(const float* x, int n, float s_t, uint8_t* q) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    uint8_t sc = oracle_e4m3_encode((amax / 6.0f) / s_t);
    float e = oracle_e4m3_decode(sc) * s_t;
    for (int i = 0; i < n; ++i) q[i] = (e == 0.0f) ? 0 : oracle_e2m1_encode(x[i] / e);
    return sc;
}

/* Tensor scale of a bf16 tensor: amax / 2688, 1 for an all-zero tensor. */
float oracle_nvfp4_tensor_scale(int64_t n, const uint16_t* w) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(bf16_to_float(w[i]));
        if (a > amax) amax = a;
    }
    return amax > 0.0f ? amax / 2688.0f : 1.0f;
}

/*
 * NVFP4 quantisation of a [rows][K] bf16 tensor (K a multiple of 16) with
 * tensor scale s_t: packed codes [rows][K/2], block scale codes [rows][K/16].
 */
void oracle_quantize_nvfp4(int64_t rows, int64_t K, const uint16_t* x, float s_t, uint8_t* codes,
                           uint8_t* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float blk[16];
        uint8_t q[16];
        for (int64_t b = 0; b < K / 16; ++b) {
            for (int i = 0; i < 16; ++i) blk[i] = bf16_to_float(x[r * K + b * 16 + i]);
            scales[r * (K / 16) + b] = nvfp4_block(blk, 16, s_t, q);
            for (int i = 0; i < 8; ++i)
                codes[r * (K / 2) + b * 8 + i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
        }
    }
}

/* Dequantised value of element k of a row (codes [K/2], scales [K/16]). */
static double nvfp4_value(const uint8_t* codes, const uint8_t* scales, int64_t k, float s_t) {
    uint8_t byte = codes[k / 2];
    uint8_t q = (k % 2) ? (byte >> 4) : (byte & 0xF);
    return (double)oracle_e2m1_decode(q) * (double)oracle_e4m3_decode(scales[k / 16]) * (double)s_t;
}

void oracle_dequantize_nvfp4(int64_t rows, int64_t K, const uint8_t* codes, const uint8_t* scales,
                             float s_t, double* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k)
            out[r * K + k] = nvfp4_value(codes + r * (K / 2), scales + r * (K / 16), k, s_t);
}

/*
 * One W4A4 expert on one quantised row (all NVFP4, rows of the weight banks
 * are [out][in]):
 *   z_f  = sum_h deq(W_up)[f,h] deq(x)[h]
 *   a_f  = fl32(max(z_f, 0)^2)
 *   H    = the row a quantised to NVFP4 in blocks of 16 features with the
 *          static tensor scale s_h
 *   y_j  = sum_f deq(W_down)[j,f] deq(H)[f]
 */
void oracle_expert_nvfp4(int64_t H, int64_t F, const uint8_t* cu, const uint8_t* su, float tu,
                         const uint8_t* cd, const uint8_t* sd, float td, const uint8_t* cx,
                         const uint8_t* sx, float tx, float th, double* y) {
    float* a = (float*)malloc((size_t)F * sizeof(float));
    double* ad = (double*)malloc((size_t)F * sizeof(double));
    double* xd = (double*)malloc((size_t)H * sizeof(double));
    for (int64_t h = 0; h < H; ++h) xd[h] = nvfp4_value(cx, sx, h, tx);
    for (int64_t f = 0; f < F; ++f) {
        double z = 0.0;
        for (int64_t h = 0; h < H; ++h)
            z += nvfp4_value(cu + f * (H / 2), su + f * (H / 16), h, tu) * xd[h];
        a[f] = (float)(z > 0.0 ? z * z : 0.0);
    }
    for (int64_t b = 0; b < F / 16; ++b) {
        uint8_t q[16];
        uint8_t sc = nvfp4_block(a + b * 16, 16, th, q);
        for (int i = 0; i < 16; ++i)
            ad[b * 16 + i] = (double)oracle_e2m1_decode(q[i]) * (double)oracle_e4m3_decode(sc) * (double)th;
    }
    for (int64_t j = 0; j < H; ++j) {
        double s = 0.0;
        for (int64_t f = 0; f < F; ++f) s += nvfp4_value(cd + j * (F / 2), sd + j * (F / 16), f, td) * ad[f];
        y[j] = s;
    }
    free(a);
    free(ad);
    free(xd);
}

/* Rows of the permuted layout: row r uses expert ex[r] at slot[ex[r]] of the given banks. */
int oracle_expert_rows_nvfp4(int64_t R, int64_t H, int64_t F, const uint8_t* cxrow, const uint8_t* sxrow,
                             const int32_t* ex, const uint8_t* cup, const uint8_t* sup, const float* tup,
                             const uint8_t* cdown, const uint8_t* sdown, const float* tdown,
                             const int32_t* slot, float tx, float th, double* y) {
    for (int64_t r = 0; r < R; ++r)
        if (slot[ex[r]] < 0) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        int64_t s = slot[ex[r]];
        oracle_expert_nvfp4(H, F, cup + s * F * (H / 2), sup + s * F * (H / 16), tup[s], cdown + s * H * (F / 2),
                            sdown + s * H * (F / 16), tdown[s], cxrow + r * (H / 2), sxrow + r * (H / 16), tx, th,
                            y + r * H);
    }
    return 0;
}

void oracle_e2m1_encode_n(int64_t n, const float* v, uint8_t* q) {
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e2m1_encode(v[i]);
}

void oracle_e2m1_decode_n(int64_t n, const uint8_t* q, float* v) {
    for (int64_t i = 0; i < n; ++i) v[i] = oracle_e2m1_decode(q[i]);
}

/*
 * RMS normalisation of the residual stream before each layer of the chained
 * stack.  [A] "Q4_K, Q3_K and Q2_K expert profiles" names a normalisation
 * among the model's steps without defining it; reading: RMSNorm with unit
 * gain, u = x / sqrt(mean(x^2) + eps), taken in fp32 with every operation
 * correctly rounded, the sum of squares in fixed point (each x^2, exact in
 * fp32, rounded to the grid 2^-16, summed exactly), and u rounded to bf16.
 */
void oracle_rmsnorm_bf16(int64_t T, int64_t H, const uint16_t* x, float eps, uint16_t* u) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        int64_t acc = 0;
        for (int64_t h = 0; h < H; ++h) {
            float v = bf16_to_float(x[t * H + h]);
            float sq = v * v;
            acc += llrint(ldexp((double)sq, 16));
        }
        float ms = (float)acc;
        ms = ms * (1.0f / 65536.0f);
        ms = ms / (float)H;
        ms = ms + eps;
        float r = sqrtf(ms);
        float rstd = 1.0f / r;
        for (int64_t h = 0; h < H; ++h) {
            float v = bf16_to_float(x[t * H + h]) * rstd;
            u[t * H + h] = float_to_bf16(v);
        }
    }
}

/*
 * bf16 rounding of doubles (one rounding, to nearest even), for values the
 * method stores in bf16.  The value is scaled so that the 8 significant bits
 * of bf16 (fewer in its subnormal range) are the integer part, rounded, and
 * scaled back; all steps are exact in double except the single rounding.
 */
void oracle_round_bf16(int64_t n, const double* v, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        double a = v[i];
        if (isnan(a)) { out[i] = 0x7FC0; continue; }
        if (a == 0.0 || isinf(a)) { out[i] = float_to_bf16((float)a); continue; }
        int e = ilogb(a) - 7;
        if (e < -133) e = -133;
        double q = ldexp(nearbyint(ldexp(a, -e)), e);
        out[i] = float_to_bf16((float)q); /* q is a bf16 value (or overflows to inf) */
    }
}

/* Array forms of the E4M3 code maps (for the tests). */
void oracle_e4m3_encode_n(int64_t n, const float* v, uint8_t* q) {
    for (int64_t i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e4m3_decode_n(int64_t n, const uint8_t* q, float* v) {
    for (int64_t i = 0; i < n; ++i) v[i] = oracle_e4m3_decode(q[i]);
}

/*
 * Calibration of the static activation scale of the ReLU^2 tensor (the
 * "scalar scale per activation tensor" of [B] s.2): the largest
 * a_f = max(z_f, 0)^2 of the bf16 model over the given rows, in fp64.
 */
double oracle_hidden_amax_bf16(int64_t R, int64_t H, int64_t F, const double* xrow, const int32_t* ex,
                               const uint16_t* wup, const int32_t* slot) {
    double amax = 0.0;
    for (int64_t r = 0; r < R; ++r) {
        const int64_t s = slot[ex[r]];
        if (s < 0) return -1.0;
        const uint16_t* wu = wup + s * F * H;
        for (int64_t f = 0; f < F; ++f) {
            double z = 0.0;
            for (int64_t h = 0; h < H; ++h) z += bf16_to_double(wu[f * H + h]) * xrow[r * H + h];
            const double a = z > 0.0 ? z * z : 0.0;
            if (a > amax) amax = a;
        }
    }
    return amax;
}
