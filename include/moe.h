/*
 * routed_expert_moe_b200 — C ABI of a routed mixture-of-experts layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer is the routed MoE block of the Nemotron 3.5 Transcribe hybrid
 * decoder as the bloomery issue page describes it (section 2 "Checkpoint
 * facts": hidden width 2688, top-6 routing over 128 experts, ungated ReLU^2
 * experts of width 1856; "FP8 uses scalar-scale E4M3 W8A8"; section 3:
 * ungated up/down expert parts).  For one batch of T tokens x[T][H]:
 *
 *   l[t][e]  = sum_h x[t][h] * Wr[e][h] (+ b[e])                 router
 *   S_t      = the K experts with the largest l[t][.], ties to the lower index
 *   w[t][k]  = softmax over l[t][S_t] (= the full softmax renormalised on S_t)
 *   y[t][k]  = W_down[S_tk] * relu(W_up[S_tk] * x[t])^2            expert
 *   out[t]   = (residual[t] +) sum_k w[t][k] * y[t][k], k in order  combine
 *
 * Conventions for every call:
 *  - Tensors are dense row-major device arrays owned by the caller; the
 *    library allocates nothing.  Device pointers must be 16-byte aligned,
 *    the workspace 256-byte aligned.
 *  - bf16 is the IEEE-like bfloat16 bit pattern (uint16); fp8 is OCP E4M3
 *    ("fn") stored as uint8.  Weight banks are [out][in]: W_up is [E][F][H],
 *    W_down is [E][H][F], the router weight is [E][H].
 *  - Every call is asynchronous on the given CUDA stream (a cudaStream_t
 *    passed as void*; NULL is the legacy default stream).  Argument errors
 *    are detected on the host and returned before anything is launched.
 *    Errors found inside kernels (an out-of-range expert index, a bounded
 *    wait that expired, a router magnitude outside the exact range) are
 *    recorded in a per-device error word that moe_check_device_error reads.
 *  - Results are deterministic: the same inputs give the same bits, on any
 *    stream, at any batch size split (no floating-point atomics).
 *  - Expert indices and the permutation are exact: the router ranks experts
 *    on logits summed in fixed point (each bf16 product rounded to 2^-40,
 *    summed exactly), computed fast in fp32 with a rigorous error bound and
 *    recomputed exactly for the few experts whose rank the bound leaves open.
 */
#ifndef ROUTED_EXPERT_MOE_H
#define ROUTED_EXPERT_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 3

typedef enum {
    MOE_OK = 0,
    MOE_EINVAL = 1,        /* invalid argument: null pointer, bad size, misalignment */
    MOE_EUNSUPPORTED = 2,  /* a valid request the library does not support (e.g. not sm_100) */
    MOE_ECUDA = 3,         /* a CUDA runtime call or a launch failed */
    MOE_ETIMEOUT = 4,      /* a bounded wait inside a kernel expired (device error word) */
    MOE_EWORKSPACE = 5,    /* workspace smaller than moe_workspace_size() */
    MOE_ERANGE = 6,        /* router inputs beyond the exact fixed-point range (device) */
    MOE_EINDEX = 7         /* an expert index outside [0, E) reached moe_permute (device) */
} moe_status;

typedef enum {
    MOE_BF16 = 0,          /* expert banks and expert activations in bf16 */
    MOE_FP8_E4M3 = 1,      /* W8A8: expert banks and expert activations in E4M3 codes */
    MOE_NVFP4 = 2,         /* W4A4: expert banks and expert activations in NVFP4 (see below) */
    MOE_FP8_B128 = 3       /* W8A8: E4M3 banks with one fp32 scale per 128 values along K (see below) */
} moe_dtype;

/* Problem size.  Limits: 0 <= T, T*K < 2^31; 1 <= E <= 256; 1 <= K <= min(E, 16);
 * 16 <= H <= 65536 and 16 <= F <= 65536, both multiples of 16 (of 32 for MOE_NVFP4).
 * Fs: width of the shared expert, 0 for none.  Cited: bloomery page s.4
 * (the model's shared experts stay on the card beside the routed ones); the
 * pages give neither its width nor how it joins the routed sum.  Reading:
 * an ungated ReLU^2 FFN of width Fs that every token passes through, added
 * with weight 1.  Fs must be a multiple of F (the kernels run it as Fs/F
 * chunks of width F, an exact split since ReLU^2 is elementwise), with
 * K + Fs/F <= 16, E + Fs/F <= 256, T*(K + Fs/F) < 2^31, and MOE_BF16 experts
 * (MOE_EUNSUPPORTED otherwise). */
typedef struct {
    int64_t T;             /* tokens */
    int32_t H;             /* hidden width (router and up-projection input, down output) */
    int32_t E;             /* routed experts */
    int32_t K;             /* experts per token */
    int32_t F;             /* expert width (up output, down input) */
    int32_t expert_dtype;  /* moe_dtype */
    int32_t Fs;            /* shared expert width (0: none) */
} moe_dims;

/* Scales of the quantised expert formats.  Ignored for MOE_BF16; required
 * (non-NULL, with every pointer named below for the format non-NULL) for the
 * three others.  Activation scales are static in every format: x_scale and
 * h_scale are finite and > 0.  Per format:
 *
 * MOE_FP8_E4M3 (bloomery page, section 2: "scalar-scale E4M3 W8A8"): real
 * value = code * scale.  Banks: w_up codes [E][F][H], w_down codes [E][H][F].
 *   w_up_scale [E], w_down_scale [E]: one scale per expert tensor.
 *   w_up_block, w_down_block: unused.
 *
 * MOE_FP8_B128 (bloomery page, section 3: the FP8 release's matrix
 * normaliser maps scalar scales to FP8_B128; the 64-value tail of K = 1856):
 * E4M3 codes with one fp32 scale per block of 128 values along K of each
 * weight row; K zero-padded to Kp(K) = 128*ceil(K/128).  Banks: w_up codes
 * [E][F][Kp(H)], w_down codes [E][H][Kp(F)] (zero codes past K).
 *   w_up_scale [E][F][Kp(H)/128], w_down_scale [E][H][Kp(F)/128].
 *   w_up_block, w_down_block: unused.
 *
 * MOE_NVFP4 (bloomery page, section 2: the NVFP4 release runs the experts
 * W4A4; the format is NVIDIA's NVFP4): E2M1 codes packed two per byte
 * (element 2i in the low nibble), one E4M3 scale per 16 consecutive elements
 * along the contraction dimension, one fp32 scale per tensor; real value =
 * e2m1(code) * e4m3(block scale) * tensor scale.  Block scales are stored
 * [rows][KSP] bytes with KSP = K/16 rounded up to a multiple of 16 (padding
 * zero; moe_quantize_nvfp4 writes this layout).  Banks: w_up codes
 * [E][F][H/2], w_down codes [E][H][F/2].
 *   w_up_scale [E], w_down_scale [E]: the tensor scales.
 *   w_up_block [E][F][KSP(H)], w_down_block [E][H][KSP(F)]: the block
 *   scales, 16-byte aligned.
 *   x and the ReLU^2 tensor are quantised inside the layer with block scales
 *   taken at run time and the static tensor scales x_scale and h_scale. */
typedef struct {
    const float* w_up_scale;    /* device; shape per format (above) */
    const float* w_down_scale;  /* device; shape per format (above) */
    float x_scale;              /* static (tensor) scale of the expert input activations */
    float h_scale;              /* static (tensor) scale of the ReLU^2 activations */
    const uint8_t* w_up_block;  /* MOE_NVFP4 only: [E][F][KSP(H)] E4M3 block scales */
    const uint8_t* w_down_block;/* MOE_NVFP4 only: [E][H][KSP(F)] E4M3 block scales */
} moe_quant_scales;
typedef moe_quant_scales moe_fp8_scales;

/* Human-readable name of a status.  Never NULL. */
const char* moe_status_string(moe_status s);

/* MOE_ABI_VERSION of the loaded library. */
int moe_abi_version(void);

/* Bytes of workspace that moe_forward needs for these dims (moe_route,
 * moe_permute and moe_expert_ffn need no more).  Host only; no device call. */
moe_status moe_workspace_size(const moe_dims* d, size_t* bytes);

/* Number of kernels one moe_forward call with these dims launches on its
 * stream, under the current test hooks (the router's shape and the
 * permutation's depend on the batch size).  Host only; no device call. */
moe_status moe_forward_launches(const moe_dims* d, int32_t* launches);

/* Router: logits, top-K, renormalised softmax weights.
 *   x         [T][H] bf16     w_router [E][H] bf16     bias [E] fp32 or NULL
 *   topk_idx  [T][K] int32    out: experts by descending logit, ties to the lower index
 *   topk_w    [T][K] fp32     out: weights, summing to 1 per token
 * Cited: bloomery page s.2 (top-6 over 128 experts); audio.cpp model page,
 * "CPU weight offload" (router and routing-weight formulas). */
moe_status moe_route(const moe_dims* d, const void* x, const void* w_router, const float* bias,
                     int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* Permutation into expert-contiguous rows: a stable counting sort of the
 * assignments i = t*K + k by expert.
 *   topk_idx [T][K] int32 in; counts [E], offsets [E+1] (exclusive scan),
 *   perm_src [T*K] (row r of the grouped layout holds assignment perm_src[r]),
 *   inv_row  [T*K] (assignment i sits in row inv_row[i]) out.
 * ws: scratch of at least moe_workspace_size() bytes; it may be NULL (with
 * ws_bytes 0) when T*K <= 4096.
 * An index outside [0, E) sets MOE_EINDEX in the device error word; the
 * outputs are then unspecified.  Cited: audio.cpp model page, "CPU weight
 * offload" (grouped expert matrix multiplication). */
moe_status moe_permute(const moe_dims* d, const int32_t* topk_idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm_src, int32_t* inv_row, void* ws,
                       size_t ws_bytes, void* stream);

/* Grouped expert FFN over the permuted rows:
 *   y_perm[r] = W_down[e] * relu(W_up[e] * x[perm_src[r] / K])^2,  e = expert of row r
 *   x [T][H] bf16; offsets [E+1] and perm_src [T*K] as from moe_permute;
 *   w_up, w_down: the banks in the layout moe_quant_scales gives for the
 *   format ([E][F][H] and [E][H][F] for bf16 and MOE_FP8_E4M3; [E][F][Kp(H)]
 *   and [E][H][Kp(F)] for MOE_FP8_B128; [E][F][H/2] and [E][H][F/2] for
 *   MOE_NVFP4);
 *   y_perm [T*K + T*Fs/F][H] bf16 out.
 * With a shared expert (d->Fs > 0): w_up_shared [Fs][H] and w_down_shared
 * [H][Fs] bf16 (both NULL when Fs = 0), and rows T*K + j*T + t of y_perm
 * receive chunk j of it for token t:
 *   W_down_s[:, jF:(j+1)F] * relu(W_up_s[jF:(j+1)F, :] * x[t])^2.
 * scales must be non-NULL for MOE_FP8_E4M3, MOE_FP8_B128 and MOE_NVFP4, with the
 * pointers moe_quant_scales names for the format; otherwise MOE_EINVAL (checked
 * on the host before any launch, also for T = 0).  Cited: bloomery page s.2 and
 * s.3 (ungated ReLU^2 experts, up/down parts). */
moe_status moe_expert_ffn(const moe_dims* d, const void* x, const int32_t* offsets,
                          const int32_t* perm_src, const void* w_up, const void* w_down,
                          const void* w_up_shared, const void* w_down_shared,
                          const moe_fp8_scales* scales, void* y_perm, void* ws, size_t ws_bytes,
                          void* stream);

/* Weighted combine: out[t] = (residual[t] +) sum_{k=0..K-1} topk_w[t][k] * y_perm[inv_row[t*K+k]]
 *                              (+ sum_j y_perm[T*K + j*T + t] with a shared expert of Fs/F chunks),
 * summed in fp32 in the order k = 0..K-1, then j = 0.., then the residual, and rounded
 * once to bf16.
 *   y_perm [T*K + T*Fs/F][H] bf16, inv_row [T*K], topk_w [T][K] fp32, residual [T][H] bf16
 *   or NULL, out [T][H] bf16 (may alias residual). */
moe_status moe_combine(const moe_dims* d, const void* y_perm, const int32_t* inv_row,
                       const float* topk_w, const void* residual, void* out, void* stream);

/* The whole layer in one call (route, permute, expert FFN, combine), all
 * intermediates in the workspace.  topk_idx / topk_w ([T][K]) may be NULL;
 * when given they receive the routing.  out may alias residual.  With
 * d->Fs > 0 the shared expert (w_up_shared [Fs][H], w_down_shared [H][Fs],
 * bf16) runs in the same expert FFN launch as the routed experts and its
 * output joins the combine with weight 1; both pointers NULL when Fs = 0. */
moe_status moe_forward(const moe_dims* d, const void* x, const void* w_router, const float* bias,
                       const void* w_up, const void* w_down, const void* w_up_shared,
                       const void* w_down_shared, const moe_fp8_scales* scales,
                       const void* residual, void* out, int32_t* topk_idx, float* topk_w,
                       void* ws, size_t ws_bytes, void* stream);

/* Row gather: out[r] = x[perm_src[r] / K] for r < rows, rows of H bf16 values
 * (16-byte aligned).  This is the step moe_expert_ffn applies to the token
 * rows before the up projection, exposed for callers that move rows between
 * devices themselves (an expert-parallel exchange: the rows a rank sends to
 * the experts' owners, and the owners' outputs back in the order received).
 *   x [src_rows][H], perm_src [rows] int32 (K = 1: a plain row index),
 *   out [rows][H].  An index outside [0, src_rows * K) sets MOE_EINDEX in
 *   the device error word and leaves that row unwritten.  H a multiple of 8.
 * Cited: audio.cpp model page, "CPU weight offload" (grouped expert matrix
 * multiplication). */
moe_status moe_gather_rows(int64_t rows, int64_t src_rows, int32_t H, int32_t K, const void* x,
                           const int32_t* perm_src, void* out, void* stream);

/* Regrouping of the rows an expert's owner receives in an expert-parallel
 * exchange (the experts split over W ranks, E_loc = E / W each).  Received
 * rows arrive source-major: from rank 0 its rows for local experts 0, 1, ...,
 * then rank 1, ...  The grouped layout moe_expert_ffn reads (with K = 1) is
 * expert-major, then source rank, then arrival order.
 *   recv_counts [W][E_loc] int64 (device): rows from rank p for local expert e;
 *   R = the sum of recv_counts (the received rows);
 *   offsets [E_loc + 1] int32 out: the grouped layout's expert offsets;
 *   perm [R] int32 out: grouped row g holds received row perm[g];
 *   inv [R] int32 out: received row i sits in grouped row inv[i].
 * W * E_loc <= 256.  Counts that are negative or do not sum to R set
 * MOE_EINDEX in the device error word and leave the outputs unwritten.  The
 * pages say nothing about several GPUs; this serves the split of the grouped
 * expert products by owner (audio.cpp model page, "CPU weight offload":
 * grouped expert matrix multiplication). */
moe_status moe_ep_regroup(int32_t W, int32_t E_loc, int64_t R, const int64_t* recv_counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv, void* stream);

/* Per-tensor E4M3 quantisation of n_tensors bf16 tensors of tensor_elems
 * elements each (an expert bank): scale[i] = amax|W_i| / 448 (1 for an
 * all-zero tensor), codes = e4m3_rne_satfinite(W / scale[i]).
 *   src [n_tensors][tensor_elems] bf16, codes same shape uint8, scales [n_tensors] fp32.
 * Cited: bloomery page s.2 ("scalar-scale E4M3 W8A8"). */
moe_status moe_quantize_fp8(int64_t n_tensors, int64_t tensor_elems, const void* src,
                            uint8_t* codes, float* scales, void* stream);

/* Activation quantisation with a static scale (the X side of W8A8):
 * codes[r][h] = e4m3_rne_satfinite(fl32(x[r][h] / x_scale)), the quotient
 * rounded to nearest in fp32.  This is the step moe_forward and
 * moe_expert_ffn apply to the permuted rows, here on rows in order.
 *   x [rows][H] bf16 (16-byte aligned), codes [rows][H] uint8; H a multiple
 * of 16; x_scale > 0 and finite.  Cited: bloomery page s.2 ("scalar-scale
 * E4M3 W8A8"). */
moe_status moe_quantize_act_fp8(int64_t rows, int32_t H, float x_scale, const void* x, uint8_t* codes,
                                void* stream);

/* FP8_B128 quantisation of n_tensors bf16 tensors [rows][K] (an expert bank):
 * per row and block of 128 values along K, scale = amax|block| / 448 (an fp32
 * division; 1 for an all-zero block), codes e4m3(fl32(W / scale)) nearest-even
 * and saturating; K is padded to Kp = 128*ceil(K/128) with zero codes.
 *   src [n_tensors][rows][K] bf16; codes [n_tensors][rows][Kp];
 *   scales [n_tensors][rows][Kp/128] fp32.  K a multiple of 16.
 * Cited: bloomery page s.3 ("Kernel dispatch": FP8_B128 with the 64-value
 * tail of K = 1856). */
moe_status moe_quantize_fp8_b128(int64_t n_tensors, int64_t rows, int32_t K, const void* src, uint8_t* codes,
                                 float* scales, void* stream);

/* NVFP4 quantisation of n_tensors bf16 tensors [rows][K] (an expert bank):
 * tensor scale t[i] = amax|W_i| / 2688 (1 for an all-zero tensor), per block
 * of 16 along K: S = e4m3(fl32(fl32(amax_b / 6) / t[i])), codes
 * e2m1(fl32(W / fl32(S * t[i]))) nearest-even, saturating at 6.
 *   src [n_tensors][rows][K] bf16; codes [n_tensors][rows][K/2];
 *   block [n_tensors][rows][KSP(K)] (padding written as zero); tscale [n_tensors] fp32.
 * K a multiple of 32.  Cited: bloomery page s.2 (NVFP4, W4A4 experts). */
moe_status moe_quantize_nvfp4(int64_t n_tensors, int64_t rows, int32_t K, const void* src, uint8_t* codes,
                              uint8_t* block, float* tscale, void* stream);

/* Activation quantisation to NVFP4 with a static tensor scale (the X side
 * of W4A4): per block of 16 along H, S = e4m3(fl32(fl32(amax_b / 6) /
 * x_scale)), codes e2m1(fl32(x / fl32(S * x_scale))).  This is the step
 * moe_forward and moe_expert_ffn apply to the permuted rows, here on rows
 * in order.  x [rows][H] bf16; codes [rows][H/2]; block [rows][KSP(H)].
 * H a multiple of 32.  Cited: bloomery page s.2 (NVFP4, W4A4 experts). */
moe_status moe_quantize_act_nvfp4(int64_t rows, int32_t H, float x_scale, const void* x, uint8_t* codes,
                                  uint8_t* block, void* stream);

/* RMS normalisation with unit gain of the residual stream between chained
 * layers: u = bf16(x / sqrt(mean(x^2) + eps)), the mean of squares taken
 * exactly (fixed point, 2^-16 per term) and the rest in correctly rounded fp32.
 *   x, u [T][H] bf16 (u may not alias x).  Cited: audio.cpp model page,
 * "Q4_K, Q3_K and Q2_K expert profiles" (the model's normalisation). */
moe_status moe_rmsnorm(int64_t T, int32_t H, float eps, const void* x, void* u, void* stream);

/* The router (as moe_route) without a caller-provided workspace.  The paper
 * has no counterpart: this entry point serves callers that cannot allocate
 * device memory for a workspace, such as code inside a host framework whose
 * pool allocator owns all device memory, or a decode loop that must not call
 * cudaMalloc because it can synchronise the device.  Its scratch is one
 * fixed 8 MiB array of device memory held by the library on every GPU that
 * loads it, until the process exits.  It allocates nothing.
 *   Limit: the partial logits of one split, T*E*8 bytes plus T*8 + E*8
 *   (each rounded up to 256 bytes), must fit in 8 MiB; at E = 128 that is
 *   T <= 8127.  Larger batches return MOE_EWORKSPACE before any launch.
 *   The first call on a device looks up the array's device address (with
 *   that device current) and should come before any stream capture.
 *   All calls share the array; calls whose kernels overlap on the GPU race.
 *   Nothing in it needs clearing between calls: each call writes all the
 *   scratch it reads.  Same arguments and results as moe_route. */
moe_status moe_route_static(const moe_dims* d, const void* x, const void* w_router, const float* bias,
                            int32_t* topk_idx, float* topk_w, void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns MOE_OK, or the first error a kernel recorded. */
moe_status moe_check_device_error(void* stream);

/* Measurement hook.  With n == MOE_STAGE_EVENTS and `events` an array of n
 * cudaEvent_t (as void*), every later moe_forward on this process records
 * events[i] on its stream before stage i and events[n-1] after the last
 * stage (stages: 0 router logits, 1 router top-K, 2 permute, 3 row gather,
 * 4 up GEMM, 5 down GEMM, 6 combine; when both projections run in one
 * launch, stage 4 holds that launch and stage 5 is empty), so a caller can
 * time each kernel in place.  n == 0 turns it off.  Host state shared by all threads. */
#define MOE_STAGE_EVENTS 8
moe_status moe_set_stage_events(void* const* events, int32_t n);

/* Test and measurement hooks (host state shared by all threads).
 * what = 1: limit of every bounded wait in nanoseconds (value <= 0 restores
 * the default of 4 s); what = 2: the grouped-GEMM producer of block 0
 * withholds its first load (value 1) so the consumer's wait must expire --
 * in the one-launch FFNs, the list's first up unit withholds its report so
 * that the down units of its entry wait in vain; 0 turns it off; what = 3: value 1 runs the grouped GEMMs of batches with
 * tiles of more than 64 tokens on CTA pairs (cta_group::2, M = 256), value 0
 * (the default) on single CTAs; what = 4: largest batch (tokens) that the
 * router computes in one launch of 8-CTA clusters split over the experts (0:
 * never; value < 0 restores the default of 256); what = 5: router of the
 * larger batches: 0 (the default) by batch size (the tensor-core router --
 * int8 slices, then exact integer products on the tensor cores -- when E <= 128,
 * else the tiled logits kernel and the top-K kernel), 1 always the two
 * kernels, 2 always the hidden-split clusters when E <= 128, 3 always the
 * tensor-core router when E <= 128; other values MOE_EINVAL; what = 6:
 * value 0 launches every kernel without programmatic stream serialization
 * (each kernel then starts only after its predecessor has finished), 1 (the
 * default) lets each kernel start while its predecessor finishes and wait
 * on the device for it; what = 7: value 1 reads the shared expert's down
 * weight through the fallback map (the plain [H][Fs] matrix, chunk j from
 * column j*F) instead of the chunked 3-D view, 0 (the default) restores the
 * view; what = 8: value 1 (the default) runs both expert projections in one
 * launch, for every expert format and with a shared expert (the down units of
 * a schedule entry start once that entry's up units have reported), 0 as two
 * launches; what = 9: bytes of a bf16 up bank's start (its first experts'
 * weights, which the FFN's first units read) that the small-batch router
 * prefetches into L2 from the clusters the device fits beside the batch's
 * (value 0: none; value < 0 restores the default of 48 MiB; clamped to the
 * bank's size; other expert dtypes: none); the prefetch changes no result.
 * The prefetching clusters come last in the router's grid: where kernels of
 * other streams hold the SMs, they can wait for SMs and so delay the
 * router's completion (value 0 avoids that).  Other `what`: MOE_EINVAL. */
moe_status moe_debug_set(int32_t what, int64_t value);

#ifdef __cplusplus
}
#endif

#endif /* ROUTED_EXPERT_MOE_H */
