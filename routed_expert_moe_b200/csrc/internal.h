// Declarations shared between the library's translation units: the plans
// that one file computes and another consumes, and every launcher that
// api.cu (or another entry point) calls.  Each struct and prototype is
// declared here once and every .cu that defines or uses it includes this
// file, so a change to a layout or a signature is seen by all of them.
#pragma once

#include <cuda.h>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace moe {

struct RouterPlan {
    int S;
    int nchunks;
    int num_sms;
    int tc;               // 1: the tensor-core router (route_tc.cu), its scratch in the P region
    size_t p_bytes, xn_bytes, wn_bytes;
};
RouterPlan router_plan(int64_t T, int H, int E, int num_sms);
size_t route_tc_scratch_bytes(int64_t T, int H, int E);
cudaError_t launch_route_tc(const uint16_t* x, const uint16_t* wr, const float* bias, int64_t T, int H, int E,
                            int K, int32_t* idx, float* w, void* scratch, int num_sms, const DevCtx& ctx,
                            cudaStream_t stream, void (*between)(cudaStream_t));
cudaError_t launch_route(const uint16_t* x, const uint16_t* wr, const float* bias, int64_t T, int H, int E,
                         int K, int32_t* idx, float* w, double* P, double* xn2, double* wn2,
                         const RouterPlan& plan, const DevCtx& ctx, cudaStream_t stream,
                         void (*between)(cudaStream_t) = nullptr, const void* warm = nullptr,
                         int64_t warm_bytes = 0);
cudaError_t launch_permute(const int32_t* idx, int64_t n, int K, int E, int32_t* counts, int32_t* offsets,
                           int32_t* perm_src, int32_t* inv_row, int4* sched, int* n_sched, int bn, int ns,
                           int* scratch, const DevCtx& ctx, cudaStream_t stream);
void set_router_small_max(int64_t v);
void set_router_split(int v);
size_t permute_scratch_ints(int64_t n, int E);
int route_launches(int64_t T, int H, int E);
size_t permute_smem_bytes(int E);
cudaError_t launch_schedule(const int32_t* offsets, int E, int bn, int4* sched, int* n_sched, int ns, int64_t T,
                            int K, cudaStream_t stream);
cudaError_t launch_gather(const uint16_t* x, const int32_t* perm_src, int64_t rows, int64_t routed_rows, int K,
                          int64_t T, int H, void* xp, bool fp8, float x_scale, int num_sms, const DevCtx& ctx,
                          cudaStream_t stream, int* zero = nullptr, int64_t n_zero = 0);
struct GemmPlan {
    int bn;
    int n_stages;
    size_t smem_bytes;
    int max_sched;
};
GemmPlan gemm_plan(int64_t T, int K, int E);
cudaError_t launch_grouped_gemm(bool fp8, bool up, const void* W, int E, int Nout, int Kdim, const void* act,
                                int64_t rows, const int4* sched, const int* n_sched, const GemmPlan& plan,
                                void* out, const float* w_scale, float in_scale, float out_scale, int num_sms,
                                int debug_withhold, const DevCtx& ctx, cudaStream_t stream, const void* Ws,
                                int n_shared);
// 3-D bf16 maps with a 128-byte swizzle, box {64, box_rows, 1}: {d0, d1, d2} with byte strides s1,
// s2; make_map_chunks views a row-major [rows][n * chunk] matrix as {chunk, rows, n}, so that a
// box never reads into the next chunk.
bool make_map3(CUtensorMap* m, const void* base, int64_t d0, int64_t d1, int64_t d2, int64_t s1, int64_t s2,
               int box_rows);
bool make_map_chunks(CUtensorMap* m, const void* base, int64_t rows, int64_t chunk, int64_t n, int box_rows);
cudaError_t launch_grouped_ffn(bool fp8, const void* w_up, const void* w_down, int E, int F, int H, const void* xp,
                               void* hb, void* y, int64_t rows, const int4* sched, const int* n_sched, int* done,
                               const GemmPlan& plan, const float* su, const float* sd, float x_scale, float h_scale,
                               int num_sms, int debug_hold, const DevCtx& ctx, cudaStream_t stream,
                               const void* w_up_s = nullptr, const void* w_down_s = nullptr, int n_shared = 0);
cudaError_t launch_grouped_gemm_pair(bool fp8, bool up, const void* W, int E, int Nout, int Kdim, const void* act,
                                     int64_t rows, const int4* sched, const int* n_sched, int bn, int max_sched,
                                     void* out, const float* w_scale, float in_scale, float out_scale,
                                     int num_sms, const DevCtx& ctx, cudaStream_t stream);
cudaError_t launch_grouped_gemm_fp4(bool up, const uint8_t* w_codes, const uint8_t* w_scales, const float* w_tscale,
                                    int E, int Nout, int Kdim, const uint8_t* a_codes, const uint8_t* a_scales,
                                    float in_tscale, float out_tscale, int64_t rows, const int4* sched,
                                    const int* n_sched, int bn, int max_sched, void* out, uint8_t* out_scale,
                                    int num_sms, int debug_withhold, const DevCtx& ctx, cudaStream_t stream);
cudaError_t launch_quantize_nvfp4(int64_t n_tensors, int64_t rows, int K, const uint16_t* src, uint8_t* codes,
                                  uint8_t* bscale, float* tscale, int num_sms, cudaStream_t stream);
cudaError_t launch_gather_nvfp4(const uint16_t* x, const int32_t* perm_src, int64_t rows, int K, int64_t T, int H,
                                float s_t, uint8_t* codes, uint8_t* bscale, int num_sms, const DevCtx& ctx,
                                cudaStream_t stream, int* zero = nullptr, int64_t n_zero = 0);
cudaError_t launch_grouped_ffn_fp4(const uint8_t* wu_codes, const uint8_t* wu_scales, const float* wu_tscale,
                                   const uint8_t* wd_codes, const uint8_t* wd_scales, const float* wd_tscale, int E,
                                   int F, int H, const uint8_t* x_codes, const uint8_t* x_scales, float x_tscale,
                                   float h_tscale, uint8_t* hb, uint8_t* hb_block, void* y, int64_t rows,
                                   const int4* sched, const int* n_sched, int bn, int max_sched, int* done,
                                   int num_sms, int debug_hold, const DevCtx& ctx, cudaStream_t stream);
size_t nvfp4_scale_row_bytes(int K);
cudaError_t launch_grouped_gemm_b128(bool up, const uint8_t* W, const float* w_scale, int E, int Nout, int Kdim,
                                     const uint8_t* act, int64_t rows, const int4* sched, const int* n_sched, int bn,
                                     int max_sched, void* out, float in_scale, float out_scale, int num_sms,
                                     int debug_withhold, const DevCtx& ctx, cudaStream_t stream);
cudaError_t launch_grouped_ffn_b128(const uint8_t* w_up, const float* su, const uint8_t* w_down, const float* sd,
                                    int E, int F, int H, const uint8_t* xp, uint8_t* hb, void* y, int64_t rows,
                                    const int4* sched, const int* n_sched, int bn, int max_sched, int* done,
                                    float x_scale, float h_scale, int num_sms, int debug_hold, const DevCtx& ctx,
                                    cudaStream_t stream);
cudaError_t launch_quantize_fp8_b128(int64_t rows, int K, const uint16_t* src, uint8_t* codes, float* scales,
                                     int num_sms, cudaStream_t stream);
cudaError_t launch_combine(const uint16_t* yp, const int32_t* inv_row, const float* w, const uint16_t* residual,
                           uint16_t* out, int64_t T, int K, int ns, int H, int num_sms, const DevCtx& ctx,
                           cudaStream_t stream);
cudaError_t launch_rmsnorm(const uint16_t* x, uint16_t* u, int64_t T, int H, float eps, int num_sms,
                           cudaStream_t stream);
cudaError_t launch_quantize(int64_t n_tensors, int64_t elems, const uint16_t* src, uint8_t* codes,
                            float* scales, int num_sms, cudaStream_t stream);


cudaError_t launch_ep_regroup(const int64_t* recv_counts, int W, int E_loc, int64_t R, int32_t* offsets,
                              int32_t* perm, int32_t* inv, const DevCtx& ctx, cudaStream_t stream);

// Token rows per schedule entry of the FP8_B128 grouped GEMM: its epilogue
// keeps one running fp32 sum per row in registers.
constexpr int kB128MaxTileRows = 128;

// Token rows per schedule entry of the one-launch FP8_B128 FFN: tiles of 64 rows run two CTAs per
// SM, which outweighs reading an expert's weights for three tiles instead of two at prefill
// (FP8_B128 prefill layer 993 -> 767 us).
constexpr int kB128OneLaunchTileRows = 64;

// Token rows per schedule entry of the NVFP4 grouped GEMM: its two TMEM
// accumulators of this many columns leave room for the scale factors.
constexpr int kFp4MaxTileRows = 224;

// Token rows per schedule entry of the one-launch FFN on sparse batches (fewer than this many
// rows per expert on average): the tile height of its two-CTA-per-SM layout.
constexpr int kFfnSparseRows = 128;

// Sizes the plans must keep: a plan is passed by value and by reference
// between files, so a field added in one place shows up as a size change here.
static_assert(sizeof(RouterPlan) == 40, "RouterPlan layout changed: update every user");
static_assert(sizeof(GemmPlan) == 24, "GemmPlan layout changed: update every user");

// Argument checks and device context for entry points defined outside api.cu.
moe_status internal_check_dims(const moe_dims* d);
moe_status internal_device(DevCtx* ctx, int* num_sms);

}  // namespace moe
