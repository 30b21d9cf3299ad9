// moe_route_static: the router without a caller-provided workspace.
//
// Some callers cannot allocate device memory for a workspace: code that runs
// inside a host framework whose pool allocator owns all device memory and
// forbids allocations outside it, or a latency-bound decode loop that must
// not call cudaMalloc because that call can synchronise the device.  For
// them this entry point keeps the router's scratch (the fp64 partial logits
// and squared norms) in one fixed array in device memory that belongs to the
// library.  It allocates nothing: no cudaMalloc, no cudaFree, no allocating
// library routine.
//
// The array is kRouteScratchBytes (8 MiB) and every GPU that loads the
// library holds it until the process exits.  All calls share it.  Nothing
// in it needs to start at zero: each call's kernels write every scratch
// entry they later read.  Two calls whose kernels overlap on the GPU (for
// example, on two streams without ordering between them) race on the array.
//
// On the first call on a device, with that device current, the host looks
// up the device address of the array once (cudaGetSymbolAddress) and keeps
// it; that first call should come before any stream capture.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kRouteScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

size_t scratch_bytes(const moe::RouterPlan& p) {
    return align256(p.p_bytes) + align256(p.xn_bytes) + p.wn_bytes;
}

// Device address of the array on the current device, looked up once per device.
moe_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ECUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MOE_ECUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_route_static(const moe_dims* d, const void* x, const void* w_router, const float* bias,
                                       int32_t* topk_idx, float* topk_w, void* stream) {
    moe_status s = moe::internal_check_dims(d);
    if (s != MOE_OK) return s;
    if (d->T > 0 && (!x || !w_router || !topk_idx || !topk_w)) return MOE_EINVAL;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_router)) % 16 != 0) return MOE_EINVAL;
    if (d->T == 0) return MOE_OK;

    // the smallest plan (one split of the hidden dimension) must fit the array; this is
    // checked before any device call
    moe::RouterPlan plan{};
    const auto resize = [&](int S) {   // the split-K kernels' scratch (never the tensor-core router's)
        plan.tc = 0;
        plan.S = S;
        plan.p_bytes = (size_t)S * (size_t)d->T * (size_t)d->E * sizeof(double);
        plan.xn_bytes = (size_t)S * (size_t)d->T * sizeof(double);
        plan.wn_bytes = (size_t)S * (size_t)d->E * sizeof(double);
    };
    resize(1);
    if (scratch_bytes(plan) > kRouteScratchBytes) return MOE_EWORKSPACE;

    moe::DevCtx ctx;
    int sms = 0;
    if ((s = moe::internal_device(&ctx, &sms)) != MOE_OK) return s;

    // the library's usual split of the hidden dimension, reduced until it fits
    plan = moe::router_plan(d->T, d->H, d->E, sms);
    // the tensor-core router only when its slices fit; otherwise the split-K kernels' own sizes
    if (!plan.tc || scratch_bytes(plan) > kRouteScratchBytes) resize(plan.S);
    while (plan.S > 1 && scratch_bytes(plan) > kRouteScratchBytes) resize(plan.S - 1);
    if (scratch_bytes(plan) > kRouteScratchBytes) return MOE_EWORKSPACE;

    void* base = nullptr;
    if ((s = scratch_address(&base)) != MOE_OK) return s;

    unsigned char* b = static_cast<unsigned char*>(base);
    double* P = reinterpret_cast<double*>(b);
    double* xn2 = reinterpret_cast<double*>(b + align256(plan.p_bytes));
    double* wn2 = reinterpret_cast<double*>(b + align256(plan.p_bytes) + align256(plan.xn_bytes));
    const cudaError_t e = moe::launch_route(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w_router),
                                            bias, d->T, d->H, d->E, d->K, topk_idx, topk_w, P, xn2, wn2, plan, ctx,
                                            static_cast<cudaStream_t>(stream), nullptr);
    if (e == cudaSuccess) return MOE_OK;
    return e == cudaErrorInvalidValue ? MOE_EINVAL : MOE_ECUDA;
}
