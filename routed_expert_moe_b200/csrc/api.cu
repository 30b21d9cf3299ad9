// C ABI (include/moe.h): argument validation, workspace layout, per-device
// setup and the launch sequence of each entry point.  All computation is in
// the kernels of route.cu, permute.cu, grouped_gemm.cu and combine.cu.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

using namespace moe;

// The per-device error word: the only device state of the library.
__device__ int g_moe_error = 0;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<int> g_debug_withhold{0};
std::atomic<int> g_gemm_pair{0};
std::atomic<int> g_fused_ffn{1};   // 1: both bf16/E4M3 projections in one launch (grouped_ffn.cu)
std::atomic<int> g_pdl{1};
std::atomic<int> g_shared_2d{0};   // 1: the shared down weight through its 2-D fallback map
// Bytes of the bf16 up weight bank (its first experts: the FFN's first units) that the decode
// router's spare clusters prefetch into L2 while routing.  On B200 at T=64: the FFN 347 ->
// 340 us and the router 20.3 -> 20.8 us at 48 MB; 64 MB and 96 MB slow the router's own loads
// more (22.0, 22.6 us) than they save.  The NVFP4 and FP8_B128 FFNs, not bound by DRAM at
// decode, gain nothing (NVFP4 layer 172.9 us either way; FP8_B128 219.0 -> 225.6 us), so
// their banks are not prefetched.
constexpr int64_t kL2WarmDefault = (int64_t)48 << 20;
std::atomic<int64_t> g_l2_warm{kL2WarmDefault};
void* g_stage_events[MOE_STAGE_EVENTS] = {};
std::atomic<int> g_stage_events_on{0};

void stage_mark(int i, cudaStream_t st) {
    if (g_stage_events_on.load()) cudaEventRecord(static_cast<cudaEvent_t>(g_stage_events[i]), st);
}
void mark_stage1(cudaStream_t st) { stage_mark(1, st); }

struct DeviceInfo {
    bool ready = false;
    moe_status status = MOE_OK;
    int num_sms = 0;
    int* err = nullptr;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

moe_status device_setup(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ECUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ECUDA;
        if (major != 10 || minor != 0) {
            d.status = MOE_EUNSUPPORTED;
        } else if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_moe_error) != cudaSuccess) {
            return MOE_ECUDA;
        }
        d.ready = true;
    }
    if (d.status != MOE_OK) return d.status;
    *out = &d;
    return MOE_OK;
}

DevCtx make_ctx(const DeviceInfo* d) { return DevCtx{d->err, g_timeout_ns.load()}; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status check_dims(const moe_dims* d) {
    if (!d) return MOE_EINVAL;
    if (d->T < 0 || d->E < 1 || d->E > 256 || d->K < 1 || d->K > 16 || d->K > d->E) return MOE_EINVAL;
    if (d->H < 16 || d->H > 65536 || d->H % 16 != 0) return MOE_EINVAL;
    if (d->F < 16 || d->F > 65536 || d->F % 16 != 0) return MOE_EINVAL;
    if (d->T * (int64_t)d->K >= (int64_t)1 << 31) return MOE_EINVAL;
    if (d->expert_dtype != MOE_BF16 && d->expert_dtype != MOE_FP8_E4M3 && d->expert_dtype != MOE_NVFP4 &&
        d->expert_dtype != MOE_FP8_B128)
        return MOE_EINVAL;
    if (d->expert_dtype == MOE_NVFP4 && (d->H % 32 != 0 || d->F % 32 != 0)) return MOE_EINVAL;
    // shared expert: chunks of the routed width, each an extra term of the combine
    if (d->Fs < 0 || d->Fs % d->F != 0) return MOE_EINVAL;
    const int ns = d->Fs / d->F;
    if (ns > 0) {
        if (d->K + ns > 16 || d->E + ns > 256) return MOE_EINVAL;
        if (d->T * (int64_t)(d->K + ns) >= (int64_t)1 << 31) return MOE_EINVAL;
        if (d->expert_dtype != MOE_BF16) return MOE_EUNSUPPORTED;
    }
    return MOE_OK;
}

int n_shared(const moe_dims* d) { return d->Fs / d->F; }
// rows of the expert layout: T*K routed rows, then T per shared-expert chunk
int64_t ffn_rows(const moe_dims* d) { return d->T * (int64_t)(d->K + n_shared(d)); }

moe_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    if (e == cudaErrorInvalidValue) return MOE_EINVAL;
    return MOE_ECUDA;
}

// Workspace layout: a bump allocator over the caller's buffer, 256-byte aligned.
struct Carve {
    size_t off = 0;
    template <typename T>
    T* take(void* base, size_t count) {
        off = (off + 255) & ~size_t(255);
        T* p = base ? reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off) : nullptr;
        off += count * sizeof(T);
        return p;
    }
};

struct RouteWs {
    double* P;
    double* xn2;
    double* wn2;
};
struct FfnWs {
    int4* sched;
    int* n_sched;
    int* perm_scratch;
    void* xp;            // permuted rows: bf16, E4M3 codes, or NVFP4 codes [rows][H/2]
    void* hb;            // ReLU^2 rows: bf16, E4M3 codes, or NVFP4 codes [rows][F/2]
    uint8_t* xp_block;   // NVFP4: block scales [rows][KSP(H)]
    uint8_t* hb_block;   // NVFP4: block scales [rows][KSP(F)]
    int* done;           // [max_sched] up units reported per schedule entry (one-launch FFN), then its claim counter
};
struct ForwardWs {
    int32_t* idx;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm_src;
    int32_t* inv_row;
    void* y_perm;
};

// Whether the expert FFN runs as one launch (every expert format; a shared expert, which only
// bf16 layers take, adds its chunks as entries of the same unit list).
bool fused_ffn(const moe_dims* d) {
    if (!g_fused_ffn.load()) return false;
    if (n_shared(d) > 0) return d->expert_dtype == MOE_BF16;
    return d->expert_dtype == MOE_BF16 || d->expert_dtype == MOE_FP8_E4M3 || d->expert_dtype == MOE_NVFP4 ||
           d->expert_dtype == MOE_FP8_B128;
}

// Plan of the expert FFN: one tile schedule for every expert dtype (FP8_B128
// caps a tile at 128 token rows: its epilogue keeps a tile's sums in registers;
// NVFP4 at 224: its accumulators share TMEM with the scale factors),
// plus the shared expert's entries (ns chunks of T rows, cut into tiles of at
// most bn).
GemmPlan ffn_plan(const moe_dims* d) {
    GemmPlan gp = gemm_plan(d->T, d->K, d->E);
    // The one-launch FFN takes sparse batches (experts average under 128 rows) in tiles of at
    // most 128 rows, which run two CTAs per SM: the skewed T=576 batch's FFN 292 -> 283 us
    // against 224-row tiles (hot experts split into more tiles; their weights re-read from L2).
    const bool sparse = d->T * d->K < (int64_t)kFfnSparseRows * d->E;
    const int cap = d->expert_dtype == MOE_FP8_B128 ? (fused_ffn(d) ? kB128OneLaunchTileRows : kB128MaxTileRows)
                    : d->expert_dtype == MOE_NVFP4    ? kFp4MaxTileRows
                    : fused_ffn(d) && sparse          ? kFfnSparseRows
                                                      : 0;
    if (cap > 0 && gp.bn > cap) {
        const int64_t rows = d->T * d->K;
        const int64_t nonempty = d->E < rows ? d->E : rows;
        gp.bn = cap;
        gp.max_sched = (int)(nonempty + (rows + cap - 1) / cap);
    }
    gp.max_sched += n_shared(d) * (int)((d->T + gp.bn - 1) / gp.bn);
    return gp;
}

RouteWs carve_route(Carve& c, void* base, const moe_dims* d, const RouterPlan& rp) {
    RouteWs r;
    r.P = c.take<double>(base, rp.p_bytes / sizeof(double));
    r.xn2 = c.take<double>(base, rp.xn_bytes / sizeof(double));
    r.wn2 = c.take<double>(base, rp.wn_bytes / sizeof(double));
    return r;
}

FfnWs carve_ffn(Carve& c, void* base, const moe_dims* d, const GemmPlan& gp) {
    FfnWs f;
    const size_t rows = (size_t)ffn_rows(d);
    f.sched = c.take<int4>(base, (size_t)gp.max_sched);
    f.n_sched = c.take<int>(base, 1);
    f.perm_scratch = c.take<int>(base, permute_scratch_ints(d->T * d->K, d->E));
    f.done = c.take<int>(base, (size_t)gp.max_sched + 1);   // + the FFN's unit claim counter
    f.xp_block = f.hb_block = nullptr;
    if (d->expert_dtype == MOE_NVFP4) {
        f.xp = c.take<uint8_t>(base, rows * d->H / 2);
        f.hb = c.take<uint8_t>(base, rows * d->F / 2);
        f.xp_block = c.take<uint8_t>(base, rows * nvfp4_scale_row_bytes(d->H));
        f.hb_block = c.take<uint8_t>(base, rows * nvfp4_scale_row_bytes(d->F));
        return f;
    }
    const size_t es = (d->expert_dtype == MOE_FP8_E4M3 || d->expert_dtype == MOE_FP8_B128) ? 1 : 2;
    f.xp = c.take<uint8_t>(base, rows * d->H * es);
    f.hb = c.take<uint8_t>(base, rows * d->F * es);
    return f;
}

ForwardWs carve_forward(Carve& c, void* base, const moe_dims* d) {
    ForwardWs f;
    const size_t rows = (size_t)d->T * d->K;
    f.idx = c.take<int32_t>(base, rows);
    f.w = c.take<float>(base, rows);
    f.counts = c.take<int32_t>(base, d->E);
    f.offsets = c.take<int32_t>(base, d->E + 1);
    f.perm_src = c.take<int32_t>(base, rows);
    f.inv_row = c.take<int32_t>(base, rows);
    f.y_perm = c.take<uint16_t>(base, (size_t)ffn_rows(d) * d->H);
    return f;
}

size_t route_ws_bytes(const moe_dims* d, int sms) {
    Carve c;
    carve_route(c, nullptr, d, router_plan(d->T, d->H, d->E, sms));
    return c.off;
}

size_t ffn_ws_bytes(const moe_dims* d) {
    Carve c;
    carve_ffn(c, nullptr, d, ffn_plan(d));
    return c.off;
}

size_t forward_ws_bytes(const moe_dims* d, int sms) {
    Carve c;
    carve_forward(c, nullptr, d);
    const size_t a = c.off;
    // route and ffn scratch are carved after the forward buffers, reusing one region
    const size_t r = route_ws_bytes(d, sms), f = ffn_ws_bytes(d);
    return ((a + 255) & ~size_t(255)) + (r > f ? r : f) + 256;
}

// Run the expert FFN given a schedule already in `fw`.
moe_status run_ffn(const moe_dims* d, const DeviceInfo* dev, const DevCtx& ctx, const GemmPlan& gp,
                   const void* x, const int32_t* perm_src, const void* w_up, const void* w_down,
                   const void* w_up_s, const void* w_down_s, const moe_fp8_scales* sc, FfnWs& fw, void* y_perm,
                   cudaStream_t st, bool marks = false) {
    const bool fp8 = d->expert_dtype == MOE_FP8_E4M3 || d->expert_dtype == MOE_FP8_B128;
    const int64_t rows = ffn_rows(d);
    const int ns = n_shared(d);
    if (d->expert_dtype == MOE_FP8_B128) {
        const int withhold_b = g_debug_withhold.load();
        const bool fusedb = fused_ffn(d);
        if (marks) stage_mark(3, st);
        // E4M3 codes of the permuted rows; they also zero the one-launch FFN's counters
        cudaError_t eb = launch_gather(static_cast<const uint16_t*>(x), perm_src, rows, rows, d->K, d->T, d->H,
                                       fw.xp, true, sc->x_scale, dev->num_sms, ctx, st,
                                       fusedb ? fw.done : nullptr, fusedb ? gp.max_sched + 1 : 0);
        if (eb != cudaSuccess) return cuda_status(eb);
        if (marks) stage_mark(4, st);
        if (fusedb) {
            eb = launch_grouped_ffn_b128(static_cast<const uint8_t*>(w_up), sc->w_up_scale,
                                         static_cast<const uint8_t*>(w_down), sc->w_down_scale, d->E, d->F, d->H,
                                         static_cast<const uint8_t*>(fw.xp), static_cast<uint8_t*>(fw.hb), y_perm,
                                         rows, fw.sched, fw.n_sched, gp.bn, gp.max_sched, fw.done, sc->x_scale,
                                         sc->h_scale, dev->num_sms, withhold_b, ctx, st);
            if (marks) stage_mark(5, st);
            return cuda_status(eb);
        }
        eb = launch_grouped_gemm_b128(true, static_cast<const uint8_t*>(w_up), sc->w_up_scale, d->E, d->F, d->H,
                                      static_cast<const uint8_t*>(fw.xp), rows, fw.sched, fw.n_sched, gp.bn,
                                      gp.max_sched, fw.hb, sc->x_scale, sc->h_scale, dev->num_sms, withhold_b, ctx, st);
        if (eb != cudaSuccess) return cuda_status(eb);
        if (marks) stage_mark(5, st);
        eb = launch_grouped_gemm_b128(false, static_cast<const uint8_t*>(w_down), sc->w_down_scale, d->E, d->H, d->F,
                                      static_cast<const uint8_t*>(fw.hb), rows, fw.sched, fw.n_sched, gp.bn,
                                      gp.max_sched, y_perm, sc->h_scale, 1.0f, dev->num_sms, 0, ctx, st);
        return cuda_status(eb);
    }
    if (d->expert_dtype == MOE_NVFP4) {
        const int withhold4 = g_debug_withhold.load();
        const bool fused4 = fused_ffn(d);
        if (marks) stage_mark(3, st);
        // the NVFP4 codes and block scales of the permuted rows; they also zero the one-launch
        // FFN's per-entry counters and its claim counter
        cudaError_t e4 = launch_gather_nvfp4(static_cast<const uint16_t*>(x), perm_src, rows, d->K, d->T, d->H,
                                             sc->x_scale, static_cast<uint8_t*>(fw.xp), fw.xp_block, dev->num_sms,
                                             ctx, st, fused4 ? fw.done : nullptr, fused4 ? gp.max_sched + 1 : 0);
        if (e4 != cudaSuccess) return cuda_status(e4);
        if (marks) stage_mark(4, st);
        if (fused4) {
            e4 = launch_grouped_ffn_fp4(static_cast<const uint8_t*>(w_up), sc->w_up_block, sc->w_up_scale,
                                        static_cast<const uint8_t*>(w_down), sc->w_down_block, sc->w_down_scale,
                                        d->E, d->F, d->H, static_cast<const uint8_t*>(fw.xp), fw.xp_block,
                                        sc->x_scale, sc->h_scale, static_cast<uint8_t*>(fw.hb), fw.hb_block, y_perm,
                                        rows, fw.sched, fw.n_sched, gp.bn, gp.max_sched, fw.done, dev->num_sms,
                                        withhold4, ctx, st);
            if (marks) stage_mark(5, st);
            return cuda_status(e4);
        }
        e4 = launch_grouped_gemm_fp4(true, static_cast<const uint8_t*>(w_up), sc->w_up_block, sc->w_up_scale, d->E,
                                     d->F, d->H, static_cast<const uint8_t*>(fw.xp), fw.xp_block, sc->x_scale,
                                     sc->h_scale, rows, fw.sched, fw.n_sched, gp.bn, gp.max_sched, fw.hb,
                                     fw.hb_block, dev->num_sms, withhold4, ctx, st);
        if (e4 != cudaSuccess) return cuda_status(e4);
        if (marks) stage_mark(5, st);
        e4 = launch_grouped_gemm_fp4(false, static_cast<const uint8_t*>(w_down), sc->w_down_block, sc->w_down_scale,
                                     d->E, d->H, d->F, static_cast<const uint8_t*>(fw.hb), fw.hb_block, sc->h_scale,
                                     1.0f, rows, fw.sched, fw.n_sched, gp.bn, gp.max_sched, y_perm, nullptr,
                                     dev->num_sms, 0, ctx, st);
        return cuda_status(e4);
    }
    if (marks) stage_mark(3, st);
    const int withhold = g_debug_withhold.load();
    // optional: tiles of more than 64 tokens on CTA pairs (one activation read per 256 weight rows)
    const bool pair = g_gemm_pair.load() && gp.bn > 64 && !withhold && ns == 0;
    const bool fused = fused_ffn(d) && !pair;
    // permuted copy of x (or of its E4M3 codes), read by the up projection in contiguous row blocks;
    // it also zeroes the one-launch FFN's per-entry counters
    cudaError_t e = launch_gather(static_cast<const uint16_t*>(x), perm_src, rows, d->T * d->K, d->K, d->T, d->H,
                                  fw.xp, fp8, fp8 ? sc->x_scale : 1.0f, dev->num_sms, ctx, st,
                                  fused ? fw.done : nullptr, fused ? gp.max_sched + 1 : 0);
    if (e != cudaSuccess) return cuda_status(e);
    if (fused) {
        if (marks) stage_mark(4, st);
        e = launch_grouped_ffn(fp8, w_up, w_down, d->E, d->F, d->H, fw.xp, fw.hb, y_perm, rows, fw.sched, fw.n_sched,
                               fw.done, gp, fp8 ? sc->w_up_scale : nullptr, fp8 ? sc->w_down_scale : nullptr,
                               fp8 ? sc->x_scale : 1.0f, fp8 ? sc->h_scale : 1.0f, dev->num_sms, withhold, ctx, st,
                               w_up_s, w_down_s, ns);
        if (marks) stage_mark(5, st);
        return cuda_status(e);
    }
    if (marks) stage_mark(4, st);
    if (pair)
        e = launch_grouped_gemm_pair(fp8, true, w_up, d->E, d->F, d->H, fw.xp, rows, fw.sched, fw.n_sched, gp.bn,
                                     gp.max_sched, fw.hb, fp8 ? sc->w_up_scale : nullptr, fp8 ? sc->x_scale : 1.0f,
                                     fp8 ? sc->h_scale : 1.0f, dev->num_sms, ctx, st);
    else
        e = launch_grouped_gemm(fp8, true, w_up, d->E, d->F, d->H, fw.xp, rows, fw.sched, fw.n_sched, gp, fw.hb,
                                fp8 ? sc->w_up_scale : nullptr, fp8 ? sc->x_scale : 1.0f, fp8 ? sc->h_scale : 1.0f,
                                dev->num_sms, withhold, ctx, st, w_up_s, ns);
    if (e != cudaSuccess) return cuda_status(e);
    if (marks) stage_mark(5, st);
    if (pair)
        e = launch_grouped_gemm_pair(fp8, false, w_down, d->E, d->H, d->F, fw.hb, rows, fw.sched, fw.n_sched, gp.bn,
                                     gp.max_sched, y_perm, fp8 ? sc->w_down_scale : nullptr,
                                     fp8 ? sc->h_scale : 1.0f, 1.0f, dev->num_sms, ctx, st);
    else
        e = launch_grouped_gemm(fp8, false, w_down, d->E, d->H, d->F, fw.hb, rows, fw.sched, fw.n_sched, gp, y_perm,
                                fp8 ? sc->w_down_scale : nullptr, fp8 ? sc->h_scale : 1.0f, 1.0f, dev->num_sms, 0,
                                ctx, st, w_down_s, ns);
    return cuda_status(e);
}

// The shared expert's weights: both given (16-byte aligned) exactly when Fs > 0.
moe_status check_shared(const moe_dims* d, const void* w_up_s, const void* w_down_s) {
    if (d->Fs == 0) return (w_up_s || w_down_s) ? MOE_EINVAL : MOE_OK;
    if (d->T > 0 && (!w_up_s || !w_down_s)) return MOE_EINVAL;
    return aligned(w_up_s, 16) && aligned(w_down_s, 16) ? MOE_OK : MOE_EINVAL;
}

moe_status check_fp8_scales(const moe_dims* d, const moe_fp8_scales* sc) {
    if (d->expert_dtype == MOE_BF16) return MOE_OK;
    if (!sc || !sc->w_up_scale || !sc->w_down_scale) return MOE_EINVAL;
    if (!(sc->x_scale > 0.0f) || !(sc->h_scale > 0.0f)) return MOE_EINVAL;
    if (!(sc->x_scale < 3.4e38f) || !(sc->h_scale < 3.4e38f)) return MOE_EINVAL;
    if (d->expert_dtype == MOE_NVFP4 && (!sc->w_up_block || !sc->w_down_block || !aligned(sc->w_up_block, 16) ||
                                         !aligned(sc->w_down_block, 16)))
        return MOE_EINVAL;
    return MOE_OK;
}

}  // namespace

namespace moe {
bool pdl_enabled() { return g_pdl.load() != 0; }
bool shared_map_2d() { return g_shared_2d.load() != 0; }
// Device context and argument checks for entry points defined in other files.
moe_status internal_check_dims(const moe_dims* d) { return check_dims(d); }
moe_status internal_device(DevCtx* ctx, int* num_sms) {
    DeviceInfo* dev = nullptr;
    const moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    *ctx = make_ctx(dev);
    *num_sms = dev->num_sms;
    return MOE_OK;
}
}  // namespace moe

extern "C" {

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_EINVAL: return "MOE_EINVAL: invalid argument";
        case MOE_EUNSUPPORTED: return "MOE_EUNSUPPORTED: not supported on this device or build";
        case MOE_ECUDA: return "MOE_ECUDA: CUDA runtime error";
        case MOE_ETIMEOUT: return "MOE_ETIMEOUT: a bounded wait inside a kernel expired";
        case MOE_EWORKSPACE: return "MOE_EWORKSPACE: workspace too small";
        case MOE_ERANGE: return "MOE_ERANGE: router inputs beyond the exact fixed-point range";
        case MOE_EINDEX: return "MOE_EINDEX: expert or row index out of range";
    }
    return "unknown moe_status";
}

int moe_abi_version(void) { return MOE_ABI_VERSION; }

moe_status moe_workspace_size(const moe_dims* d, size_t* bytes) {
    moe_status s = check_dims(d);
    if (s != MOE_OK) return s;
    if (!bytes) return MOE_EINVAL;
    // plans depend on the SM count only through the router split; size for
    // the largest split any device can choose
    *bytes = forward_ws_bytes(d, 1024);
    return MOE_OK;
}

moe_status moe_forward_launches(const moe_dims* d, int32_t* launches) {
    moe_status s = check_dims(d);
    if (s != MOE_OK) return s;
    if (!launches) return MOE_EINVAL;
    if (d->T == 0) {
        *launches = 0;
        return MOE_OK;
    }
    int n = route_launches(d->T, d->H, d->E);
    n += permute_scratch_ints(d->T * d->K, d->E) == 0 ? 1 : 3;   // one block, or histogram + scan + scatter
    // row gather, up and down projections (one launch or two), combine
    const bool pair = (d->expert_dtype == MOE_BF16 || d->expert_dtype == MOE_FP8_E4M3) && g_gemm_pair.load() &&
                      gemm_plan(d->T, d->K, d->E).bn > 64;
    n += 1 + (fused_ffn(d) && !pair ? 1 : 2) + 1;
    *launches = n;
    return MOE_OK;
}

moe_status moe_route(const moe_dims* d, const void* x, const void* w_router, const float* bias,
                     int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
    moe_status s = check_dims(d);
    if (s != MOE_OK) return s;
    if (d->T > 0 && (!x || !w_router || !topk_idx || !topk_w || !ws)) return MOE_EINVAL;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(ws, 256)) return MOE_EINVAL;
    if (d->T == 0) return MOE_OK;
    DeviceInfo* dev = nullptr;
    if ((s = device_setup(&dev)) != MOE_OK) return s;
    const RouterPlan rp = router_plan(d->T, d->H, d->E, dev->num_sms);
    Carve c;
    RouteWs rw = carve_route(c, ws, d, rp);
    if (c.off > ws_bytes) return MOE_EWORKSPACE;
    return cuda_status(launch_route(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w_router), bias,
                                    d->T, d->H, d->E, d->K, topk_idx, topk_w, rw.P, rw.xn2, rw.wn2, rp,
                                    make_ctx(dev), static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const moe_dims* d, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                       int32_t* perm_src, int32_t* inv_row, void* ws, size_t ws_bytes, void* stream) {
    moe_status s = check_dims(d);
    if (s != MOE_OK) return s;
    if (!counts || !offsets) return MOE_EINVAL;
    if (d->T > 0 && (!topk_idx || !perm_src || !inv_row)) return MOE_EINVAL;
    const size_t need = permute_scratch_ints(d->T * d->K, d->E) * sizeof(int);
    if (need > 0 && (!ws || ws_bytes < need)) return MOE_EWORKSPACE;
    if (!aligned(ws, 256)) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    if ((s = device_setup(&dev)) != MOE_OK) return s;
    return cuda_status(launch_permute(topk_idx, d->T * d->K, d->K, d->E, counts, offsets, perm_src, inv_row, nullptr,
                                      nullptr, 16, 0, static_cast<int*>(ws), make_ctx(dev),
                                      static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(const moe_dims* d, const void* x, const int32_t* offsets, const int32_t* perm_src,
                          const void* w_up, const void* w_down, const void* w_up_shared, const void* w_down_shared,
                          const moe_fp8_scales* scales, void* y_perm, void* ws, size_t ws_bytes, void* stream) {
    moe_status s = check_dims(d);
    if (s != MOE_OK) return s;
    if ((s = check_fp8_scales(d, scales)) != MOE_OK) return s;
    if ((s = check_shared(d, w_up_shared, w_down_shared)) != MOE_OK) return s;
    if (d->T > 0 && (!x || !offsets || !perm_src || !w_up || !w_down || !y_perm || !ws)) return MOE_EINVAL;
    if (!aligned(x, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) || !aligned(y_perm, 16) || !aligned(ws, 256))
        return MOE_EINVAL;
    if (d->T == 0) return MOE_OK;
    DeviceInfo* dev = nullptr;
    if ((s = device_setup(&dev)) != MOE_OK) return s;
    const GemmPlan gp = ffn_plan(d);
    Carve c;
    FfnWs fw = carve_ffn(c, ws, d, gp);
    if (c.off > ws_bytes) return MOE_EWORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_schedule(offsets, d->E, gp.bn, fw.sched, fw.n_sched, n_shared(d), d->T, d->K, st);
    if (e != cudaSuccess) return cuda_status(e);
    return run_ffn(d, dev, make_ctx(dev), gp, x, perm_src, w_up, w_down, w_up_shared, w_down_shared, scales, fw,
                   y_perm, st);
}

moe_status moe_combine(const moe_dims* d, const void* y_perm, const int32_t* inv_row, const float* topk_w,
                       const void* residual, void* out, void* stream) {
    moe_status s = check_dims(d);
    if (s != MOE_OK) return s;
    if (d->T > 0 && (!y_perm || !inv_row || !topk_w || !out)) return MOE_EINVAL;
    if (!aligned(y_perm, 16) || !aligned(residual, 16) || !aligned(out, 16)) return MOE_EINVAL;
    if (d->T == 0) return MOE_OK;
    DeviceInfo* dev = nullptr;
    if ((s = device_setup(&dev)) != MOE_OK) return s;
    return cuda_status(launch_combine(static_cast<const uint16_t*>(y_perm), inv_row, topk_w,
                                      static_cast<const uint16_t*>(residual), static_cast<uint16_t*>(out), d->T,
                                      d->K, n_shared(d), d->H, dev->num_sms, make_ctx(dev),
                                      static_cast<cudaStream_t>(stream)));
}

moe_status moe_forward(const moe_dims* d, const void* x, const void* w_router, const float* bias, const void* w_up,
                       const void* w_down, const void* w_up_shared, const void* w_down_shared,
                       const moe_fp8_scales* scales, const void* residual, void* out, int32_t* topk_idx,
                       float* topk_w, void* ws, size_t ws_bytes, void* stream) {
    moe_status s = check_dims(d);
    if (s != MOE_OK) return s;
    if ((s = check_fp8_scales(d, scales)) != MOE_OK) return s;
    if ((s = check_shared(d, w_up_shared, w_down_shared)) != MOE_OK) return s;
    if (d->T > 0 && (!x || !w_router || !w_up || !w_down || !out || !ws)) return MOE_EINVAL;
    if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) ||
        !aligned(residual, 16) || !aligned(out, 16) || !aligned(ws, 256))
        return MOE_EINVAL;
    if (d->T == 0) return MOE_OK;
    DeviceInfo* dev = nullptr;
    if ((s = device_setup(&dev)) != MOE_OK) return s;
    if (ws_bytes < forward_ws_bytes(d, dev->num_sms)) return MOE_EWORKSPACE;
    const DevCtx ctx = make_ctx(dev);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    Carve c;
    ForwardWs fw = carve_forward(c, ws, d);
    const size_t scratch = (c.off + 255) & ~size_t(255);
    void* sbase = static_cast<uint8_t*>(ws) + scratch;
    int32_t* idx = topk_idx ? topk_idx : fw.idx;
    float* w = topk_w ? topk_w : fw.w;

    const RouterPlan rp = router_plan(d->T, d->H, d->E, dev->num_sms);
    Carve cr;
    RouteWs rw = carve_route(cr, sbase, d, rp);
    stage_mark(0, st);
    // the bf16 up bank's leading bytes (expert 0 first), bounded by its size
    const int64_t warm =
        d->expert_dtype == MOE_BF16 ? std::min(g_l2_warm.load(), (int64_t)d->E * d->F * d->H * 2) : 0;
    cudaError_t e = launch_route(static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w_router), bias, d->T,
                                 d->H, d->E, d->K, idx, w, rw.P, rw.xn2, rw.wn2, rp, ctx, st,
                                 g_stage_events_on.load() ? mark_stage1 : nullptr, w_up, warm);
    if (e != cudaSuccess) return cuda_status(e);

    const GemmPlan gp = ffn_plan(d);
    Carve cf;
    FfnWs ffw = carve_ffn(cf, sbase, d, gp);   // reuses the router scratch region
    stage_mark(2, st);
    e = launch_permute(idx, d->T * d->K, d->K, d->E, fw.counts, fw.offsets, fw.perm_src, fw.inv_row, ffw.sched,
                       ffw.n_sched, gp.bn, n_shared(d), ffw.perm_scratch, ctx, st);
    if (e != cudaSuccess) return cuda_status(e);
    s = run_ffn(d, dev, ctx, gp, x, fw.perm_src, w_up, w_down, w_up_shared, w_down_shared, scales, ffw, fw.y_perm,
                st, true);
    if (s != MOE_OK) return s;
    stage_mark(6, st);
    e = launch_combine(static_cast<const uint16_t*>(fw.y_perm), fw.inv_row, w,
                       static_cast<const uint16_t*>(residual), static_cast<uint16_t*>(out), d->T, d->K,
                       n_shared(d), d->H, dev->num_sms, ctx, st);
    stage_mark(7, st);
    return cuda_status(e);
}

moe_status moe_gather_rows(int64_t rows, int64_t src_rows, int32_t H, int32_t K, const void* x,
                           const int32_t* perm_src, void* out, void* stream) {
    if (rows < 0 || src_rows < 0 || K < 1 || H < 8 || H % 8 != 0 || rows >= ((int64_t)1 << 31)) return MOE_EINVAL;
    if (rows == 0) return MOE_OK;
    if (!x || !perm_src || !out || !aligned(x, 16) || !aligned(out, 16)) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_gather(static_cast<const uint16_t*>(x), perm_src, rows, rows, K, src_rows, H, out,
                                     false, 1.0f, dev->num_sms, make_ctx(dev), static_cast<cudaStream_t>(stream)));
}

moe_status moe_ep_regroup(int32_t W, int32_t E_loc, int64_t R, const int64_t* recv_counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv, void* stream) {
    if (W < 1 || E_loc < 1 || (int64_t)W * E_loc > 256 || R < 0 || R >= ((int64_t)1 << 31)) return MOE_EINVAL;
    if (!recv_counts || !offsets || (R > 0 && (!perm || !inv))) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_ep_regroup(recv_counts, W, E_loc, R, offsets, perm, inv, make_ctx(dev),
                                         static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_fp8(int64_t n_tensors, int64_t tensor_elems, const void* src, uint8_t* codes,
                            float* scales, void* stream) {
    if (n_tensors < 0 || tensor_elems < 0 || n_tensors > ((int64_t)1 << 31)) return MOE_EINVAL;
    if (n_tensors == 0 || tensor_elems == 0) return MOE_OK;
    if (!src || !codes || !scales || !aligned(src, 16) || !aligned(scales, 4)) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_quantize(n_tensors, tensor_elems, static_cast<const uint16_t*>(src), codes, scales,
                                       dev->num_sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_fp8_b128(int64_t n_tensors, int64_t rows, int32_t K, const void* src, uint8_t* codes,
                                 float* scales, void* stream) {
    if (n_tensors < 0 || rows < 0 || K < 16 || K > 65536 || K % 16 != 0) return MOE_EINVAL;
    if (n_tensors == 0 || rows == 0) return MOE_OK;
    if (!src || !codes || !scales || !aligned(codes, 4) || !aligned(scales, 4)) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_quantize_fp8_b128(n_tensors * rows, K, static_cast<const uint16_t*>(src), codes, scales,
                                                dev->num_sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_nvfp4(int64_t n_tensors, int64_t rows, int32_t K, const void* src, uint8_t* codes,
                              uint8_t* block, float* tscale, void* stream) {
    if (n_tensors < 0 || rows < 0 || K < 32 || K > 65536 || K % 32 != 0) return MOE_EINVAL;
    if (n_tensors == 0 || rows == 0) return MOE_OK;
    if (!src || !codes || !block || !tscale || !aligned(src, 16) || !aligned(codes, 8) || !aligned(tscale, 4))
        return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_quantize_nvfp4(n_tensors, rows, K, static_cast<const uint16_t*>(src), codes, block,
                                             tscale, dev->num_sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_act_nvfp4(int64_t rows, int32_t H, float x_scale, const void* x, uint8_t* codes,
                                  uint8_t* block, void* stream) {
    if (rows < 0 || H < 32 || H > 65536 || H % 32 != 0) return MOE_EINVAL;
    if (!(x_scale > 0.0f) || !(x_scale < 3.4e38f)) return MOE_EINVAL;
    if (rows == 0) return MOE_OK;
    if (!x || !codes || !block || !aligned(x, 16) || !aligned(codes, 8)) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_gather_nvfp4(static_cast<const uint16_t*>(x), nullptr, rows, 1, rows, H, x_scale,
                                           codes, block, dev->num_sms, make_ctx(dev),
                                           static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_act_fp8(int64_t rows, int32_t H, float x_scale, const void* x, uint8_t* codes,
                                void* stream) {
    if (rows < 0 || H < 16 || H > 65536 || H % 16 != 0) return MOE_EINVAL;
    if (!(x_scale > 0.0f) || !(x_scale < 3.4e38f)) return MOE_EINVAL;
    if (rows == 0) return MOE_OK;
    if (!x || !codes || !aligned(x, 16) || !aligned(codes, 16)) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_gather(static_cast<const uint16_t*>(x), nullptr, rows, rows, 1, rows, H, codes, true,
                                     x_scale, dev->num_sms, make_ctx(dev), static_cast<cudaStream_t>(stream)));
}

moe_status moe_rmsnorm(int64_t T, int32_t H, float eps, const void* x, void* u, void* stream) {
    if (T < 0 || H < 16 || H > 65536 || H % 16 != 0 || !(eps >= 0.0f)) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!x || !u || x == u || !aligned(x, 16) || !aligned(u, 16)) return MOE_EINVAL;
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    return cuda_status(launch_rmsnorm(static_cast<const uint16_t*>(x), static_cast<uint16_t*>(u), T, H, eps,
                                      dev->num_sms, static_cast<cudaStream_t>(stream)));
}

moe_status moe_check_device_error(void* stream) {
    DeviceInfo* dev = nullptr;
    moe_status s = device_setup(&dev);
    if (s != MOE_OK) return s;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ECUDA;
    int v = 0;
    if (cudaMemcpy(&v, dev->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ECUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(dev->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ECUDA;
        return static_cast<moe_status>(v);
    }
    return MOE_OK;
}

moe_status moe_set_stage_events(void* const* events, int32_t n) {
    if (n == 0) {
        g_stage_events_on.store(0);
        return MOE_OK;
    }
    if (n != MOE_STAGE_EVENTS || !events) return MOE_EINVAL;
    for (int i = 0; i < n; ++i) {
        if (!events[i]) return MOE_EINVAL;
        g_stage_events[i] = events[i];
    }
    g_stage_events_on.store(1);
    return MOE_OK;
}

moe_status moe_debug_set(int32_t what, int64_t value) {
    if (what == 1) {
        g_timeout_ns.store(value > 0 ? (uint64_t)value : kDefaultTimeoutNs);
        return MOE_OK;
    }
    if (what == 2) {
        g_debug_withhold.store(value ? 1 : 0);
        return MOE_OK;
    }
    if (what == 3) {
        g_gemm_pair.store(value ? 1 : 0);
        return MOE_OK;
    }
    if (what == 4) {
        set_router_small_max(value);
        return MOE_OK;
    }
    if (what == 6) {
        g_pdl.store(value ? 1 : 0);
        return MOE_OK;
    }
    if (what == 7) {
        g_shared_2d.store(value ? 1 : 0);
        return MOE_OK;
    }
    if (what == 8) {
        g_fused_ffn.store(value ? 1 : 0);
        return MOE_OK;
    }
    if (what == 9) {
        g_l2_warm.store(value < 0 ? kL2WarmDefault : value);
        return MOE_OK;
    }
    if (what == 5) {
        if (value < 0 || value > 3) return MOE_EINVAL;
        set_router_split((int)value);
        return MOE_OK;
    }
    return MOE_EINVAL;
}

}  // extern "C"
