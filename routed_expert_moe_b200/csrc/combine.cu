// Memory-bound kernels around the expert products: the weighted combine, the
// RMS normalisation of the chained stack, and the per-tensor E4M3 weight
// quantiser.  All are HBM-bound streams: one warp per row, 16-byte accesses.
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

// out[t] = (residual[t] +) sum_{k=0..K-1} w[t][k] * y_perm[inv_row[t*K+k]]
// in fp32, k ascending (descending routing logit), one rounding to bf16.
// One warp per (token, chunk of 64 16-byte vectors), grid-stride: lane
// k < K loads the token's k-th row index and weight, the others get them by
// shuffle; each lane then loads two vectors of all K rows at once (2K loads
// in flight).  Small batches thus still spread over the whole GPU.
// KMAX (8 or 16) bounds K + ns at compile time so that the vectors stay in
// registers.  With a shared expert of ns chunks, slots k = K + j add row
// T*K + j*T + t with weight 1 after the routed terms (the shared expert joins
// the routed sum with weight 1).
constexpr int CB_THREADS = 256;

template <int KMAX>
__global__ void __launch_bounds__(CB_THREADS) combine_kernel(const uint16_t* __restrict__ yp,
                                                             const int32_t* __restrict__ inv_row,
                                                             const float* __restrict__ w,
                                                             const uint16_t* residual, uint16_t* out,
                                                             int64_t T, int K, int ns, int H,
                                                             int64_t rows, DevCtx ctx) {
    pdl_enter();
    const int lane = threadIdx.x % 32;
    const int nv = H / 8;
    const int wpb = blockDim.x / 32;
    const int64_t warps = (int64_t)gridDim.x * wpb;
    const int nchunk = (nv + 63) / 64;
    for (int64_t item = (int64_t)blockIdx.x * wpb + threadIdx.x / 32; item < T * nchunk; item += warps) {
        const int64_t t = item / nchunk;
        const int v0 = (int)(item - t * nchunk) * 64 + lane;
        int my_r = 0;
        float my_w = 0.0f;
        if (lane < K) {
            my_r = inv_row[t * K + lane];
            my_w = w[t * K + lane];
            if (my_r < 0 || my_r >= rows) {
                record_error(ctx.err, MOE_EINDEX);
                my_r = 0;
                my_w = 0.0f;
            }
        } else if (lane < K + ns) {
            my_r = (int)(T * K + (lane - K) * T + t);
            my_w = 1.0f;
        }
        const int KT = K + ns;   // terms of the sum
        const uint4* src[KMAX];
        float wk[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            const int r = __shfl_sync(0xffffffffu, my_r, k);
            wk[k] = __shfl_sync(0xffffffffu, my_w, k);
            src[k] = reinterpret_cast<const uint4*>(yp + (int64_t)r * H);
        }
        const uint4* res = residual ? reinterpret_cast<const uint4*>(residual + t * H) : nullptr;
        uint4* dst = reinterpret_cast<uint4*>(out + t * H);
        if (v0 < nv) {
            const int v1 = v0 + 32;
            const bool has1 = v1 < nv;
            uint4 q0[KMAX], q1[KMAX];
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k < KT) {
                    q0[k] = src[k][v0];
                    if (has1) q1[k] = src[k][v1];
                }
            }
            uint4 r0, r1;
            if (res) {
                r0 = res[v0];
                if (has1) r1 = res[v1];
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (half == 1 && !has1) break;
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll
                for (int k = 0; k < KMAX; ++k) {
                    if (k >= KT) break;
                    const uint4 q = half ? q1[k] : q0[k];
                    const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[2 * j] = __fmaf_rn(wk[k], __uint_as_float(qq[j] << 16), acc[2 * j]);
                        acc[2 * j + 1] = __fmaf_rn(wk[k], __uint_as_float(qq[j] & 0xFFFF0000u), acc[2 * j + 1]);
                    }
                }
                if (res) {
                    const uint4 r4 = half ? r1 : r0;
                    const uint32_t qq[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[2 * j] = __fadd_rn(__uint_as_float(qq[j] << 16), acc[2 * j]);
                        acc[2 * j + 1] = __fadd_rn(__uint_as_float(qq[j] & 0xFFFF0000u), acc[2 * j + 1]);
                    }
                }
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * j]));
                    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * j + 1]));
                    o[j] = lo | (hi << 16);
                }
                dst[half ? v1 : v0] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

// u = bf16(x / sqrt(mean(x^2) + eps)): sum of squares in fixed point (each
// x^2, exact in fp32, rounded to 2^-16 and summed exactly in int64), the rest
// in correctly rounded fp32, so the result is bit-reproducible anywhere.
__global__ void __launch_bounds__(256) rmsnorm_kernel(const uint16_t* __restrict__ x,
                                                      uint16_t* __restrict__ u, int64_t T, int H,
                                                      float eps) {
    pdl_enter();
    const int lane = threadIdx.x % 32;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    const int nv = H / 8;
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; t < T; t += warps) {
        const uint4* xr = reinterpret_cast<const uint4*>(x + t * H);
        long long acc = 0;
        for (int v = lane; v < nv; v += 32) {
            const uint4 q = xr[v];
            const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float f = __uint_as_float((j & 1) ? (qq[j / 2] & 0xFFFF0000u) : (qq[j / 2] << 16));
                acc += __float2ll_rn(__fmul_rn(__fmul_rn(f, f), 65536.0f));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        float ms = __ll2float_rn(acc);
        ms = __fmul_rn(ms, 1.0f / 65536.0f);
        ms = __fdiv_rn(ms, (float)H);
        ms = __fadd_rn(ms, eps);
        const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(ms));
        uint4* ur = reinterpret_cast<uint4*>(u + t * H);
        for (int v = lane; v < nv; v += 32) {
            const uint4 q = xr[v];
            const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float a = __fmul_rn(__uint_as_float(qq[j] << 16), rstd);
                const float b = __fmul_rn(__uint_as_float(qq[j] & 0xFFFF0000u), rstd);
                o[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a)) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b)) << 16);
            }
            ur[v] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// amax over each tensor (as the bits of |v|, which order like the values).
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ src, int64_t elems,
                                                   unsigned int* __restrict__ amax_bits) {
    pdl_enter();
    const int64_t tensor = blockIdx.y;
    const uint16_t* p = src + tensor * elems;
    uint32_t m = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < elems; i += stride) {
        const uint32_t b = ((uint32_t)p[i] << 16) & 0x7FFFFFFFu;
        m = max(m, b);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) atomicMax(&amax_bits[tensor], m);
}

// scale = amax / 448 (1 for an all-zero tensor), in place over the amax bits.
__global__ void finalize_scale_kernel(float* scales, int64_t n) {
    pdl_enter();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        const float amax = __uint_as_float(reinterpret_cast<unsigned int*>(scales)[i]);
        scales[i] = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    }
}

__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ src, int64_t elems,
                                                       const float* __restrict__ scales,
                                                       uint8_t* __restrict__ codes) {
    pdl_enter();
    const int64_t tensor = blockIdx.y;
    const float s = scales[tensor];
    const uint16_t* p = src + tensor * elems;
    uint8_t* q = codes + tensor * elems;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < elems; i += stride) {
        const float v = __uint_as_float((uint32_t)p[i] << 16);
        q[i] = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(v, s), __NV_SATFINITE, __NV_E4M3);
    }
}

// ----------------------------------------------------------------------------- host

static unsigned grid_rows(int64_t rows, int num_sms) {
    int64_t b = (rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 8;
    if (b > cap) b = cap;
    return (unsigned)(b > 0 ? b : 1);
}

cudaError_t launch_combine(const uint16_t* yp, const int32_t* inv_row, const float* w,
                           const uint16_t* residual, uint16_t* out, int64_t T, int K, int ns, int H,
                           int num_sms, const DevCtx& ctx, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    // warps per block: small batches spread over the SMs, large ones 8 per block
    const int64_t items = T * ((H / 8 + 63) / 64);
    int64_t wpb = items / num_sms;
    if (wpb < 1) wpb = 1;
    if (wpb > CB_THREADS / 32) wpb = CB_THREADS / 32;
    const int64_t cap = (int64_t)num_sms * 16;
    int64_t blocks = (items + wpb - 1) / wpb;
    if (blocks > cap) blocks = cap;
    const dim3 grid((unsigned)blocks), block((unsigned)(32 * wpb));
    const int64_t rows = T * K;   // routed rows: the range inv_row may name
    if (K + ns <= 8)
        return launch_k(combine_kernel<8>, grid, block, 0, stream, yp, inv_row, w, residual, out, T, K, ns, H, rows,
                        ctx);
    return launch_k(combine_kernel<16>, grid, block, 0, stream, yp, inv_row, w, residual, out, T, K, ns, H, rows,
                    ctx);
}

cudaError_t launch_rmsnorm(const uint16_t* x, uint16_t* u, int64_t T, int H, float eps, int num_sms,
                           cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    return launch_k(rmsnorm_kernel, dim3(grid_rows(T, num_sms)), dim3(256), 0, stream, x, u, T, H, eps);
}

cudaError_t launch_quantize(int64_t n_tensors, int64_t elems, const uint16_t* src, uint8_t* codes,
                            float* scales, int num_sms, cudaStream_t stream) {
    if (n_tensors == 0 || elems == 0) return cudaSuccess;
    cudaError_t err = cudaMemsetAsync(scales, 0, (size_t)n_tensors * sizeof(float), stream);
    if (err != cudaSuccess) return err;
    int64_t bx = (elems + 255) / 256;
    const int64_t cap = (n_tensors >= num_sms) ? 4 : (int64_t)num_sms * 8 / n_tensors + 1;
    if (bx > cap) bx = cap;
    for (int64_t t0 = 0; t0 < n_tensors; t0 += 65535) {
        const int64_t nt = n_tensors - t0 < 65535 ? n_tensors - t0 : 65535;
        amax_kernel<<<dim3((unsigned)bx, (unsigned)nt), 256, 0, stream>>>(
            src + t0 * elems, elems, reinterpret_cast<unsigned int*>(scales) + t0);
    }
    finalize_scale_kernel<<<(unsigned)((n_tensors + 255) / 256), 256, 0, stream>>>(scales, n_tensors);
    for (int64_t t0 = 0; t0 < n_tensors; t0 += 65535) {
        const int64_t nt = n_tensors - t0 < 65535 ? n_tensors - t0 : 65535;
        quantize_kernel<<<dim3((unsigned)bx, (unsigned)nt), 256, 0, stream>>>(src + t0 * elems, elems,
                                                                              scales + t0, codes + t0 * elems);
    }
    return cudaGetLastError();
}

}  // namespace moe
