// FP8 (E4M3) quantisation for the projection GEMMs (the ULTRA-HSTU review in
// the pages: its mixed-precision item keeps most of the layer in bf16 and runs
// the matrix multiplications in FP8).  Activations are scaled per row, weights
// per output column, so that the largest magnitude maps to 448, the largest
// finite E4M3 value:  inv = 448 / amax, scale = amax / 448 (float32, correctly
// rounded), code = E4M3(x * inv) rounded to nearest even and saturated; an
// all-zero row gets scale 1.  The GEMM multiplies the float32 accumulator by
// the row and column scales in its epilogue.
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace hstu {

namespace {

constexpr float kE4M3Max = 448.f;

// two E4M3 codes, lo in the low byte
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ void bf16x8(const uint4 &w, float *v)
{
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; e++) {
        v[2 * e] = __uint_as_float(ww[e] << 16);
        v[2 * e + 1] = __uint_as_float(ww[e] & 0xffff0000u);
    }
}

// one warp per row, eight elements per lane and pass
__global__ void __launch_bounds__(256)
quantize_rows_kernel(const __nv_bfloat16 *__restrict__ x, int64_t ldx, int64_t R, int K, unsigned char *__restrict__ q,
                     int64_t ldq, float *__restrict__ scale)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < R; row += warps) {
        const __nv_bfloat16 *xr = x + row * ldx;
        float amax = 0.f;
        for (int c = lane * 8; c < K; c += 256) {
            float v[8];
            bf16x8(*reinterpret_cast<const uint4 *>(xr + c), v);
#pragma unroll
            for (int e = 0; e < 8; e++)
                amax = fmaxf(amax, fabsf(v[e]));
        }
#pragma unroll
        for (int off = 16; off; off >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float inv = amax > 0.f ? __fdiv_rn(kE4M3Max, amax) : 1.f;
        if (lane == 0)
            scale[row] = amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
        unsigned char *qr = q + row * ldq;
        for (int c = lane * 8; c < K; c += 256) {
            float v[8];
            bf16x8(*reinterpret_cast<const uint4 *>(xr + c), v);
            uint2 out;
            out.x = e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)) |
                    (e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)) << 16);
            out.y = e4m3x2(__fmul_rn(v[4], inv), __fmul_rn(v[5], inv)) |
                    (e4m3x2(__fmul_rn(v[6], inv), __fmul_rn(v[7], inv)) << 16);
            *reinterpret_cast<uint2 *>(qr + c) = out;
        }
    }
}

// one thread per output column n of w [K, N]: its amax over K, then its codes
// written as row n of q [N, K]
__global__ void __launch_bounds__(256)
quantize_cols_kernel(const __nv_bfloat16 *__restrict__ w, int64_t K, int N, unsigned char *__restrict__ q,
                     float *__restrict__ scale)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N)
        return;
    float amax = 0.f;
    for (int64_t k = 0; k < K; k++)
        amax = fmaxf(amax, fabsf(__bfloat162float(w[k * N + n])));
    const float inv = amax > 0.f ? __fdiv_rn(kE4M3Max, amax) : 1.f;
    scale[n] = amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f;
    // sixteen codes per 16-byte store (K is a multiple of 16); the loads of each
    // k are coalesced across the block's columns
    unsigned char *qr = q + (int64_t)n * K;
    for (int64_t k = 0; k < K; k += 16) {
        uint32_t c[8];
#pragma unroll
        for (int e = 0; e < 8; e++)
            c[e] = e4m3x2(__fmul_rn(__bfloat162float(w[(k + 2 * e) * N + n]), inv),
                          __fmul_rn(__bfloat162float(w[(k + 2 * e + 1) * N + n]), inv));
        *reinterpret_cast<uint4 *>(qr + k) = make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16),
                                                        c[4] | (c[5] << 16), c[6] | (c[7] << 16));
    }
}

}  // namespace

cudaError_t launch_quantize_rows_e4m3(const void *x, int64_t ldx, int64_t R, int K, void *q, int64_t ldq,
                                      float *scale, cudaStream_t stream)
{
    if (R == 0)
        return cudaSuccess;
    const unsigned blocks = (unsigned)std::min<int64_t>((R + 7) / 8, (int64_t)device_info().sms * 8);
    quantize_rows_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(x), ldx, R, K,
                                                     static_cast<unsigned char *>(q), ldq, scale);
    return cudaGetLastError();
}

cudaError_t launch_quantize_cols_e4m3(const void *w, int64_t K, int N, void *q, float *scale, cudaStream_t stream)
{
    if (N == 0)
        return cudaSuccess;
    quantize_cols_kernel<<<(N + 255) / 256, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(w), K, N,
                                                              static_cast<unsigned char *>(q), scale);
    return cudaGetLastError();
}

}  // namespace hstu
