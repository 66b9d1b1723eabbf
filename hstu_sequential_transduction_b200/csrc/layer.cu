// Projection GEMMs and the LayerNorm-gate of the HSTU transduction layer
// ("DLRMv4 Brings Sequence-Based Recommendation Training to MLPerf", section
// "Model Architecture": a projection producing the layer's internal
// representations, then a gated transformation of the attention output).
//
//   f1:   [U | V | Q | K] = SiLU(X W1 + b1)   (bias + SiLU fused in the epilogue;
//         the four blocks are column ranges of one output, so the attention
//         reads Q, K, V in place through row strides: no split copies)
//   gate: G = LayerNorm(O) * U                 (fp32 stats; each warp walks a strided
//         set of tokens with the next tokens' O and U rows already in flight)
//   f2:   Y = G W2 + b2
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace hstu {

namespace {

// ---- fp32 GEMM on CUDA cores ---------------------------------------------------
constexpr int FT = 64, FK = 16;

__global__ void __launch_bounds__(256)
gemm_f32_kernel(const float *__restrict__ A, int64_t lda, const float *__restrict__ Bm,
                const float *__restrict__ bias, float *__restrict__ C, int64_t ldc, int64_t M, int N,
                int K, int silu)
{
    __shared__ float sA[FK][FT + 1];
    __shared__ float sB[FK][FT];
    const int64_t m0 = (int64_t)blockIdx.y * FT;
    const int n0 = blockIdx.x * FT;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += FK) {
        for (int e = threadIdx.x; e < FT * FK; e += 256) {
            int r = e / FK, c = e % FK;
            sA[c][r] = (m0 + r < M && k0 + c < K) ? A[(m0 + r) * lda + k0 + c] : 0.f;
            int rb = e / FT, cb = e % FT;
            sB[rb][cb] = (k0 + rb < K && n0 + cb < N) ? Bm[(int64_t)(k0 + rb) * N + n0 + cb] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < FK; kk++) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                a[i] = sA[kk][ty * 4 + i];
                b[i] = sB[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++)
                    acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int64_t row = m0 + ty * 4 + i;
        if (row >= M)
            continue;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int col = n0 + tx * 4 + j;
            if (col >= N)
                continue;
            float x = acc[i][j] + (bias ? bias[col] : 0.f);
            C[row * ldc + col] = silu ? silu_precise(x) : x;
        }
    }
}

// ---- LayerNorm(O) * U ----------------------------------------------------------
template <typename T>
__device__ __forceinline__ float ld(const T *p);
template <>
__device__ __forceinline__ float ld<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ void st(T *p, float v);
template <>
__device__ __forceinline__ void st<float>(float *p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

// VPT contiguous elements of a row as floats, with the widest aligned vector loads.
template <typename T, int VPT>
__device__ __forceinline__ void load_vec(const T *p, float *x)
{
    constexpr int BYTES = VPT * (int)sizeof(T);
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
        for (int b = 0; b < BYTES / 16; b++) {
            const uint4 w = __ldg(reinterpret_cast<const uint4 *>(p) + b);
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
            if constexpr (sizeof(T) == 2) {
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&u[k]);
                    x[8 * b + 2 * k] = __low2float(h);
                    x[8 * b + 2 * k + 1] = __high2float(h);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 4; k++)
                    x[4 * b + k] = __uint_as_float(u[k]);
            }
        }
    } else {
#pragma unroll
        for (int e = 0; e < VPT; e++)
            x[e] = ld<T>(p + e);
    }
}

template <typename T, int VPT>
__device__ __forceinline__ void store_vec(T *p, const float *y)
{
    constexpr int BYTES = VPT * (int)sizeof(T);
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
        for (int b = 0; b < BYTES / 16; b++) {
            uint4 w;
            if constexpr (sizeof(T) == 2) {
                w.x = pack_bf16(y[8 * b], y[8 * b + 1]);
                w.y = pack_bf16(y[8 * b + 2], y[8 * b + 3]);
                w.z = pack_bf16(y[8 * b + 4], y[8 * b + 5]);
                w.w = pack_bf16(y[8 * b + 6], y[8 * b + 7]);
            } else {
                w.x = __float_as_uint(y[4 * b]);
                w.y = __float_as_uint(y[4 * b + 1]);
                w.z = __float_as_uint(y[4 * b + 2]);
                w.w = __float_as_uint(y[4 * b + 3]);
            }
            reinterpret_cast<uint4 *>(p)[b] = w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < VPT; e++)
            st<T>(p + e, y[e]);
    }
}

// One warp per token at a time; lane l holds features l*VPT .. l*VPT + VPT - 1,
// moved with 16-byte vector loads and stores (memory-bound: read O and U, write
// G).  Each warp walks the tokens warp, warp + W, ... (W = warps of the grid):
// gamma and beta stay in registers, and the O and U rows of the next two tokens
// are kept in flight as raw 16-byte words while this token is normalised.
template <typename T, int VPT>
struct RawRow {
    static constexpr int WORDS = VPT * (int)sizeof(T) / 16;  // 16-byte words per lane
    uint4 w[WORDS];
};

template <typename T, int VPT>
__device__ __forceinline__ void raw_load(const T *p, RawRow<T, VPT> &r)
{
#pragma unroll
    for (int b = 0; b < RawRow<T, VPT>::WORDS; b++)
        r.w[b] = __ldg(reinterpret_cast<const uint4 *>(p) + b);
}

template <typename T, int VPT>
__device__ __forceinline__ void raw_unpack(const RawRow<T, VPT> &r, float *x)
{
#pragma unroll
    for (int b = 0; b < RawRow<T, VPT>::WORDS; b++) {
        const uint32_t u[4] = {r.w[b].x, r.w[b].y, r.w[b].z, r.w[b].w};
        if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162 *>(&u[k]);
                x[8 * b + 2 * k] = __low2float(h);
                x[8 * b + 2 * k + 1] = __high2float(h);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 4; k++)
                x[4 * b + k] = __uint_as_float(u[k]);
        }
    }
}

template <typename T, int VPT>
__global__ void __launch_bounds__(256)
norm_gate_kernel(const T *__restrict__ O, int64_t ldo, const T *__restrict__ U, int64_t ldu,
                 const float *__restrict__ gamma, const float *__restrict__ beta, float eps,
                 T *__restrict__ G, int64_t ldg, int64_t Trows)
{
    static_assert(VPT * sizeof(T) % 16 == 0, "16-byte words per lane");
    constexpr int F = 32 * VPT;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (row >= Trows)
        return;
    float ga[VPT], be[VPT];
    RawRow<T, VPT> o0, u0, o1, u1;  // this token's and the next one's rows
    raw_load<T, VPT>(O + row * ldo + lane * VPT, o0);
    raw_load<T, VPT>(U + row * ldu + lane * VPT, u0);
    if (row + nwarps < Trows) {
        raw_load<T, VPT>(O + (row + nwarps) * ldo + lane * VPT, o1);
        raw_load<T, VPT>(U + (row + nwarps) * ldu + lane * VPT, u1);
    }
    load_vec<float, VPT>(gamma + lane * VPT, ga);
    load_vec<float, VPT>(beta + lane * VPT, be);
    for (; row < Trows; row += nwarps) {
        float x[VPT], u[VPT];
        raw_unpack<T, VPT>(o0, x);
        raw_unpack<T, VPT>(u0, u);
        o0 = o1;
        u0 = u1;
        const int64_t r2 = row + 2 * nwarps;  // the token after next
        if (r2 < Trows) {
            raw_load<T, VPT>(O + r2 * ldo + lane * VPT, o1);
            raw_load<T, VPT>(U + r2 * ldu + lane * VPT, u1);
        }
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < VPT; e++)
            sum += x[e];
#pragma unroll
        for (int off = 16; off; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float mean = sum * (1.0f / F);
        float var = 0.f;
#pragma unroll
        for (int e = 0; e < VPT; e++) {
            const float d = x[e] - mean;
            var += d * d;
        }
#pragma unroll
        for (int off = 16; off; off >>= 1)
            var += __shfl_xor_sync(0xffffffffu, var, off);
        const float rstd = rsqrtf(var * (1.0f / F) + eps);
#pragma unroll
        for (int e = 0; e < VPT; e++)
            x[e] = ((x[e] - mean) * rstd * ga[e] + be[e]) * u[e];
        store_vec<T, VPT>(G + row * ldg + lane * VPT, x);
    }
}

// The same for rows narrower than 16 bytes per lane (bf16 F <= 128, fp32 F = 64):
// the next token's O and U are loaded as floats before this token is reduced.
template <typename T, int VPT>
__global__ void __launch_bounds__(256)
norm_gate_narrow_kernel(const T *__restrict__ O, int64_t ldo, const T *__restrict__ U, int64_t ldu,
                 const float *__restrict__ gamma, const float *__restrict__ beta, float eps,
                 T *__restrict__ G, int64_t ldg, int64_t Trows)
{
    constexpr int F = 32 * VPT;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (row >= Trows)
        return;
    float ga[VPT], be[VPT], x[VPT], u[VPT];
    load_vec<T, VPT>(O + row * ldo + lane * VPT, x);
    load_vec<T, VPT>(U + row * ldu + lane * VPT, u);
    load_vec<float, VPT>(gamma + lane * VPT, ga);
    load_vec<float, VPT>(beta + lane * VPT, be);
    for (; row < Trows; row += nwarps) {
        const int64_t nrow = row + nwarps;
        float xn[VPT], un[VPT];
        if (nrow < Trows) {
            load_vec<T, VPT>(O + nrow * ldo + lane * VPT, xn);
            load_vec<T, VPT>(U + nrow * ldu + lane * VPT, un);
        }
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < VPT; e++)
            sum += x[e];
#pragma unroll
        for (int off = 16; off; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float mean = sum * (1.0f / F);
        float var = 0.f;
#pragma unroll
        for (int e = 0; e < VPT; e++) {
            const float d = x[e] - mean;
            var += d * d;
        }
#pragma unroll
        for (int off = 16; off; off >>= 1)
            var += __shfl_xor_sync(0xffffffffu, var, off);
        const float rstd = rsqrtf(var * (1.0f / F) + eps);
        float y[VPT];
#pragma unroll
        for (int e = 0; e < VPT; e++)
            y[e] = ((x[e] - mean) * rstd * ga[e] + be[e]) * u[e];
        store_vec<T, VPT>(G + row * ldg + lane * VPT, y);
        if (nrow < Trows) {
#pragma unroll
            for (int e = 0; e < VPT; e++) {
                x[e] = xn[e];
                u[e] = un[e];
            }
        }
    }
}

template <typename T>
cudaError_t norm_gate_t(const T *O, int64_t ldo, const T *U, int64_t ldu, const float *gamma,
                        const float *beta, float eps, T *G, int64_t ldg, int64_t Trows, int F,
                        cudaStream_t stream)
{
    // two resident blocks per SM, each warp walking a strided set of tokens
    const int64_t want = (Trows * 32 + 255) / 256;
    const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)device_info().sms * 2));
    switch (F) {
    case 64: norm_gate_narrow_kernel<T, 2><<<blocks, 256, 0, stream>>>(O, ldo, U, ldu, gamma, beta, eps, G, ldg, Trows); break;
    case 128:
        if constexpr (sizeof(T) == 2)
            norm_gate_narrow_kernel<T, 4><<<blocks, 256, 0, stream>>>(O, ldo, U, ldu, gamma, beta, eps, G, ldg, Trows);
        else
            norm_gate_kernel<T, 4><<<blocks, 256, 0, stream>>>(O, ldo, U, ldu, gamma, beta, eps, G, ldg, Trows);
        break;
    case 256: norm_gate_kernel<T, 8><<<blocks, 256, 0, stream>>>(O, ldo, U, ldu, gamma, beta, eps, G, ldg, Trows); break;
    case 512: norm_gate_kernel<T, 16><<<blocks, 256, 0, stream>>>(O, ldo, U, ldu, gamma, beta, eps, G, ldg, Trows); break;
    case 1024: norm_gate_kernel<T, 32><<<blocks, 256, 0, stream>>>(O, ldo, U, ldu, gamma, beta, eps, G, ldg, Trows); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// Backward of G = LayerNorm(O) * U, per token over F features (the gate of
// the "HSTU Architecture" section): with xh = (x - mean) rstd, ln = xh g + b,
// dy = dG U:  dU = dG ln,  dO = rstd (dy g - mean(dy g) - xh mean(dy g xh)),
// dgamma += dy xh, dbeta += dy.  One warp per token (grid-stride over tokens),
// two passes over the token's row (the second re-reads it from L1) so few
// values stay live; each lane keeps its features' parameter gradients in
// registers across tokens, each warp stores them once to its shared-memory
// slot, and each block adds the sum of its slots to the outputs.
template <typename T, int VPT>
__global__ void __launch_bounds__(256)
norm_gate_bwd_kernel(const T *__restrict__ dG, int64_t ldd, const T *__restrict__ O, int64_t ldo,
                     const T *__restrict__ U, int64_t ldu, const float *__restrict__ gamma,
                     const float *__restrict__ beta, float eps, T *__restrict__ dO, int64_t lddo,
                     T *__restrict__ dU, int64_t lddu, float *__restrict__ dgamma, float *__restrict__ dbeta,
                     int64_t Trows, int cat)
{
    constexpr int F = 32 * VPT;
    extern __shared__ float slots[];  // [warps][2][F]
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    float *sg = slots + wid * 2 * F, *sb = sg + F;
    float pg[VPT], pb[VPT];
#pragma unroll
    for (int e = 0; e < VPT; e++) {
        pg[e] = 0.f;
        pb[e] = 0.f;
    }
    const int64_t warps = (int64_t)gridDim.x * nw;
    for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < Trows; row += warps) {
        const int64_t fo = lane * VPT;
        float x[VPT];
        load_vec<T, VPT>(O + row * ldo + fo, x);
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < VPT; e++)
            sum += x[e];
#pragma unroll
        for (int off = 16; off; off >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float mean = sum * (1.0f / F);
        float var = 0.f;
#pragma unroll
        for (int e = 0; e < VPT; e++) {
            x[e] -= mean;
            var += x[e] * x[e];
        }
#pragma unroll
        for (int off = 16; off; off >>= 1)
            var += __shfl_xor_sync(0xffffffffu, var, off);
        const float rstd = rsqrtf(var * (1.0f / F) + eps);
        // pass 1: the two row means of the LayerNorm backward, parameter gradients
        float s1 = 0.f, s2 = 0.f;
        {
            float u[VPT], dg[VPT], ga[VPT];
            load_vec<T, VPT>(U + row * ldu + fo, u);
            load_vec<T, VPT>(dG + row * ldd + fo, dg);
            load_vec<float, VPT>(gamma + fo, ga);
#pragma unroll
            for (int e = 0; e < VPT; e++) {
                const float xh = x[e] * rstd, dy = dg[e] * u[e];
                pg[e] = fmaf(dy, xh, pg[e]);
                pb[e] += dy;
                s1 = fmaf(dy, ga[e], s1);
                s2 = fmaf(dy * ga[e], xh, s2);
            }
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            s1 += __shfl_xor_sync(0xffffffffu, s1, off);
            s2 += __shfl_xor_sync(0xffffffffu, s2, off);
        }
        const float m1 = s1 * (1.0f / F), m2 = s2 * (1.0f / F);
        // pass 2: dO and dU
        {
            float u[VPT], dg[VPT], ga[VPT], be[VPT], dx[VPT], du[VPT];
            load_vec<T, VPT>(U + row * ldu + fo, u);
            load_vec<T, VPT>(dG + row * ldd + fo, dg);
            load_vec<float, VPT>(gamma + fo, ga);
            load_vec<float, VPT>(beta + fo, be);
#pragma unroll
            for (int e = 0; e < VPT; e++) {
                const float xh = x[e] * rstd;
                du[e] = dg[e] * fmaf(xh, ga[e], be[e]);
                dx[e] = rstd * (dg[e] * u[e] * ga[e] - m1 - xh * m2);
            }
            if (cat) {
                // output projection over [U | O | G]: dG is the last block of a
                // row whose first two blocks are the direct gradients of U and O
                float cu[VPT], co[VPT];
                load_vec<T, VPT>(dG + row * ldd - 2 * F + fo, cu);
                load_vec<T, VPT>(dG + row * ldd - F + fo, co);
#pragma unroll
                for (int e = 0; e < VPT; e++) {
                    du[e] += cu[e];
                    dx[e] += co[e];
                }
            }
            store_vec<T, VPT>(dO + row * lddo + fo, dx);
            store_vec<T, VPT>(dU + row * lddu + fo, du);
        }
    }
#pragma unroll
    for (int e = 0; e < VPT; e++) {
        sg[lane * VPT + e] = pg[e];
        sb[lane * VPT + e] = pb[e];
    }
    __syncthreads();
    for (int f = threadIdx.x; f < F; f += blockDim.x) {
        float a = 0.f, b = 0.f;
        for (int w = 0; w < nw; w++) {
            a += slots[w * 2 * F + f];
            b += slots[w * 2 * F + F + f];
        }
        atomicAdd(dgamma + f, a);
        atomicAdd(dbeta + f, b);
    }
}

template <typename T>
cudaError_t norm_gate_bwd_t(const T *dG, int64_t ldd, const T *O, int64_t ldo, const T *U, int64_t ldu,
                            const float *gamma, const float *beta, float eps, T *dO, int64_t lddo, T *dU,
                            int64_t lddu, float *dgamma, float *dbeta, int64_t Trows, int F, int cat,
                            cudaStream_t stream)
{
    const int64_t want = (Trows * 32 + 255) / 256;
    const unsigned blocks = (unsigned)std::min<int64_t>(want, (int64_t)device_info().sms * 8);
    const size_t smem = (size_t)8 * 2 * F * sizeof(float);  // 8 warps x (dgamma, dbeta) slots
    if (smem > 48 * 1024) {
        cudaError_t e = cudaErrorInvalidValue;
        switch (F) {
        case 1024: e = cudaFuncSetAttribute(norm_gate_bwd_kernel<T, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)smem); break;
        default: break;
        }
        if (e != cudaSuccess)
            return e;
    }
#define HSTU_NGB(V)                                                                                                 \
    norm_gate_bwd_kernel<T, V><<<blocks, 256, smem, stream>>>(dG, ldd, O, ldo, U, ldu, gamma, beta, eps, dO, lddo, \
                                                              dU, lddu, dgamma, dbeta, Trows, cat)
    switch (F) {
    case 64: HSTU_NGB(2); break;
    case 128: HSTU_NGB(4); break;
    case 256: HSTU_NGB(8); break;
    case 512: HSTU_NGB(16); break;
    case 1024: HSTU_NGB(32); break;
    default: return cudaErrorInvalidValue;
    }
#undef HSTU_NGB
    return cudaGetLastError();
}

// out[n] += sum over rows of A[row, n] (bf16 rows of N columns, fp32 sums): each
// block sums 256 columns over a chunk of rows, one atomic per column.
__global__ void __launch_bounds__(256)
colsum_bf16_kernel(const __nv_bfloat16 *__restrict__ A, int64_t lda, int64_t Trows, int N, int64_t chunk,
                   float *__restrict__ out)
{
    const int n = blockIdx.x * 256 + threadIdx.x;
    if (n >= N)
        return;
    const int64_t r0 = (int64_t)blockIdx.y * chunk, r1 = r0 + chunk < Trows ? r0 + chunk : Trows;
    float acc = 0.f;
    for (int64_t r = r0; r < r1; r++)
        acc += __bfloat162float(A[r * lda + n]);
    atomicAdd(out + n, acc);
}

}  // namespace

cudaError_t launch_gemm_f32(const float *A, int64_t lda, const float *Bm, const float *bias,
                            float *C, int64_t ldc, int64_t M, int N, int K, bool silu,
                            cudaStream_t stream)
{
    if (M == 0)
        return cudaSuccess;
    dim3 grid((N + FT - 1) / FT, (unsigned)((M + FT - 1) / FT));
    gemm_f32_kernel<<<grid, 256, 0, stream>>>(A, lda, Bm, bias, C, ldc, M, N, K, silu);
    return cudaGetLastError();
}

cudaError_t launch_norm_gate_bwd(const void *dG, int64_t ldd, const void *O, int64_t ldo, const void *U,
                                 int64_t ldu, const float *gamma, const float *beta, float eps, void *dO,
                                 int64_t lddo, void *dU, int64_t lddu, float *dgamma, float *dbeta, int64_t T,
                                 int F, bool cat, cudaStream_t stream)
{
    if (T == 0)
        return cudaSuccess;
    return norm_gate_bwd_t(static_cast<const __nv_bfloat16 *>(dG), ldd, static_cast<const __nv_bfloat16 *>(O), ldo,
                           static_cast<const __nv_bfloat16 *>(U), ldu, gamma, beta, eps,
                           static_cast<__nv_bfloat16 *>(dO), lddo, static_cast<__nv_bfloat16 *>(dU), lddu, dgamma,
                           dbeta, T, F, cat ? 1 : 0, stream);
}

// out[t] = [a[t] | b[t] | c[t]], each `bytes` wide (a multiple of 4), rows strided
__global__ void __launch_bounds__(256)
concat3_kernel(const unsigned char *__restrict__ a, int64_t lda, const unsigned char *__restrict__ b, int64_t ldb,
               const unsigned char *__restrict__ c, int64_t ldc, unsigned char *__restrict__ out, int64_t Trows,
               int64_t bytes)
{
    const int64_t words = bytes >> 2, total = Trows * 3 * words;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = e / (3 * words), r = e - row * 3 * words, blk = r / words, w = r - blk * words;
        const unsigned char *src = blk == 0 ? a + row * lda : blk == 1 ? b + row * ldb : c + row * ldc;
        reinterpret_cast<uint32_t *>(out + row * 3 * bytes)[blk * words + w] = reinterpret_cast<const uint32_t *>(src)[w];
    }
}

cudaError_t launch_concat3(const void *a, int64_t lda, const void *b, int64_t ldb, const void *c, int64_t ldc,
                           void *out, int64_t T, int64_t bytes, cudaStream_t stream)
{
    if (T == 0)
        return cudaSuccess;
    const int64_t total = T * 3 * (bytes / 4);
    const unsigned blocks = (unsigned)std::min<int64_t>((total + 255) / 256, (int64_t)device_info().sms * 8);
    concat3_kernel<<<blocks, 256, 0, stream>>>(static_cast<const unsigned char *>(a), lda,
                                               static_cast<const unsigned char *>(b), ldb,
                                               static_cast<const unsigned char *>(c), ldc,
                                               static_cast<unsigned char *>(out), T, bytes);
    return cudaGetLastError();
}

cudaError_t launch_colsum_bf16(const void *A, int64_t lda, int64_t T, int N, float *out, cudaStream_t stream)
{
    if (T == 0 || N == 0)
        return cudaSuccess;
    const int64_t chunks = std::min<int64_t>((T + 127) / 128, 256);
    const int64_t chunk = (T + chunks - 1) / chunks;
    dim3 grid((N + 255) / 256, (unsigned)((T + chunk - 1) / chunk));
    colsum_bf16_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(A), lda, T, N, chunk, out);
    return cudaGetLastError();
}

cudaError_t launch_norm_gate(bool bf16, const void *O, int64_t ldo, const void *U, int64_t ldu,
                             const float *gamma, const float *beta, float eps, void *G,
                             int64_t ldg, int64_t T, int F, cudaStream_t stream)
{
    if (T == 0)
        return cudaSuccess;
    if (bf16)
        return norm_gate_t(static_cast<const __nv_bfloat16 *>(O), ldo, static_cast<const __nv_bfloat16 *>(U),
                           ldu, gamma, beta, eps, static_cast<__nv_bfloat16 *>(G), ldg, T, F, stream);
    return norm_gate_t(static_cast<const float *>(O), ldo, static_cast<const float *>(U), ldu, gamma,
                       beta, eps, static_cast<float *>(G), ldg, T, F, stream);
}

}  // namespace hstu
