// Attention truncation on jagged batches (the ULTRA-HSTU review in the pages:
// N layers over the whole history, then M layers over its most recent segment).
// Because candidates sit at the end of each sequence, the kept tokens of a
// sequence are its last min(hist, keep) + n_t rows: the new batch is a gather
// of every sequence's tail.  One kernel: every block scans the kept counts
// into shared memory, then copies rows in 16-byte chunks; each output row finds
// its sequence by binary search in the new offsets.
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace hstu {

namespace {

// kept tokens of sequence b, with the offsets and targets clamped into [0, T]
// so that malformed sequence data never reads outside the input
__device__ __forceinline__ int64_t kept_rows(const int64_t *off, const int32_t *nt, int b, int64_t T, int keep,
                                             int64_t *src_begin)
{
    int64_t s0 = min(max(off[b], (int64_t)0), T), s1 = min(max(off[b + 1], (int64_t)0), T);
    const int64_t L = max(s1 - s0, (int64_t)0);
    const int64_t n_t = nt ? min(max((int64_t)nt[b], (int64_t)0), L) : 0;
    const int64_t kept = min(L - n_t, (int64_t)keep) + n_t;
    *src_begin = s0 + L - kept;
    return kept;
}

// inclusive sum over the block's 256 threads (8 warps)
__device__ __forceinline__ int64_t block_inclusive_scan(int64_t v, int64_t *warp_tot, int64_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d)
            v += y;
    }
    if (lane == 31)
        warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int64_t t = lane < 8 ? warp_tot[lane] : 0;
#pragma unroll
        for (int d = 1; d < 8; d <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, t, d);
            if (lane >= d)
                t += y;
        }
        if (lane < 8)
            warp_tot[lane] = t;
    }
    __syncthreads();
    if (warp > 0)
        v += warp_tot[warp - 1];
    *total = warp_tot[7];
    __syncthreads();  // warp_tot is reused by the next chunk
    return v;
}

// Every block scans the kept counts into shared memory (the batch's B+1 new
// offsets and B source starts), block 0 also writes the offsets out, then the
// blocks copy the kept rows: 16-byte (or 4-byte) chunks, grid-stride, four
// loads in flight per thread before their stores.
template <bool VEC>
__global__ void __launch_bounds__(256)
truncate_kernel(const int64_t *__restrict__ off, const int32_t *__restrict__ nt, int B, int64_t T, int keep,
                const unsigned char *__restrict__ in, unsigned char *__restrict__ out, int64_t row_bytes,
                int64_t *__restrict__ out_off)
{
    extern __shared__ int64_t smem[];
    int64_t *s_off = smem;            // [B + 1]
    int64_t *s_src = smem + B + 1;    // [B]
    __shared__ int64_t warp_tot[8];
    int64_t carry = 0;
    for (int c0 = 0; c0 < B; c0 += 256) {
        const int b = c0 + threadIdx.x;
        int64_t src = 0;
        const int64_t v = b < B ? kept_rows(off, nt, b, T, keep, &src) : 0;
        int64_t tot;
        const int64_t inc = block_inclusive_scan(v, warp_tot, &tot);
        if (b < B) {
            s_off[b + 1] = carry + inc;
            s_src[b] = src;
        }
        carry += tot;
    }
    if (threadIdx.x == 0)
        s_off[0] = 0;
    __syncthreads();
    if (blockIdx.x == 0)
        for (int b = threadIdx.x; b <= B; b += blockDim.x)
            out_off[b] = s_off[b];
    // sequences that break the jagged rules can overlap; `out` holds T rows
    const int64_t Tout = min(s_off[B], T);
    using Chunk = typename std::conditional<VEC, uint4, uint32_t>::type;
    const int64_t chunks = row_bytes / (int64_t)sizeof(Chunk);
    const int64_t total = Tout * chunks;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    constexpr int U = 4;
    for (int64_t e0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e0 < total; e0 += U * stride) {
        int64_t dst[U], srcb[U];
        Chunk val[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t e = e0 + u * stride;
            dst[u] = -1;
            if (e < total) {
                const int64_t r = e / chunks, c = e - r * chunks;
                // sequence of output row r: the last b with s_off[b] <= r
                int lo = 0, hi = B - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s_off[mid] <= r)
                        lo = mid;
                    else
                        hi = mid - 1;
                }
                const int64_t src = s_src[lo] + (r - s_off[lo]);
                dst[u] = r * chunks + c;
                srcb[u] = src * chunks + c;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (dst[u] >= 0)
                val[u] = reinterpret_cast<const Chunk *>(in)[srcb[u]];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (dst[u] >= 0)
                reinterpret_cast<Chunk *>(out)[dst[u]] = val[u];
    }
}

}  // namespace

cudaError_t launch_jagged_truncate(const int64_t *off, const int32_t *nt, int B, int64_t T, int keep,
                                   int64_t row_bytes, const void *in, void *out, int64_t *out_off,
                                   cudaStream_t stream)
{
    const size_t smem = (size_t)(2 * B + 1) * sizeof(int64_t);
    if (B > kTruncateMaxSeqs)
        return cudaErrorInvalidValue;
    const bool vec = (row_bytes & 15) == 0;
    auto kern = vec ? truncate_kernel<true> : truncate_kernel<false>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    const int64_t chunks = std::max<int64_t>(1, T * (vec ? row_bytes / 16 : row_bytes / 4));
    // about four chunks per thread; at most 4 blocks of 256 threads per SM
    const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>((chunks + 1023) / 1024, (int64_t)device_info().sms * 4));
    kern<<<blocks, 256, smem, stream>>>(off, nt, B, T, keep, static_cast<const unsigned char *>(in),
                                        static_cast<unsigned char *>(out), row_bytes, out_off);
    return cudaGetLastError();
}

}  // namespace hstu
