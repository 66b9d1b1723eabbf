// Projection GEMMs of the transduction layer on sm_100a: TMA + tcgen05 (TMEM).
//
//   C[M, N] = act(A[M, K] B[K, N] + bias[N]),  act = SiLU for f1, identity for f2
//
// ("DLRMv4 Brings Sequence-Based Recommendation Training to MLPerf", section
// "Model Architecture": the projection that produces U, V, Q, K, and the output
// projection after the gate.)  Persistent tiles of 128 x BN (BN = 256 or
// 128): warp 0 streams A (K-major, 128 rows x 64 columns) and B (the weight,
// row-major so N-contiguous: an MN-major operand, 64 K-rows x 64 columns per
// box) through a 4-stage ring; warp 1 owns two TMEM accumulators and issues
// tcgen05.mma from one thread; warps 2-9 read one accumulator row by row, add
// the bias, apply SiLU and store bf16 while the next tile accumulates in the
// other.  Bias and activation never make a separate pass over HBM.
#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace hstu {

namespace {

constexpr int GBM = 128, GBK = 64, GSTAGES = 4;
constexpr int kEpiWarpsG = 8;  // two per TMEM lane quarter, each half of the columns
constexpr int kThreadsG = 64 + 32 * kEpiWarpsG;
constexpr int kRegA = GBM * 128;  // 128 rows x 128 B
constexpr int kRegB = GBK * 128;  // 64 K-rows x 128 B (64 N columns)

template <int BN>
struct GL {
    static constexpr int A = 0;
    static constexpr int B = A + GSTAGES * kRegA;
    static constexpr int BAR = B + GSTAGES * (BN / 64) * kRegB;
    static constexpr int NBAR = 2 * GSTAGES + 4;  // full, empty, acc_full[2], acc_empty[2]
    static constexpr int MISC = BAR + NBAR * 8;
    static constexpr int BYTES = MISC + 64;
};

// Persistent: CTA c computes output tiles c, c + gridDim.x, ... (row-block
// major, so consecutive tiles reuse the same A rows from L2).  The TMA ring
// runs across tile boundaries and the accumulator is double-buffered in
// TMEM, so the epilogue of one tile overlaps the MMAs of the next.
template <int BN>
__global__ void __launch_bounds__(kThreadsG, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __nv_bfloat16 *__restrict__ bias, __nv_bfloat16 *__restrict__ C, int64_t ldc, int64_t M,
               int N, int K, int silu, WsHeader *hdr)
{
    using LY = GL<BN>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / GBK;
    const int tiles_n = N / BN;
    const int tiles = (int)((M + GBM - 1) / GBM) * tiles_n;
    auto full_bar = [&](int s) { return base + LY::BAR + 8u * s; };
    auto empty_bar = [&](int s) { return base + LY::BAR + 8u * (GSTAGES + s); };
    auto accf_bar = [&](int b) { return base + LY::BAR + 8u * (2 * GSTAGES + b); };
    auto acce_bar = [&](int b) { return base + LY::BAR + 8u * (2 * GSTAGES + 2 + b); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + LY::MISC + 8);

    if (threadIdx.x == 0) {
        for (int i = 0; i < LY::NBAR; i++)
            mbar_init(base + LY::BAR + 8u * i, i >= 2 * GSTAGES + 2 ? kEpiWarpsG : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmA);
        tma_prefetch(&tmB);
    }
    if (warp == 1)
        tmem_alloc(base + LY::MISC, 2 * BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + LY::MISC);

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;  // k-tiles issued by this CTA, across its output tiles
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int m0 = (tile / tiles_n) * GBM, n0 = (tile % tiles_n) * BN;
                for (int kt = 0; kt < nk; kt++, it++) {
                    const int s = it % GSTAGES;
                    if (it >= GSTAGES && !(ok = mbar_wait(empty_bar(s), ((it / GSTAGES) - 1) & 1, abort_flag, hdr)))
                        break;
                    mbar_expect_tx(full_bar(s), kRegA + (BN / 64) * kRegB);
                    tma_load_2d(base + LY::A + s * kRegA, &tmA, kt * GBK, m0, full_bar(s));
                    for (int r = 0; r < BN / 64; r++)
                        tma_load_2d(base + LY::B + (s * (BN / 64) + r) * kRegB, &tmB, n0 + 64 * r, kt * GBK,
                                    full_bar(s));
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(GBM, BN, 0, 1);
            int it = 0, lt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, lt++) {
                const int ab = lt & 1;
                // the epilogue must have drained this accumulator (tile lt - 2)
                if (lt >= 2 && !(ok = mbar_wait(acce_bar(ab), ((lt >> 1) - 1) & 1, abort_flag, hdr)))
                    break;
                tc_fence_after();
                for (int kt = 0; kt < nk; kt++, it++) {
                    const int s = it % GSTAGES;
                    if (!(ok = mbar_wait(full_bar(s), (it / GSTAGES) & 1, abort_flag, hdr)))
                        break;
                    tc_fence_after();
                    for (int ks = 0; ks < GBK / 16; ks++) {
                        const uint64_t a = smem_desc_sw128(base + LY::A + s * kRegA + ks * 32, 16, 1024);
                        const uint64_t b =
                            smem_desc_sw128(base + LY::B + s * (BN / 64) * kRegB + ks * 2048, kRegB, 1024);
                        umma_bf16(tmem + ab * BN, a, b, idesc, (kt > 0 || ks > 0));
                    }
                    umma_commit(empty_bar(s));
                }
                umma_commit(accf_bar(ab));
            }
        }
    } else {
        const int ew = warp - 2, half = ew >> 2, quarter = warp & 3;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        constexpr int CW = BN / 2;  // columns per epilogue thread
        int lt = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, lt++) {
            const int ab = lt & 1;
            if (!mbar_wait(accf_bar(ab), (lt >> 1) & 1, abort_flag, hdr))
                break;
            tc_fence_after();
            const int64_t row = (int64_t)(tile / tiles_n) * GBM + quarter * 32 + lane;
            const int n0 = (tile % tiles_n) * BN + half * CW;
            __nv_bfloat16 *crow = C + row * ldc + n0;
#pragma unroll 1
            for (int cc = 0; cc < CW; cc += 32) {
                float v[32];
                tmem_ld32(trow + ab * BN + half * CW + cc, v);
                tmem_wait_ld();
                if (row < M) {
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) {
                            x[e] = v[8 * u + e] + (bias ? __bfloat162float(bias[n0 + cc + 8 * u + e]) : 0.f);
                            if (silu)
                                x[e] = silu_fast(x[e]);
                        }
                        uint4 w;
                        w.x = pack_bf16(x[0], x[1]);
                        w.y = pack_bf16(x[2], x[3]);
                        w.z = pack_bf16(x[4], x[5]);
                        w.w = pack_bf16(x[6], x[7]);
                        *reinterpret_cast<uint4 *>(crow + cc + 8 * u) = w;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(acce_bar(ab));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, 2 * BN);
}

int num_sms()
{
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    }
    return n;
}

template <int BN>
cudaError_t gemm_tc_launch(const void *A, int64_t lda, const void *Bm, const void *bias, void *C, int64_t ldc,
                           int64_t M, int N, int K, bool silu, WsHeader *hdr, cudaStream_t stream)
{
    CUtensorMap ma, mb;
    cudaError_t e = make_tensor_map_2d(&ma, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, M, K, lda * 2, 64, GBM,
                                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_tensor_map_2d(&mb, Bm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, N, (int64_t)N * 2, 64, GBK,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess)
        return e;
    const size_t bytes = GL<BN>::BYTES + 1024;
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess)
        return e;
    const int64_t tiles = ((M + GBM - 1) / GBM) * (N / BN);
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, num_sms());
    gemm_tc_kernel<BN><<<grid, kThreadsG, bytes, stream>>>(ma, mb, static_cast<const __nv_bfloat16 *>(bias),
                                                          static_cast<__nv_bfloat16 *>(C), ldc, M, N, K, silu, hdr);
    return cudaGetLastError();
}

}  // namespace

bool gemm_tc_supported(const void *A, int64_t lda, const void *Bm, void *C, int64_t ldc, int64_t M, int N, int K)
{
    const bool aligned = ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(Bm) |
                           reinterpret_cast<uintptr_t>(C)) & 15u) == 0;
    return aligned && M > 0 && M < ((int64_t)1 << 31) - GBM && K % GBK == 0 && K > 0 && N % 128 == 0 &&
           lda % 8 == 0 && ldc % 8 == 0;
}

cudaError_t launch_gemm_tc(const void *A, int64_t lda, const void *Bm, const void *bias, void *C, int64_t ldc,
                           int64_t M, int N, int K, bool silu, WsHeader *hdr, cudaStream_t stream)
{
    if (M == 0)
        return cudaSuccess;
    if (N % 256 == 0)
        return gemm_tc_launch<256>(A, lda, Bm, bias, C, ldc, M, N, K, silu, hdr, stream);
    return gemm_tc_launch<128>(A, lda, Bm, bias, C, ldc, M, N, K, silu, hdr, stream);
}

}  // namespace hstu
