// Projection GEMMs of the transduction layer on sm_100a: TMA + tcgen05 (TMEM).
//
//   C[M, N] = epi(A[M, K] B[K, N])
//
// ("DLRMv4 Brings Sequence-Based Recommendation Training to MLPerf", section
// "Model Architecture": the projection that produces U, V, Q, K, and the output
// projection after the gate; their gradients for the layer backward.)
// Persistent tiles of 128 x BN (BN = 256 when it divides N, else 128 with a
// partial last column tile; N a multiple of 32): warp 0 streams A and B
// through a 4-stage ring of 64-deep k-slices; warp 1 owns two TMEM
// accumulators and issues tcgen05.mma from one thread; warps 2-9 read one
// accumulator row by row while the next tile accumulates in the other.
//
// Operand layouts (bf16, 128-byte swizzled k-slices of 64 elements):
//   A K-major: A[m][k] row-major ([M, K]);  A MN-major: stored as X[k][m] ([K, M])
//   B MN-major: B[k][n] row-major ([K, N]); B K-major: stored as W[n][k] ([N, K])
// so that the layer backward's products dY W2^T, dZ W1^T (B K-major) and
// G^T dY, X^T dZ (A MN-major, K = tokens) need no transposed copies.  A may be
// three stored matrices concatenated along their columns (the output
// projection over [U | O | G]).  The E4M3 instantiation (F8) takes K-major A
// and B codes in slices of 128 and kind::f8f6f4 MMAs of K = 32.
// Epilogues (the chunk's bias, scales and dSiLU factors are fetched while its
// TMEM load is in flight; bf16 outputs leave through 32 x 32 swizzled boxes,
// two per warp used in turn, and TMA stores):
//   EPI_ACT    bf16 out = acc (x row scale x column scale for F8) + bias,
//              optionally SiLU as h (1 + tanh h), h = x / 2 (forward projections);
//   EPI_DSILU  bf16 out = aux * SiLU'(acc + bias) (the SiLU backward fused into
//              the recompute of the pre-activation);
//   EPI_RED    fp32 out += acc through a swizzled staging box and a TMA bulk
//              reduce-add; the k range is split across CTAs (weight gradients,
//              whose K is the token count).
#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace hstu {

namespace {

constexpr int GBM = 128, GBK = 64, GSTAGES = 4;
constexpr int kEpiWarpsG = 8;  // two per TMEM lane quarter, each half of the columns
constexpr int kThreadsG = 64 + 32 * kEpiWarpsG;
constexpr int kRegA = GBM * 128;  // 128 rows x 128 B
constexpr int kReg64 = 64 * 128;  // a 64 x 64 bf16 box

enum GemmEpi { EPI_ACT = 0, EPI_DSILU = 1, EPI_RED = 2 };

template <int BN, int EPI>
struct GL {
    static constexpr int A = 0;
    static constexpr int B = A + GSTAGES * kRegA;
    // output staging per epilogue warp, two boxes used in turn (a box is rewritten
    // once the TMA store two boxes back has read it): EPI_RED 4 KB fp32 boxes;
    // otherwise 2 KB bf16 boxes of 32 rows x 32 columns (64-byte swizzle)
    static constexpr int STG = B + GSTAGES * BN * 128;
    static constexpr int BAR = STG + kEpiWarpsG * (EPI == EPI_RED ? 2 * 4096 : 2 * 2048);
    static constexpr int NBAR = 2 * GSTAGES + 4;  // full, empty, acc_full[2], acc_empty[2]
    static constexpr int MISC = BAR + NBAR * 8;
    static constexpr int BYTES = MISC + 64;
};

struct GemmArgs {
    const __nv_bfloat16 *bias;  // [N] or null
    const __nv_bfloat16 *aux;   // EPI_DSILU: [M, N] with row stride ldaux
    int64_t ldaux;
    void *C;                    // bf16 (EPI_ACT, EPI_DSILU) or unused (EPI_RED: through tmC)
    int64_t ldc;
    int64_t M;
    int N, K, silu, splits;
    int a_seg;                  // > 0: A is three stored matrices of a_seg columns each
    const float *sa, *sb;       // E4M3 operands: scale of each row of A and of each column of B
    WsHeader *hdr;
};

// SiLU(z) = h (1 + tanh h), h = z / 2: one MUFU op (tanh.approx, relative error
// about 2^-11, below the bf16 output's rounding)
__device__ __forceinline__ float silu_tanh(float z)
{
    const float h = 0.5f * z;
    return fmaf(h, tanh_approx(h), h);
}

__device__ __forceinline__ float silu_grad_tanh(float z)
{
    // SiLU'(z) = sigma(z) (1 + z (1 - sigma(z))) with sigma(z) = (1 + tanh(z/2)) / 2
    const float h = 0.5f * z, t = tanh_approx(h);
    const float a = 1.f + t;
    return 0.5f * fmaf(a, fmaf(-h, t, h), a);
}

// Persistent: CTA c takes work units c, c + gridDim.x, ...; unit = (tile, k split),
// tiles row-block major so consecutive tiles reuse the same A rows from L2.
template <int BN, bool A_MN, bool B_K, int EPI, bool F8>
__global__ void __launch_bounds__(kThreadsG, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA1,
               const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, const GemmArgs g)
{
    using LY = GL<BN, EPI>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int KE = F8 ? 128 : GBK;     // K elements per 128-byte slice
    const int nk = (g.K + KE - 1) / KE;    // the TMA zero-fills past K
    const int per = (nk + g.splits - 1) / g.splits;  // k-slices per split
    // N a multiple of 32: the last column tile may be partial (its B columns past
    // N load as zeros, its output chunks past N are skipped)
    const int tiles_n = (g.N + BN - 1) / BN;
    const int tiles = (int)((g.M + GBM - 1) / GBM) * tiles_n;
    const int units = tiles * g.splits;
    auto full_bar = [&](int s) { return base + LY::BAR + 8u * s; };
    auto empty_bar = [&](int s) { return base + LY::BAR + 8u * (GSTAGES + s); };
    auto accf_bar = [&](int b) { return base + LY::BAR + 8u * (2 * GSTAGES + b); };
    auto acce_bar = [&](int b) { return base + LY::BAR + 8u * (2 * GSTAGES + 2 + b); };
    auto krange = [&](int u, int &k0, int &k1) {
        const int sp = u % g.splits;
        k0 = sp * per;
        k1 = min(nk, k0 + per);
    };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + LY::MISC + 8);

    if (threadIdx.x == 0) {
        for (int i = 0; i < LY::NBAR; i++)
            mbar_init(base + LY::BAR + 8u * i, i >= 2 * GSTAGES + 2 ? kEpiWarpsG : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmA);
        if (g.a_seg) {
            tma_prefetch(&tmA1);
            tma_prefetch(&tmA2);
        }
        tma_prefetch(&tmB);
        if (EPI == EPI_RED)
            tma_prefetch(&tmC);
    }
    if (warp == 1)
        tmem_alloc(base + LY::MISC, 2 * BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + LY::MISC);

    if (warp == 0) {
        // the stored matrix holding stored column x of A, and x within it
        auto a_map = [&](int x, int &xl) -> const CUtensorMap * {
            if (!g.a_seg) {
                xl = x;
                return &tmA;
            }
            const int seg = min(x / g.a_seg, 2);  // past the end: the last matrix's zero fill
            xl = x - seg * g.a_seg;
            return seg == 0 ? &tmA : seg == 1 ? &tmA1 : &tmA2;
        };
        if (lane == 0) {
            int it = 0;  // k-slices issued by this CTA, across its units
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const int tile = u / g.splits;
                const int m0 = (tile / tiles_n) * GBM, n0 = (tile % tiles_n) * BN;
                int k0, k1;
                krange(u, k0, k1);
                for (int kt = k0; kt < k1; kt++, it++) {
                    const int s = it % GSTAGES;
                    if (it >= GSTAGES && !(ok = mbar_wait(empty_bar(s), ((it / GSTAGES) - 1) & 1, abort_flag, g.hdr)))
                        break;
                    mbar_expect_tx(full_bar(s), kRegA + BN * 128);
                    const uint32_t sa = base + LY::A + s * kRegA, sb = base + LY::B + s * BN * 128;
                    if (A_MN) {
                        for (int r = 0; r < 2; r++) {
                            int xl;
                            const CUtensorMap *ma = a_map(m0 + 64 * r, xl);
                            tma_load_2d(sa + r * kReg64, ma, xl, kt * KE, full_bar(s));
                        }
                    } else {
                        int xl;
                        const CUtensorMap *ma = a_map(kt * KE, xl);
                        tma_load_2d(sa, ma, xl, m0, full_bar(s));
                    }
                    if (B_K) {
                        tma_load_2d(sb, &tmB, kt * KE, n0, full_bar(s));
                    } else {
                        for (int r = 0; r < BN / 64; r++)
                            tma_load_2d(sb + r * kReg64, &tmB, n0 + 64 * r, kt * KE, full_bar(s));
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc =
                F8 ? idesc_e4m3(GBM, BN, A_MN ? 1 : 0, B_K ? 0 : 1) : idesc_bf16(GBM, BN, A_MN ? 1 : 0, B_K ? 0 : 1);
            int it = 0, lt = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, lt++) {
                const int ab = lt & 1;
                int k0, k1;
                krange(u, k0, k1);
                // the epilogue must have drained this accumulator (unit lt - 2)
                if (lt >= 2 && !(ok = mbar_wait(acce_bar(ab), ((lt >> 1) - 1) & 1, abort_flag, g.hdr)))
                    break;
                tc_fence_after();
                for (int kt = k0; kt < k1; kt++, it++) {
                    const int s = it % GSTAGES;
                    if (!(ok = mbar_wait(full_bar(s), (it / GSTAGES) & 1, abort_flag, g.hdr)))
                        break;
                    tc_fence_after();
                    // four 32-byte k-steps per slice: K = 16 bf16 or K = 32 E4M3 each
                    for (int ks = 0; ks < 4; ks++) {
                        const uint32_t sa = base + LY::A + s * kRegA, sb = base + LY::B + s * BN * 128;
                        const uint64_t a = A_MN ? smem_desc_sw128(sa + ks * 2048, kReg64, 1024)
                                                : smem_desc_sw128(sa + ks * 32, 16, 1024);
                        const uint64_t b = B_K ? smem_desc_sw128(sb + ks * 32, 16, 1024)
                                               : smem_desc_sw128(sb + ks * 2048, kReg64, 1024);
                        if (F8)
                            umma_e4m3(tmem + ab * BN, a, b, idesc, (kt > k0 || ks > 0));
                        else
                            umma_bf16(tmem + ab * BN, a, b, idesc, (kt > k0 || ks > 0));
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
        int lt = 0, nstage = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, lt++) {
            const int ab = lt & 1;
            const int tile = u / g.splits;
            int k0, k1;
            krange(u, k0, k1);
            if (!mbar_wait(accf_bar(ab), (lt >> 1) & 1, abort_flag, g.hdr))
                break;
            tc_fence_after();
            const int64_t rowbase = (int64_t)(tile / tiles_n) * GBM + quarter * 32;
            const int64_t row = rowbase + lane;
            const int n0 = (tile % tiles_n) * BN + half * CW;
#pragma unroll 1
            for (int cc = 0; cc < CW && n0 + cc < g.N; cc += 32) {
                float v[32];
                tmem_ld32(trow + ab * BN + half * CW + cc, v);
                if (EPI == EPI_RED) {
                    tmem_wait_ld();
                    // [32 rows x 32 columns] fp32 box, 128-byte swizzled, two buffers per warp
                    if (k1 <= k0)
                        continue;  // an empty split adds nothing
                    const int bsel = nstage & 1;
                    unsigned char *stg = sm + LY::STG + (ew * 2 + bsel) * 4096;
                    if (lane == 0 && nstage >= 2)
                        bulk_wait_read1();  // the box written two stages ago has been read
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; c++)
                        *reinterpret_cast<float4 *>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                            make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_reduce_add_2d(&tmC, n0 + cc, (int)rowbase, smem_u32(stg));
                        bulk_commit();
                    }
                    nstage++;
                    continue;
                }
                // the chunk's bias (and E4M3 column scales, and the dSiLU factor row)
                // are fetched while the TMEM load is in flight
                const bool live = row < g.M;
                uint4 bw[4], aw[4];
                float4 sc[8];
                const bool bias_vec = (reinterpret_cast<uintptr_t>(g.bias) & 15u) == 0;
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    if (!g.bias) {
                        bw[u] = make_uint4(0, 0, 0, 0);
                    } else if (bias_vec) {
                        bw[u] = reinterpret_cast<const uint4 *>(g.bias + n0 + cc)[u];
                    } else {
                        const unsigned short *b16 = reinterpret_cast<const unsigned short *>(g.bias + n0 + cc + 8 * u);
                        bw[u] = make_uint4(b16[0] | ((uint32_t)b16[1] << 16), b16[2] | ((uint32_t)b16[3] << 16),
                                           b16[4] | ((uint32_t)b16[5] << 16), b16[6] | ((uint32_t)b16[7] << 16));
                    }
                    if (EPI == EPI_DSILU)
                        aw[u] = live ? reinterpret_cast<const uint4 *>(g.aux + row * g.ldaux + n0 + cc)[u]
                                     : make_uint4(0, 0, 0, 0);
                }
                if (F8) {
#pragma unroll
                    for (int u = 0; u < 8; u++)
                        sc[u] = reinterpret_cast<const float4 *>(g.sb + n0 + cc)[u];
                }
                const float rs = F8 && live ? g.sa[row] : 1.f;
                tmem_wait_ld();
                uint4 packed[4];
                {
#pragma unroll
                    for (int u4 = 0; u4 < 4; u4++) {
                        const uint32_t bb[4] = {bw[u4].x, bw[u4].y, bw[u4].z, bw[u4].w};
                        const uint32_t ab4[4] = {aw[u4].x, aw[u4].y, aw[u4].z, aw[u4].w};
                        float x[8];
#pragma unroll
                        for (int e = 0; e < 8; e++) {
                            const float bias = __uint_as_float(e & 1 ? bb[e >> 1] & 0xffff0000u : bb[e >> 1] << 16);
                            float acc = v[8 * u4 + e];
                            if (F8) {
                                const float4 s4 = sc[(8 * u4 + e) >> 2];
                                const int q = e & 3;
                                acc *= rs * (q == 0 ? s4.x : q == 1 ? s4.y : q == 2 ? s4.z : s4.w);
                            }
                            x[e] = acc + bias;
                            if (EPI == EPI_DSILU) {
                                const float da = __uint_as_float(e & 1 ? ab4[e >> 1] & 0xffff0000u : ab4[e >> 1] << 16);
                                x[e] = da * silu_grad_tanh(x[e]);
                            } else if (g.silu) {
                                x[e] = silu_tanh(x[e]);
                            }
                        }
                        packed[u4] = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                                                pack_bf16(x[6], x[7]));
                    }
                }
                // this warp's 32 rows x 32 columns through shared memory and one TMA
                // store (coalesced; rows past M are dropped by the tensor map)
                unsigned char *stg = sm + LY::STG + (ew * 2 + (nstage & 1)) * 2048;
                if (lane == 0 && nstage >= 2)
                    bulk_wait_read1();  // the box written two stores ago has been read out
                nstage++;
                __syncwarp();
#pragma unroll
                for (int u4 = 0; u4 < 4; u4++)
                    *reinterpret_cast<uint4 *>(stg + lane * 64 + ((u4 ^ ((lane >> 1) & 3)) << 4)) = packed[u4];
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmC, n0 + cc, (int)rowbase, smem_u32(stg));
                    bulk_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(acce_bar(ab));
        }
        if (lane == 0)
            bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, 2 * BN);
}

template <int BN, bool A_MN, bool B_K, int EPI, bool F8 = false>
cudaError_t gemm_tc_launch(const GemmOperands &op, GemmArgs g, cudaStream_t stream)
{
    CUtensorMap ma, ma1, ma2, mb, mc;
    cudaError_t e = cudaSuccess;
    const void *abase[3] = {op.A, op.A1, op.A2};
    const int64_t ald[3] = {op.lda, op.lda1, op.lda2};
    CUtensorMap *amap[3] = {&ma, &ma1, &ma2};
    for (int i = 0; i < (g.a_seg ? 3 : 1) && e == cudaSuccess; i++) {
        if (F8)    // E4M3 [M, K]: box 128 k x 128 m
            e = make_tensor_map_2d(amap[i], abase[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, g.M, g.K, ald[i], 128, GBM,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
        else if (A_MN)  // stored [K, M]: box 64 m x 64 k
            e = make_tensor_map_2d(amap[i], abase[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.K,
                                   g.a_seg ? g.a_seg : g.M, ald[i] * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
        else       // [M, K]: box 64 k x 128 m
            e = make_tensor_map_2d(amap[i], abase[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.M,
                                   g.a_seg ? g.a_seg : g.K, ald[i] * 2, 64, GBM, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!g.a_seg)
        ma1 = ma2 = ma;  // unused
    if (e == cudaSuccess) {
        if (F8)   // E4M3 stored [N, K]: box 128 k x BN n
            e = make_tensor_map_2d(&mb, op.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.N, g.K, op.ldb, 128, BN,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
        else if (B_K)  // stored [N, K]: box 64 k x BN n
            e = make_tensor_map_2d(&mb, op.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.N, g.K, op.ldb * 2, 64, BN,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
        else      // [K, N]: box 64 n x 64 k
            e = make_tensor_map_2d(&mb, op.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.K, g.N, op.ldb * 2, 64, GBK,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (e == cudaSuccess) {
        if (EPI == EPI_RED)  // fp32 [M, N]: box 32 columns x 32 rows, 128-byte swizzle
            e = make_tensor_map_2d(&mc, op.C32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.M, g.N, g.ldc * 4, 32, 32,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
        else                 // bf16 [M, N]: box 32 columns x 32 rows, 64-byte swizzle
            e = make_tensor_map_2d(&mc, g.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.M, g.N, g.ldc * 2, 32, 32,
                                   CU_TENSOR_MAP_SWIZZLE_64B);
    }
    if (e != cudaSuccess)
        return e;
    const size_t bytes = GL<BN, EPI>::BYTES + 1024;
    e = cudaFuncSetAttribute(gemm_tc_kernel<BN, A_MN, B_K, EPI, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bytes);
    if (e != cudaSuccess)
        return e;
    const int64_t units = ((g.M + GBM - 1) / GBM) * ((g.N + BN - 1) / BN) * g.splits;
    const unsigned grid = (unsigned)std::min<int64_t>(units, device_info().sms);
    gemm_tc_kernel<BN, A_MN, B_K, EPI, F8><<<grid, kThreadsG, bytes, stream>>>(ma, ma1, ma2, mb, mc, g);
    return cudaGetLastError();
}

template <int BN, int EPI>
cudaError_t gemm_dispatch_layout(const GemmOperands &op, const GemmArgs &g, cudaStream_t stream)
{
    if (op.a_mn && op.b_k)
        return gemm_tc_launch<BN, true, true, EPI>(op, g, stream);
    if (op.a_mn)
        return gemm_tc_launch<BN, true, false, EPI>(op, g, stream);
    if (op.b_k)
        return gemm_tc_launch<BN, false, true, EPI>(op, g, stream);
    return gemm_tc_launch<BN, false, false, EPI>(op, g, stream);
}

}  // namespace

bool gemm_tc_ok(const GemmOperands &op, int64_t M, int N, int K)
{
    const bool aligned = ((reinterpret_cast<uintptr_t>(op.A) | reinterpret_cast<uintptr_t>(op.B) |
                           reinterpret_cast<uintptr_t>(op.C) | reinterpret_cast<uintptr_t>(op.C32) |
                           reinterpret_cast<uintptr_t>(op.aux)) & 15u) == 0;
    // K need not be a multiple of 64 (slices past K read zeros); a K-major operand
    // needs K % 8 == 0 for its 16-byte rows, an MN-major A needs M % 64 == 0
    const bool k_ok = K > 0 && K < ((int64_t)1 << 31) - GBK && ((op.a_mn && !op.b_k) || K % 8 == 0);
    const bool mn_ok = !op.a_mn || M % 64 == 0;
    // a concatenated A: three bases, 64-column pieces, and exactly three of them
    const bool seg_ok =
        op.a_seg == 0 ||
        (op.a_seg > 0 && op.a_seg % 64 == 0 && op.A1 && op.A2 && op.lda1 % 8 == 0 && op.lda2 % 8 == 0 &&
         ((reinterpret_cast<uintptr_t>(op.A1) | reinterpret_cast<uintptr_t>(op.A2)) & 15u) == 0 &&
         (op.a_mn ? M : (int64_t)K) == 3 * (int64_t)op.a_seg);
    return aligned && mn_ok && k_ok && seg_ok && M > 0 && M < ((int64_t)1 << 31) - GBM && N > 0 && N % 32 == 0 &&
           op.lda % 8 == 0 &&
           op.ldb % 8 == 0 && op.ldc % 8 == 0 && (!op.aux || op.ldaux % 8 == 0);
}

cudaError_t launch_gemm_tc_ex(const GemmOperands &op, int64_t M, int N, int K, GemmEpilogue epi, bool silu,
                              int splits, WsHeader *hdr, cudaStream_t stream)
{
    if (M == 0)
        return cudaSuccess;
    GemmArgs g{};
    g.bias = static_cast<const __nv_bfloat16 *>(op.bias);
    g.aux = static_cast<const __nv_bfloat16 *>(op.aux);
    g.ldaux = op.ldaux;
    g.C = op.C;
    g.ldc = op.ldc;
    g.M = M;
    g.N = N;
    g.K = K;
    g.silu = silu;
    g.splits = std::max(1, std::min(splits, (K + GBK - 1) / GBK));
    g.a_seg = op.a_seg;
    g.hdr = hdr;
    switch (epi) {
    case GEMM_RED_F32:
        return gemm_dispatch_layout<128, EPI_RED>(op, g, stream);
    case GEMM_DSILU:
        return N % 256 == 0 ? gemm_dispatch_layout<256, EPI_DSILU>(op, g, stream)
                            : gemm_dispatch_layout<128, EPI_DSILU>(op, g, stream);
    default:
        return N % 256 == 0 ? gemm_dispatch_layout<256, EPI_ACT>(op, g, stream)
                            : gemm_dispatch_layout<128, EPI_ACT>(op, g, stream);
    }
}

bool gemm_e4m3_ok(const void *A, int64_t lda, const void *B, int64_t ldb, const void *C, int64_t ldc, int64_t M,
                  int N, int K)
{
    const bool aligned = ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) |
                           reinterpret_cast<uintptr_t>(C)) & 15u) == 0;
    return aligned && M > 0 && M < ((int64_t)1 << 31) - GBM && N > 0 && N % 128 == 0 && K > 0 && K % 16 == 0 &&
           lda % 16 == 0 && ldb % 16 == 0 && ldc % 8 == 0;
}

cudaError_t launch_gemm_e4m3(const void *A, int64_t lda, const float *sa, const void *B, int64_t ldb,
                             const float *sb, const void *bias, void *C, int64_t ldc, int64_t M, int N, int K,
                             bool silu, WsHeader *hdr, cudaStream_t stream)
{
    if (M == 0)
        return cudaSuccess;
    GemmOperands op{};
    op.A = A;
    op.lda = lda;
    op.B = B;
    op.ldb = ldb;
    op.b_k = true;
    GemmArgs g{};
    g.bias = static_cast<const __nv_bfloat16 *>(bias);
    g.C = C;
    g.ldc = ldc;
    g.M = M;
    g.N = N;
    g.K = K;
    g.silu = silu;
    g.splits = 1;
    g.sa = sa;
    g.sb = sb;
    g.hdr = hdr;
    return N % 256 == 0 ? gemm_tc_launch<256, false, true, EPI_ACT, true>(op, g, stream)
                        : gemm_tc_launch<128, false, true, EPI_ACT, true>(op, g, stream);
}

bool gemm_tc_supported(const void *A, int64_t lda, const void *Bm, void *C, int64_t ldc, int64_t M, int N, int K)
{
    GemmOperands op{};
    op.A = A;
    op.lda = lda;
    op.B = Bm;
    op.ldb = N;
    op.C = C;
    op.ldc = ldc;
    return gemm_tc_ok(op, M, N, K);
}

cudaError_t launch_gemm_tc(const void *A, int64_t lda, const void *Bm, const void *bias, void *C, int64_t ldc,
                           int64_t M, int N, int K, bool silu, WsHeader *hdr, cudaStream_t stream)
{
    GemmOperands op{};
    op.A = A;
    op.lda = lda;
    op.B = Bm;
    op.ldb = N;
    op.bias = bias;
    op.C = C;
    op.ldc = ldc;
    return launch_gemm_tc_ex(op, M, N, K, GEMM_ACT, silu, 1, hdr, stream);
}

}  // namespace hstu
