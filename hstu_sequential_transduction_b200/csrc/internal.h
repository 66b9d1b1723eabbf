// Host-side launchers shared between the kernel files and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hstu {

struct WsHeader;
struct AttnParams;

// SM count and L2 size of the current device (cached per device).
struct DeviceInfo {
    int sms = 148;
    int64_t l2_bytes = 126 << 20;
};
DeviceInfo device_info();

// Tile rows of the work items each attention implementation consumes: 64 for
// the fp32 kernels (the work list is always sized for this, the finer tiling),
// 128 for the tcgen05 kernels.
constexpr int kF32Tile = 64;
constexpr int kTcTile = 128;

cudaError_t launch_schedule(const int64_t *off, const int32_t *nt, int B, int64_t T, int max_len,
                            int tile, int is_bwd, int2 *items, int capacity, WsHeader *hdr,
                            int32_t *count_out, cudaStream_t stream);

cudaError_t launch_debug_indices(const int64_t *off, const int64_t *ts, const int32_t *nt, int B,
                                 int lo, int hi, int nb, bool own, const int64_t *rows, int64_t n,
                                 int32_t *pos_out, int32_t *bkt_out, cudaStream_t stream);

// bf16 attention on tcgen05 / TMA (sm_100a), 128-row tiles, head dims 64 and 128.
// tensor_maps_available: the driver exposes cuTensorMapEncodeTiled (without it no
// tcgen05 kernel can run).  attn_tc_supported: the shape is one the kernels take.
bool tensor_maps_available();
bool attn_tc_supported(const AttnParams &p);
cudaError_t launch_attn_fwd_tc(const AttnParams &p, int grid_items, cudaStream_t stream);
// 2-D bf16 tensor map over [rows, cols] with a row stride, 64 x 128 boxes, 128B swizzle.
cudaError_t make_row_tensor_map(CUtensorMap *map, const void *base, int64_t rows, int cols,
                                int64_t row_stride_elems);
// General 2-D tensor map (row stride in bytes, box of box_cols x box_rows elements).
cudaError_t make_tensor_map_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype,
                               int64_t rows, int64_t cols, int64_t row_stride_bytes, int box_cols,
                               int box_rows, CUtensorMapSwizzle swizzle);
// bf16 backward on tcgen05 (head dims 64, 128), key tiles of 128 rows; dq_acc
// receives dQ / (0.5 * inv_n) (apply that scale when converting).
cudaError_t launch_attn_bwd_tc(const AttnParams &p, int grid_items, cudaStream_t stream);

// fp32 attention on CUDA cores, 64-row tiles.
cudaError_t launch_attn_fwd_f32(const AttnParams &p, int grid_items, cudaStream_t stream);
cudaError_t launch_attn_bwd_f32(const AttnParams &p, int grid_items, cudaStream_t stream);

// dq (bf16, rows of stride sdq, 16-byte aligned) <- scale * dq_acc (fp32 [T, H d]).
cudaError_t launch_convert_dq(const float *acc, void *dq, int64_t T, int H, int d, int64_t sdq,
                              float scale, cudaStream_t stream);

// C[M, N] = act(A[M, K] B[K, N] + bias[N]) on tcgen05 / TMA (sm_100a); act =
// SiLU if silu.  Row strides lda, ldc in elements; B is dense [K, N]; K a
// multiple of 8, N of 32.  hdr receives a timeout flag if a pipeline wait ever
// gives up.  launch_gemm_f32 is the same in fp32 on CUDA cores.
bool gemm_tc_supported(const void *A, int64_t lda, const void *Bm, void *C, int64_t ldc, int64_t M, int N, int K);
cudaError_t launch_gemm_tc(const void *A, int64_t lda, const void *Bm, const void *bias, void *C, int64_t ldc,
                           int64_t M, int N, int K, bool silu, WsHeader *hdr, cudaStream_t stream);
cudaError_t launch_gemm_f32(const float *A, int64_t lda, const float *Bm, const float *bias,
                            float *C, int64_t ldc, int64_t M, int N, int K, bool silu,
                            cudaStream_t stream);

// General tcgen05 GEMM C[M, N] = epi(A B) (bf16 operands, fp32 accumulation).
//   A: a_mn = false -> A[m][k] at A + m*lda + k;  a_mn = true -> at A + k*lda + m
//   B: b_k = false  -> B[k][n] at B + k*ldb + n;  b_k = true  -> at B + n*ldb + k
//   GEMM_ACT:    C bf16 = acc + bias (optionally SiLU)
//   GEMM_DSILU:  C bf16 = aux * SiLU'(acc + bias), aux bf16 [M, N] (row stride ldaux)
//   GEMM_RED_F32: C32 fp32 += acc, the k range split over `splits` CTAs (C32 must
//                 hold its initial value, e.g. zeros); ldc in elements.
// A may be the column concatenation of three stored matrices with the same row
// count: a_seg > 0 (a multiple of 64) is the width of each, A, A1, A2 their
// bases and lda, lda1, lda2 their row strides.  The stored columns are K for a
// K-major A and M for an MN-major A, so the concatenation runs along K or M.
enum GemmEpilogue { GEMM_ACT = 0, GEMM_DSILU = 1, GEMM_RED_F32 = 2 };
struct GemmOperands {
    const void *A;
    int64_t lda;
    const void *A1, *A2;
    int64_t lda1, lda2;
    int a_seg;
    bool a_mn;
    const void *B;
    int64_t ldb;
    bool b_k;
    const void *bias;
    const void *aux;
    int64_t ldaux;
    void *C;
    float *C32;
    int64_t ldc;
};
bool gemm_tc_ok(const GemmOperands &op, int64_t M, int N, int K);
cudaError_t launch_gemm_tc_ex(const GemmOperands &op, int64_t M, int N, int K, GemmEpilogue epi, bool silu,
                              int splits, WsHeader *hdr, cudaStream_t stream);

// E4M3 GEMM on tcgen05 (kind::f8f6f4): C bf16 [M, N] = (A B^T) * sa[m] * sb[n]
// + bias[n], optionally SiLU.  A codes [M, K] (row stride lda bytes), B codes
// [N, K] (row stride ldb bytes), both K-major; sa [M], sb [N] float32.
bool gemm_e4m3_ok(const void *A, int64_t lda, const void *B, int64_t ldb, const void *C, int64_t ldc, int64_t M,
                  int N, int K);
cudaError_t launch_gemm_e4m3(const void *A, int64_t lda, const float *sa, const void *B, int64_t ldb,
                             const float *sb, const void *bias, void *C, int64_t ldc, int64_t M, int N, int K,
                             bool silu, WsHeader *hdr, cudaStream_t stream);
// Per-row E4M3 quantisation of a bf16 [R, K] matrix (row stride ldx elements):
// codes [R, K] (row stride ldq bytes) and scales [R]; K a multiple of 8.
cudaError_t launch_quantize_rows_e4m3(const void *x, int64_t ldx, int64_t R, int K, void *q, int64_t ldq,
                                      float *scale, cudaStream_t stream);
// Per-column E4M3 quantisation of a bf16 weight [K, N]: codes [N, K] (the
// transpose) and scales [N].
cudaError_t launch_quantize_cols_e4m3(const void *w, int64_t K, int N, void *q, float *scale, cudaStream_t stream);

// G[t, :] = LayerNorm(O[t, :]) * U[t, :] over F features.
cudaError_t launch_norm_gate(bool bf16, const void *O, int64_t ldo, const void *U, int64_t ldu,
                             const float *gamma, const float *beta, float eps, void *G,
                             int64_t ldg, int64_t T, int F, cudaStream_t stream);

// Backward of G = LayerNorm(O) * U (bf16): writes dO and dU (row strides in
// elements) and adds the parameter gradients to dgamma, dbeta (fp32 [F]).
cudaError_t launch_norm_gate_bwd(const void *dG, int64_t ldd, const void *O, int64_t ldo, const void *U,
                                 int64_t ldu, const float *gamma, const float *beta, float eps, void *dO,
                                 int64_t lddo, void *dU, int64_t lddu, float *dgamma, float *dbeta, int64_t T,
                                 int F, bool cat, cudaStream_t stream);
// cat: dG is the last F-wide block of rows [dU' | dO' | dG] whose first two
// blocks (direct gradients through an output projection over [U | O | G]) are
// added to dU and dO.
// out[t, :] = [a[t, :] | b[t, :] | c[t, :]], each block `bytes` wide (a multiple
// of 4); row strides lda, ldb, ldc in bytes.
cudaError_t launch_concat3(const void *a, int64_t lda, const void *b, int64_t ldb, const void *c, int64_t ldc,
                           void *out, int64_t T, int64_t bytes, cudaStream_t stream);
// out[n] += sum over T rows of A[row, n] (bf16 A, fp32 out).
cudaError_t launch_colsum_bf16(const void *A, int64_t lda, int64_t T, int N, float *out, cudaStream_t stream);

// Attention truncation (at most kTruncateMaxSeqs sequences: the new offsets
// live in shared memory): out_off [B+1] = offsets of every sequence's last
// min(hist, keep) history tokens plus its candidates; out = those rows of in
// (row_bytes a multiple of 4; 16-byte copies when it is a multiple of 16).
constexpr int kTruncateMaxSeqs = 12288;
cudaError_t launch_jagged_truncate(const int64_t *off, const int32_t *nt, int B, int64_t T, int keep,
                                   int64_t row_bytes, const void *in, void *out, int64_t *out_off,
                                   cudaStream_t stream);

}  // namespace hstu
