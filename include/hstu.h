/*
 * libhstu: B200 (sm_100a) HSTU jagged pointwise attention and transduction layer.
 *
 * What the calls compute (sources: "NVIDIA generative recommenders" summary,
 * section "HSTU Architecture"; "DLRMv4 Brings Sequence-Based Recommendation
 * Training to MLPerf", sections "Model Architecture", "HSTU Hyperparameters"
 * and "Computation Cost Analysis", Table 7):
 *
 *   for each sequence b (rows seq_offsets[b] .. seq_offsets[b+1]-1, local i, j)
 *   and each head:
 *     s_ij = q_i . k_j + rab_pos[clamp(p_i - p_j, pos_lo, pos_hi) - pos_lo]
 *                      + rab_time[min(NB-1, floor(log2(1 + max(t_i - t_j, 0))))]
 *     P_ij = SiLU(s_ij) * inv_n   if key j is visible from query i, else 0
 *     O_i  = sum_j P_ij v_j
 *   visibility: with n_t = num_targets[b] (0 when num_targets is NULL) the last
 *   n_t tokens are candidates; history rows see j <= i, candidate rows see the
 *   whole history and themselves.  p_i = i for history tokens and
 *   L_b - n_t for candidates (i with hstu_attn_desc.cand_positions = 1).
 *   Timestamps are integer seconds.
 *
 *   Layer: [U | V | Q | K] = SiLU(X W1 + b1) (column blocks in that order, each
 *   [T, H, d] with d fastest); O = attention(Q, K, V);
 *   G = LayerNorm_{H*d_v}(O; gamma, beta, eps) * U;  Y = G W2 + b2.
 *
 * Conventions for every call:
 *  - Pointers to tensors are DEVICE pointers; descriptors and size outputs are
 *    host memory.  The caller owns every buffer; the library allocates nothing
 *    and keeps no state between calls.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued asynchronously; no call synchronizes the host except
 *    hstu_check_device_flag.
 *  - Layouts: values are row-major jagged [T, H, d] (T = seq_offsets[B]),
 *    seq_offsets int64 [B+1], timestamps int64 [T], num_targets int32 [B] or
 *    NULL, rab_pos float32 [pos_hi - pos_lo + 1], rab_time float32 [NB] (one
 *    row per head, [H, ...], with hstu_attn_desc.per_head_tables).
 *    Weights are row-major.  dtype HSTU_BF16 means bf16 values/weights with
 *    fp32 accumulation (P is rounded to bf16 before P V); HSTU_F32 is fp32
 *    throughout.
 *  - Argument errors are found on the host before any launch and return
 *    HSTU_ERR_INVALID_ARG / HSTU_ERR_UNSUPPORTED / HSTU_ERR_WORKSPACE with
 *    nothing enqueued.  Inconsistent device data (seq_offsets not starting at 0,
 *    decreasing, exceeding T or max_seq_len; num_targets outside [0, L_b])
 *    never faults: the scheduler drops the offending sequences and records a
 *    flag in the workspace, which hstu_check_device_flag reports.  Kernels
 *    never trap.
 */
#ifndef HSTU_H
#define HSTU_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HSTU_OK = 0,
    HSTU_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad range */
    HSTU_ERR_UNSUPPORTED = 2,  /* a head dim the dtype's kernels do not take, d_qk != d_v, ... */
    HSTU_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
    HSTU_ERR_CUDA = 4,         /* a CUDA runtime call failed */
    HSTU_ERR_DEVICE_CHECK = 5  /* the device-side input check flagged the last call */
} hstu_status;

typedef enum { HSTU_F32 = 0, HSTU_BF16 = 1 } hstu_dtype;

/* Test hook of the bounded pipeline waits (hstu_attn_desc.debug_checks; bf16
 * hstu_attn_fwd and hstu_attn_fwd_noalloc only, HSTU_ERR_UNSUPPORTED elsewhere).
 * Every wait of the attention forward's pipeline gives up after about a
 * millisecond instead of about two seconds, and the first CTA withholds the
 * load of its first key tile, so its waits run out: the call still returns
 * HSTU_OK, its kernel ends without a fault, leaves that CTA's share of the
 * output unwritten, and sets bit 32 (timeout) of the workspace flag, which
 * hstu_check_device_flag reports.  The next ordinary call on the same
 * workspace clears the flag.  For tests of the timeout path only. */
#define HSTU_DEBUG_WAIT_TEST 2

typedef struct {
    int32_t num_seqs;         /* B >= 0 */
    int32_t max_seq_len;      /* >= every L_b; sizes the schedule */
    int64_t total_tokens;     /* T = seq_offsets[B] */
    int32_t num_heads;        /* H >= 1 */
    int32_t d_qk;             /* per-head query/key width: 64 or 128 (bf16, tcgen05 kernels), 32 or 64 (fp32) */
    int32_t d_v;              /* per-head value width: equal to d_qk */
    int32_t dtype;            /* hstu_dtype of q, k, v, out and their gradients */
    float inv_n;              /* the 1/N scale applied after SiLU */
    int32_t pos_lo, pos_hi;   /* rab_pos covers distances pos_lo..pos_hi */
    int32_t num_time_buckets; /* NB >= 1 */
    /* 0, or HSTU_DEBUG_WAIT_TEST (hstu_attn_fwd only; see below).  The device
     * input checks of seq_offsets and num_targets always run. */
    int32_t debug_checks;
    /* Semi-local attention (the ULTRA-HSTU review's local + global windows):
     * local_window > 0 keeps, of the pairs the causal/candidate rule keeps,
     * those whose query is fewer than local_window positions after the key or
     * whose key is among the first global_window tokens of its sequence.
     * local_window = 0 keeps the full mask; both must be >= 0. */
    int32_t local_window;
    int32_t global_window;
    /* 1: the attention forward computes Q K^T on the tensor cores in FP8 (the
     * mixed-precision item of the ULTRA-HSTU review): q and k are quantised per
     * (token, head) row to E4M3 inside hstu_attn_fwd (the scaling of
     * hstu_quantize_rows_e4m3) and the scores are rescaled by the two row scales;
     * P V stays bf16.  bf16 with d_qk = d_v = 128 only (HSTU_ERR_UNSUPPORTED
     * otherwise); the backward, the layer calls and hstu_attn_fwd_noalloc reject
     * it.  0: bf16 scores. */
    int32_t fp8_qk;
    /* Where the candidates sit on the positional axis (the pages fix p_i = i
     * for history tokens; they do not say where a candidate sits).  0: every
     * candidate of sequence b at position L_b - n_t, the first position after
     * the history (candidates are a set, not a continuation of each other).
     * 1: candidate i at its own index i.  Visibility is the same in both: a
     * candidate sees the whole history and itself.  The semi-local window
     * measures distances on the same axis. */
    int32_t cand_positions;
    /* 0: one rab_pos [pos_hi - pos_lo + 1] and one rab_time [NB] table, shared
     * by all heads.  1: one table per head, rab_pos [H, pos_hi - pos_lo + 1]
     * and rab_time [H, NB] row-major, head h adding row h; the bias-table
     * gradients then have the same [H, ...] shapes (each head's pairs summed
     * into its own row). */
    int32_t per_head_tables;
} hstu_attn_desc;

typedef struct {
    hstu_attn_desc attn;      /* attention part; dtype also types x, w1, b1, w2, b2, y */
    int32_t d_model;          /* D: width of X and Y (a multiple of 32 for bf16) */
    float ln_eps;             /* LayerNorm epsilon (1e-5 in the workloads) */
    /* Input of the output projection.  0: G = LayerNorm(O) U, H d_v wide, as in
     * the layer equation.  1: the concatenation [U | O | G], 3 H d_v wide (the
     * output-projection row of Table 7 on the DLRMv4 page counts that width; the
     * pages do not name the blocks, these are the layer's three H d_v-wide
     * tensors at that point), so that Y = U W2[0:F] + O W2[F:2F] + G W2[2F:3F]
     * + b2 with F = H d_v.  w2 and dw2 are then [3 H d_v, D]. */
    int32_t output_concat;
    /* 1: the projections f1 and f2 run in FP8 (the mixed-precision item of the
     * ULTRA-HSTU review: matrix multiplications in FP8, the rest in bf16).  X and
     * G are quantised per row to E4M3 inside the call; w1 and w2 are E4M3
     * weight packs made by hstu_quantize_weight_e4m3 from the bf16 weights.
     * Forward only, bf16 only, output_concat 0, D a multiple of 128. */
    int32_t fp8_projections;
} hstu_layer_desc;

/* Human-readable name of a status code (static string). */
const char *hstu_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int hstu_version(void);

/*
 * Bytes of device workspace an attention call needs (is_bwd = 0 forward,
 * 1 backward).  The workspace must be 256-byte aligned; its contents need no
 * initialisation and are scratch between calls.
 */
hstu_status hstu_attn_workspace_size(const hstu_attn_desc *desc, int is_bwd, size_t *bytes);

/* Bytes of device workspace hstu_layer_fwd needs. */
hstu_status hstu_layer_workspace_size(const hstu_layer_desc *desc, size_t *bytes);

/*
 * Attention forward: out[T, H, d_v] (overwritten; rows of all sequences
 * written, including empty-attention rows, which are zero).
 * q, k: [T, H, d_qk]; v, out: [T, H, d_v], all of desc->dtype.
 */
hstu_status hstu_attn_fwd(const hstu_attn_desc *desc, const void *q, const void *k,
                          const void *v, const int64_t *seq_offsets, const int64_t *timestamps,
                          const int32_t *num_targets, const float *rab_pos,
                          const float *rab_time, void *out, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * Attention backward for the loss sum(O * dout): dq, dk [T, H, d_qk],
 * dv [T, H, d_v] (desc->dtype) and the float32 bias-table gradients
 * d_rab_pos [pos_hi - pos_lo + 1], d_rab_time [NB], summed over all pairs and
 * heads ([H, ...], each head's pairs in its own row, with per_head_tables).  Every output is overwritten, not accumulated.  The pair
 * gradient is dS_ij = (dout_i . v_j) * SiLU'(s_ij) * inv_n.
 */
hstu_status hstu_attn_bwd(const hstu_attn_desc *desc, const void *q, const void *k,
                          const void *v, const int64_t *seq_offsets, const int64_t *timestamps,
                          const int32_t *num_targets, const float *rab_pos,
                          const float *rab_time, const void *dout, void *dq, void *dk, void *dv,
                          float *d_rab_pos, float *d_rab_time, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * One transduction layer forward.  x [T, D]; w1 [D, H(2 d_v + 2 d_qk)];
 * b1 [H(2 d_v + 2 d_qk)]; w2 [H d_v, D] ([3 H d_v, D] with output_concat);
 * b2 [D] (dtype of the desc);
 * ln_gamma, ln_beta float32 [H d_v]; y [T, D] (overwritten).
 * saved_uvqk [T, H(2 d_v + 2 d_qk)] and saved_o [T, H d_v] are optional
 * (NULL = not kept); when given they receive SiLU(X W1 + b1) and the
 * attention output, as a training step would keep them.
 */
hstu_status hstu_layer_fwd(const hstu_layer_desc *desc, const void *x, const void *w1,
                           const void *b1, const void *w2, const void *b2,
                           const float *ln_gamma, const float *ln_beta,
                           const int64_t *seq_offsets, const int64_t *timestamps,
                           const int32_t *num_targets, const float *rab_pos,
                           const float *rab_time, void *y, void *saved_uvqk, void *saved_o,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Bytes of device workspace hstu_layer_bwd needs (256-byte aligned, scratch).
 */
hstu_status hstu_layer_bwd_workspace_size(const hstu_layer_desc *desc, size_t *bytes);

/*
 * One transduction layer backward for the loss sum(Y * dy) (the layer of
 * hstu_layer_fwd; the DLRMv4 page's "Computation Cost Analysis" counts its
 * GEMMs three times over the forward's).  bf16 only.
 * Inputs: the forward's x, w1, b1, w2, ln_gamma, ln_beta, bias tables and
 * sequence data; saved_uvqk = SiLU(X W1 + b1) and saved_o = the attention
 * output, as hstu_layer_fwd keeps them; dy [T, D] (bf16).
 * Outputs (all overwritten): dx [T, D] (bf16); dw1 [D, W], db1 [W],
 * dw2 [H d_v, D] ([3 H d_v, D] with output_concat), db2 [D], d_ln_gamma,
 * d_ln_beta [H d_v], d_rab_pos and d_rab_time shaped as the tables (all
 * float32; W = H(2 d_v + 2 d_qk)).
 * The pre-activation X W1 + b1 is recomputed (its SiLU derivative is applied
 * in that GEMM's epilogue), and G = LayerNorm(O) U from saved_o and U.
 * Requires D, H d_v and W multiples of 128 (HSTU_ERR_UNSUPPORTED otherwise);
 * every pointer 16-byte aligned (HSTU_ERR_INVALID_ARG).
 */
hstu_status hstu_layer_bwd(const hstu_layer_desc *desc, const void *x, const void *w1, const void *b1,
                           const void *w2, const float *ln_gamma, const float *ln_beta,
                           const int64_t *seq_offsets, const int64_t *timestamps,
                           const int32_t *num_targets, const float *rab_pos, const float *rab_time,
                           const void *saved_uvqk, const void *saved_o, const void *dy, void *dx,
                           float *dw1, float *db1, float *dw2, float *db2, float *d_ln_gamma,
                           float *d_ln_beta, float *d_rab_pos, float *d_rab_time, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * Attention truncation (the "ULTRA-HSTU (Meta)" review, "Attention
 * Truncation"): the first layers run over whole histories, the remaining ones
 * over each history's most recent segment only.  Sequence b (rows
 * seq_offsets[b] .. seq_offsets[b+1]-1, n_t = num_targets[b] candidates at its
 * end, 0 when num_targets is NULL, hist = L_b - n_t) keeps its last
 * min(hist, keep) history tokens and all of its candidates, in order.
 *   in          [total_tokens, row_bytes] bytes of any per-token tensor (layer
 *               activations, timestamps); device.
 *   out         room for total_tokens rows (the kept count is never larger);
 *               receives the kept rows, packed; device.
 *   out_offsets [num_seqs + 1] int64, device: the kept batch's seq_offsets.
 * num_targets serves the kept batch unchanged.  Positions restart at 0 in the
 * kept batch; the bias uses only differences of positions and timestamps, so
 * every pair that survives the cut keeps its bias.  row_bytes must be a
 * positive multiple of 4; in and out 16-byte aligned when row_bytes is a
 * multiple of 16, else 4-byte aligned (HSTU_ERR_INVALID_ARG otherwise; also
 * for keep < 0).  At most 12288 sequences per call (HSTU_ERR_UNSUPPORTED
 * above).  Sequence data outside the jagged rules is clamped to
 * [0, total_tokens]: the rows written are then unspecified, but nothing is
 * read or written outside in and out.
 */
hstu_status hstu_jagged_truncate(int32_t num_seqs, int64_t total_tokens, int32_t keep,
                                 const int64_t *seq_offsets, const int32_t *num_targets, const void *in,
                                 int64_t row_bytes, void *out, int64_t *out_offsets, void *stream);

/*
 * FP8 (E4M3) projections.  Format and scaling (the pages name neither): E4M3
 * (largest finite 448), round to nearest even with saturation; activations
 * scaled per row and weights per output column so that the largest magnitude
 * maps to 448: inv = 448 / amax, scale = amax / 448 (float32), code =
 * E4M3(x * inv); an all-zero row or column has scale 1.
 *
 * Weight pack (device memory, hstu_e4m3_weight_bytes(K, N) bytes, 16-byte
 * aligned): the codes of W^T, uint8 [N][K] (row n = output column n), then at
 * byte offset align256(N K) the float32 scales [N].
 */
size_t hstu_e4m3_weight_bytes(int32_t K, int32_t N);

/* Quantise a bf16 weight w [K, N] (row-major, device) into a weight pack.
 * K a multiple of 16. */
hstu_status hstu_quantize_weight_e4m3(const void *w, int32_t K, int32_t N, void *pack, void *stream);

/* Quantise the rows of a bf16 matrix x [rows, K] (device, 16-byte aligned, K a
 * multiple of 16): codes uint8 [rows, K] and scales float32 [rows] (device). */
hstu_status hstu_quantize_rows_e4m3(const void *x, int64_t rows, int32_t K, void *codes, float *scales,
                                    void *stream);

/* y bf16 [M, N] = (dec(codes) scales) (dec(W) w_scales)^T + bias, optionally
 * SiLU: the FP8 projection GEMM on the tensor cores (tcgen05 kind::f8f6f4,
 * float32 accumulation).  codes [M, K] and scales [M] from
 * hstu_quantize_rows_e4m3, wpack from hstu_quantize_weight_e4m3 (K x N),
 * bias bf16 [N] or NULL.  N a multiple of 128, K of 16 (HSTU_ERR_UNSUPPORTED).
 * workspace: at least 256 bytes of device memory (256-byte aligned); its flag
 * reports a stalled pipeline through hstu_check_device_flag. */
hstu_status hstu_gemm_e4m3(const void *codes, const float *scales, int64_t M, int32_t K, const void *wpack,
                           int32_t N, const void *bias, int32_t apply_silu, void *y, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * Attention forward that allocates nothing (no counterpart on the HSTU
 * pages; it exists for callers, not for the method).  Same computation,
 * arguments and layouts as hstu_attn_fwd, without the workspace: some callers
 * cannot allocate device memory at all, such as a plugin inside a host
 * framework that owns every device allocation and passes it only input and
 * output buffers, or a latency-critical path that may not call cudaMalloc
 * because it can synchronize the device.  The scheduler's scratch lives in a
 * static device array of about 512 KiB that every GPU loading this library
 * holds until exit; problems needing more than 65536 work items
 * (ceil(T / 64) + B) return HSTU_ERR_UNSUPPORTED before anything is enqueued.
 * The first call on each device looks the array's address up (with that
 * device current) and should come before any stream capture.  Calls share
 * the array, so calls that overlap on the GPU race and must be serialized by
 * the caller.  The device input-check flag is kept in that array and is not
 * reported; inconsistent sequences are still dropped, never read out of range.
 */
hstu_status hstu_attn_fwd_noalloc(const hstu_attn_desc *desc, const void *q, const void *k,
                                  const void *v, const int64_t *seq_offsets,
                                  const int64_t *timestamps, const int32_t *num_targets,
                                  const float *rab_pos, const float *rab_time, void *out,
                                  void *stream);

/*
 * Synchronizes `stream` and reports the device-side input check of the most
 * recent call that used `workspace`: HSTU_OK or HSTU_ERR_DEVICE_CHECK.  The
 * flag's bits (1 = seq_offsets[0] != 0, 2 = a sequence decreasing or past T,
 * 4 = a sequence longer than max_seq_len, 8 = num_targets outside [0, L_b],
 * 16 = seq_offsets[B] != T, 32 = a pipeline wait of a tcgen05 kernel ran
 * out: the kernel gave up instead of hanging, and its output is incomplete)
 * are stored in *bits when bits is not NULL.
 */
hstu_status hstu_check_device_flag(const void *workspace, int32_t *bits, void *stream);

/*
 * Test hook: the bias indices the attention kernels use for n global token
 * pairs (rows[2e], rows[2e+1]) = (i, j) of the same sequence.  Writes
 * pos_index[e] = clamp(p_i - p_j, lo, hi) - lo and bucket[e] (int32, device).
 * Pairs whose rows lie in different sequences get -1 in both outputs.
 */
hstu_status hstu_debug_bias_indices(const hstu_attn_desc *desc, const int64_t *seq_offsets,
                                    const int64_t *timestamps, const int32_t *num_targets,
                                    const int64_t *rows, int64_t n, int32_t *pos_index,
                                    int32_t *bucket, void *stream);

/*
 * Test hook: run the jagged tile scheduler alone.  Writes the work list the
 * attention kernels consume, as int32 pairs (sequence, tile) in processing
 * order, into items[2 * max_items] and the count into *count (device).
 * `flag` is a device buffer of at least 256 bytes (the workspace header);
 * its first int32 receives the input-check bits.  Forward tiles are query
 * tiles of `tile_rows` rows; backward tiles are key tiles.  Returns
 * HSTU_ERR_WORKSPACE if max_items is below the bound ceil(T / tile_rows) + B.
 */
hstu_status hstu_debug_schedule(const hstu_attn_desc *desc, const int64_t *seq_offsets,
                                const int32_t *num_targets, int is_bwd, int32_t tile_rows,
                                int32_t *items, int32_t max_items, int32_t *count,
                                int32_t *flag, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H */
