// C ABI of libhstu: argument validation, workspace carving and kernel dispatch.
// Every check that can fail runs on the host before anything is enqueued.
#include <climits>
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "internal.h"

using namespace hstu;

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hstu_status check_attn_desc(const hstu_attn_desc *d)
{
    if (!d)
        return HSTU_ERR_INVALID_ARG;
    if (d->num_seqs < 0 || d->max_seq_len < 0 || d->total_tokens < 0 || d->num_heads < 1 ||
        d->num_time_buckets < 1 || d->pos_hi < d->pos_lo || !std::isfinite(d->inv_n) ||
        d->local_window < 0 || d->global_window < 0)
        return HSTU_ERR_INVALID_ARG;
    if (d->dtype != HSTU_F32 && d->dtype != HSTU_BF16)
        return HSTU_ERR_INVALID_ARG;
    if ((int64_t)d->pos_hi - d->pos_lo + 1 > (1 << 24))
        return HSTU_ERR_UNSUPPORTED;
    if (d->d_qk != d->d_v)
        return HSTU_ERR_UNSUPPORTED;
    // bf16 runs on the tcgen05 kernels only, which take head dims 64 and 128
    if (d->dtype == HSTU_BF16 && d->d_qk != 64 && d->d_qk != 128)
        return HSTU_ERR_UNSUPPORTED;
    if (d->dtype == HSTU_F32 && d->d_qk != 32 && d->d_qk != 64)
        return HSTU_ERR_UNSUPPORTED;
    if (d->fp8_qk != 0 && d->fp8_qk != 1)
        return HSTU_ERR_INVALID_ARG;
    if (d->debug_checks != 0 && d->debug_checks != HSTU_DEBUG_WAIT_TEST)
        return HSTU_ERR_INVALID_ARG;
    if (d->fp8_qk && (d->dtype != HSTU_BF16 || d->d_qk != 128))
        return HSTU_ERR_UNSUPPORTED;
    if ((d->cand_positions != 0 && d->cand_positions != 1) ||
        (d->per_head_tables != 0 && d->per_head_tables != 1))
        return HSTU_ERR_INVALID_ARG;
    // per-head tables are indexed with 32-bit offsets
    if (d->per_head_tables && (((int64_t)d->pos_hi - d->pos_lo + 1) * d->num_heads > INT_MAX ||
                               (int64_t)d->num_time_buckets * d->num_heads > INT_MAX))
        return HSTU_ERR_UNSUPPORTED;
    if (max_items(d->total_tokens, d->num_seqs, kF32Tile) > INT_MAX / 4 ||
        d->total_tokens * d->num_heads > ((int64_t)1 << 40))
        return HSTU_ERR_UNSUPPORTED;
    return HSTU_OK;
}

size_t elem_bytes(const hstu_attn_desc *d) { return d->dtype == HSTU_BF16 ? 2 : 4; }

size_t items_bytes(const hstu_attn_desc *d)
{
    return align256(sizeof(int2) * (size_t)max_items(d->total_tokens, d->num_seqs, kF32Tile));
}

size_t attn_ws(const hstu_attn_desc *d, int is_bwd)
{
    size_t b = sizeof(WsHeader) + items_bytes(d);
    if (is_bwd && d->dtype == HSTU_BF16)
        b += align256(sizeof(float) * (size_t)d->total_tokens * d->num_heads * d->d_qk);
    if (!is_bwd && d->fp8_qk)  // E4M3 codes of q and k, then their row scales
        b += 2 * align256((size_t)d->total_tokens * d->num_heads * d->d_qk) +
             2 * align256(sizeof(float) * (size_t)d->total_tokens * d->num_heads);
    return b;
}

hstu_status check_ws(void *ws, size_t have, size_t need)
{
    if (need && (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)))
        return HSTU_ERR_WORKSPACE;
    return have < need ? HSTU_ERR_WORKSPACE : HSTU_OK;
}

hstu_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA; }

#define HSTU_TRY(x)                        \
    do {                                   \
        hstu_status _s = (x);              \
        if (_s != HSTU_OK)                 \
            return _s;                     \
    } while (0)

#define HSTU_CUDA(x) HSTU_TRY(cuda_status(x))

// The bf16 attention runs on the tcgen05 kernels and nowhere else: a driver
// without the tensor-map encoder is a CUDA error, a shape those kernels do not
// take is unsupported.
hstu_status tc_status(const AttnParams &p)
{
    if (!tensor_maps_available())
        return HSTU_ERR_CUDA;
    return attn_tc_supported(p) ? HSTU_OK : HSTU_ERR_UNSUPPORTED;
}

AttnParams base_params(const hstu_attn_desc *d, const int64_t *off, const int64_t *ts,
                       const int32_t *nt, const float *rp, const float *rt, void *ws)
{
    AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.seq_offsets = off;
    p.timestamps = ts;
    p.num_targets = nt;
    p.rab_pos = rp;
    p.rab_time = rt;
    p.B = d->num_seqs;
    p.H = d->num_heads;
    p.dqk = d->d_qk;
    p.dv = d->d_v;
    p.max_seq_len = d->max_seq_len;
    p.T = d->total_tokens;
    p.inv_n = d->inv_n;
    p.pos_lo = d->pos_lo;
    p.pos_hi = d->pos_hi;
    p.nb = d->num_time_buckets;
    p.lw = d->local_window;
    p.gw = d->global_window;
    p.cand_own = d->cand_positions;
    p.pos_hstride = d->per_head_tables ? (int64_t)d->pos_hi - d->pos_lo + 1 : 0;
    p.time_hstride = d->per_head_tables ? d->num_time_buckets : 0;
    p.hdr = static_cast<WsHeader *>(ws);
    const bool wait_test = d->debug_checks == HSTU_DEBUG_WAIT_TEST;
    p.wait_limit = wait_test ? kTestWaitLimitCycles : kWaitLimitCycles;
    p.withhold_first_k = wait_test ? 1 : 0;
    p.items = reinterpret_cast<const int2 *>(static_cast<char *>(ws) + sizeof(WsHeader));
    return p;
}

// The bias-table gradients are sums over pairs: zeroed before every backward.
hstu_status zero_table_grads(const hstu_attn_desc *d, float *d_rab_pos, float *d_rab_time, cudaStream_t st)
{
    const size_t rows = d->per_head_tables ? (size_t)d->num_heads : 1;
    HSTU_CUDA(cudaMemsetAsync(d_rab_pos, 0, sizeof(float) * rows * (size_t)(d->pos_hi - d->pos_lo + 1), st));
    return cuda_status(cudaMemsetAsync(d_rab_time, 0, sizeof(float) * rows * d->num_time_buckets, st));
}

int grid_items(const hstu_attn_desc *d, int tile = kF32Tile)
{
    return (int)max_items(d->total_tokens, d->num_seqs, tile);
}

// The work list always has room for the 64-row bound, the largest of all tilings.
hstu_status schedule(const hstu_attn_desc *d, const int64_t *off, const int32_t *nt, int is_bwd,
                     void *ws, cudaStream_t stream, int tile = kF32Tile)
{
    int2 *items = reinterpret_cast<int2 *>(static_cast<char *>(ws) + sizeof(WsHeader));
    return cuda_status(launch_schedule(off, nt, d->num_seqs, d->total_tokens, d->max_seq_len,
                                       tile, is_bwd, items, grid_items(d),
                                       static_cast<WsHeader *>(ws), nullptr, stream));
}

// Attention forward on explicit row strides (used by the layer as well).
hstu_status attn_fwd_strided(const hstu_attn_desc *d, const void *q, int64_t sq, const void *k,
                             int64_t sk, const void *v, int64_t sv, const int64_t *off,
                             const int64_t *ts, const int32_t *nt, const float *rp, const float *rt,
                             void *out, int64_t so, void *ws, cudaStream_t stream)
{
    AttnParams p = base_params(d, off, ts, nt, rp, rt, ws);
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = out;
    p.sq = sq;
    p.sk = sk;
    p.sv = sv;
    p.so = so;
    if (d->dtype == HSTU_BF16) {
        HSTU_TRY(tc_status(p));
        HSTU_TRY(schedule(d, off, nt, 0, ws, stream, kTcTile));
        return cuda_status(launch_attn_fwd_tc(p, grid_items(d, kTcTile), stream));
    }
    HSTU_TRY(schedule(d, off, nt, 0, ws, stream));
    return cuda_status(launch_attn_fwd_f32(p, grid_items(d), stream));
}

// Attention backward with explicit row strides (elements) for every tensor; the
// fp32 path needs dense dq, dk, dv (it zeroes them as whole buffers).
hstu_status attn_bwd_strided(const hstu_attn_desc *desc, const void *q, int64_t sq, const void *k, int64_t sk,
                             const void *v, int64_t sv, const int64_t *seq_offsets, const int64_t *timestamps,
                             const int32_t *num_targets, const float *rab_pos, const float *rab_time,
                             const void *dout, int64_t sdo, void *dq, int64_t sdq, void *dk, int64_t sdk, void *dv,
                             int64_t sdv, float *d_rab_pos, float *d_rab_time, void *workspace, cudaStream_t st)
{
    HSTU_TRY(zero_table_grads(desc, d_rab_pos, d_rab_time, st));
    const int64_t row = (int64_t)desc->num_heads * desc->d_qk;
    const size_t tensor_bytes = (size_t)desc->total_tokens * row * elem_bytes(desc);
    const bool bf16 = desc->dtype == HSTU_BF16;
    AttnParams p = base_params(desc, seq_offsets, timestamps, num_targets, rab_pos, rab_time, workspace);
    p.q = q;
    p.k = k;
    p.v = v;
    p.sq = sq;
    p.sk = sk;
    p.sv = sv;
    p.dout = dout;
    p.sdo = sdo;
    p.dq = dq;
    p.dk = dk;
    p.dvv = dv;
    p.sdq = sdq;
    p.sdk = sdk;
    p.sdv = sdv;
    p.d_rab_pos = d_rab_pos;
    p.d_rab_time = d_rab_time;
    if (bf16) {
        p.dq_acc = reinterpret_cast<float *>(static_cast<char *>(workspace) + sizeof(WsHeader) +
                                             items_bytes(desc));
        HSTU_CUDA(cudaMemsetAsync(p.dq_acc, 0, sizeof(float) * (size_t)desc->total_tokens * row, st));
        HSTU_TRY(tc_status(p));
        HSTU_TRY(schedule(desc, seq_offsets, num_targets, 1, workspace, st, kTcTile));
        HSTU_CUDA(launch_attn_bwd_tc(p, grid_items(desc, kTcTile), st));
        return cuda_status(launch_convert_dq(p.dq_acc, dq, desc->total_tokens, desc->num_heads,
                                             desc->d_qk, sdq, 0.5f * desc->inv_n, st));
    }
    if (sdq != row || sdk != row || sdv != row)
        return HSTU_ERR_UNSUPPORTED;
    if (tensor_bytes) {
        HSTU_CUDA(cudaMemsetAsync(dk, 0, tensor_bytes, st));
        HSTU_CUDA(cudaMemsetAsync(dv, 0, tensor_bytes, st));
        HSTU_CUDA(cudaMemsetAsync(dq, 0, tensor_bytes, st));
    }
    HSTU_TRY(schedule(desc, seq_offsets, num_targets, 0, workspace, st));
    return cuda_status(launch_attn_bwd_f32(p, grid_items(desc), st));
}

}  // namespace

extern "C" {

const char *hstu_status_string(int status)
{
    switch (status) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARG: return "HSTU_ERR_INVALID_ARG: invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED: unsupported shape or dtype";
    case HSTU_ERR_WORKSPACE: return "HSTU_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA: a CUDA runtime call failed";
    case HSTU_ERR_DEVICE_CHECK: return "HSTU_ERR_DEVICE_CHECK: device-side input check failed";
    default: return "unknown hstu_status";
    }
}

int hstu_version(void) { return kVersion; }

hstu_status hstu_attn_workspace_size(const hstu_attn_desc *desc, int is_bwd, size_t *bytes)
{
    HSTU_TRY(check_attn_desc(desc));
    if (!bytes)
        return HSTU_ERR_INVALID_ARG;
    *bytes = attn_ws(desc, is_bwd);
    return HSTU_OK;
}

hstu_status hstu_attn_fwd(const hstu_attn_desc *desc, const void *q, const void *k, const void *v,
                          const int64_t *seq_offsets, const int64_t *timestamps,
                          const int32_t *num_targets, const float *rab_pos, const float *rab_time,
                          void *out, void *workspace, size_t workspace_bytes, void *stream)
{
    HSTU_TRY(check_attn_desc(desc));
    if (!seq_offsets || !rab_pos || !rab_time)
        return HSTU_ERR_INVALID_ARG;
    if (desc->total_tokens > 0 && (!q || !k || !v || !out || !timestamps))
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return HSTU_ERR_INVALID_ARG;
    HSTU_TRY(check_ws(workspace, workspace_bytes, attn_ws(desc, 0)));
    const int64_t row = (int64_t)desc->num_heads * desc->d_qk;
    if (desc->fp8_qk) {
        // q and k to E4M3 per (token, head) row, then the FP8-score kernel
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        const int64_t T = desc->total_tokens, R = T * desc->num_heads;
        char *cur = static_cast<char *>(workspace) + sizeof(WsHeader) + items_bytes(desc);
        char *q8 = cur;
        char *k8 = q8 + align256((size_t)R * 128);
        float *sq = reinterpret_cast<float *>(k8 + align256((size_t)R * 128));
        float *sk = reinterpret_cast<float *>(reinterpret_cast<char *>(sq) + align256(sizeof(float) * R));
        HSTU_CUDA(launch_quantize_rows_e4m3(q, 128, R, 128, q8, 128, sq, st));
        HSTU_CUDA(launch_quantize_rows_e4m3(k, 128, R, 128, k8, 128, sk, st));
        AttnParams p = base_params(desc, seq_offsets, timestamps, num_targets, rab_pos, rab_time, workspace);
        p.q = q;
        p.k = k;
        p.v = v;
        p.o = out;
        p.sq = p.sk = p.sv = p.so = row;
        p.q8 = q8;
        p.k8 = k8;
        p.sq8 = sq;
        p.sk8 = sk;
        HSTU_TRY(tc_status(p));
        HSTU_TRY(schedule(desc, seq_offsets, num_targets, 0, workspace, st, kTcTile));
        return cuda_status(launch_attn_fwd_tc(p, grid_items(desc, kTcTile), st));
    }
    return attn_fwd_strided(desc, q, row, k, row, v, row, seq_offsets, timestamps, num_targets,
                            rab_pos, rab_time, out, row, workspace, static_cast<cudaStream_t>(stream));
}

hstu_status hstu_attn_bwd(const hstu_attn_desc *desc, const void *q, const void *k, const void *v,
                          const int64_t *seq_offsets, const int64_t *timestamps,
                          const int32_t *num_targets, const float *rab_pos, const float *rab_time,
                          const void *dout, void *dq, void *dk, void *dv, float *d_rab_pos,
                          float *d_rab_time, void *workspace, size_t workspace_bytes, void *stream)
{
    HSTU_TRY(check_attn_desc(desc));
    if (desc->fp8_qk || desc->debug_checks)  // forward-only options
        return HSTU_ERR_UNSUPPORTED;
    if (!seq_offsets || !rab_pos || !rab_time || !d_rab_pos || !d_rab_time)
        return HSTU_ERR_INVALID_ARG;
    if (desc->total_tokens > 0 &&
        (!q || !k || !v || !dout || !dq || !dk || !dv || !timestamps))
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return HSTU_ERR_INVALID_ARG;
    HSTU_TRY(check_ws(workspace, workspace_bytes, attn_ws(desc, 1)));
    const int64_t row = (int64_t)desc->num_heads * desc->d_qk;
    return attn_bwd_strided(desc, q, row, k, row, v, row, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                            dout, row, dq, row, dk, row, dv, row, d_rab_pos, d_rab_time, workspace,
                            static_cast<cudaStream_t>(stream));
}

static hstu_status check_layer_desc(const hstu_layer_desc *d)
{
    if (!d)
        return HSTU_ERR_INVALID_ARG;
    HSTU_TRY(check_attn_desc(&d->attn));
    if (d->attn.fp8_qk || d->attn.debug_checks)  // standalone attention forward only
        return HSTU_ERR_UNSUPPORTED;
    if (d->d_model < 1 || !(d->ln_eps >= 0.f) || !std::isfinite(d->ln_eps) ||
        (d->output_concat != 0 && d->output_concat != 1) || (d->fp8_projections != 0 && d->fp8_projections != 1))
        return HSTU_ERR_INVALID_ARG;
    if (d->fp8_projections && (d->attn.dtype != HSTU_BF16 || d->output_concat || d->d_model % 128))
        return HSTU_ERR_UNSUPPORTED;
    const int F = d->attn.num_heads * d->attn.d_v;
    if (F != 64 && F != 128 && F != 256 && F != 512 && F != 1024)
        return HSTU_ERR_UNSUPPORTED;
    if (d->attn.dtype == HSTU_BF16 && (d->d_model % 32 || F % 32))
        return HSTU_ERR_UNSUPPORTED;
    return HSTU_OK;
}

static int layer_width(const hstu_attn_desc *a) { return a->num_heads * (2 * a->d_v + 2 * a->d_qk); }

// the concatenated output projection reads [U | O | G] straight from its three
// buffers on the tcgen05 GEMM (bf16); the fp32 path copies it first
static bool layer_cat_copy(const hstu_layer_desc *d)
{
    return d->output_concat && d->attn.dtype != HSTU_BF16;
}

static size_t layer_ws(const hstu_layer_desc *d, bool keep_uvqk, bool keep_o)
{
    const hstu_attn_desc *a = &d->attn;
    const size_t eb = elem_bytes(a), T = (size_t)a->total_tokens;
    size_t b = attn_ws(a, 0);
    if (!keep_uvqk)
        b += align256(T * layer_width(a) * eb);
    if (!keep_o)
        b += align256(T * a->num_heads * a->d_v * eb);
    b += align256(T * a->num_heads * a->d_v * eb);  // G
    if (layer_cat_copy(d))
        b += align256(T * 3 * a->num_heads * a->d_v * eb);  // [U | O | G]
    if (d->fp8_projections)  // E4M3 codes and row scales of X and of G
        b += align256(T * d->d_model) + align256(T * 4) + align256(T * a->num_heads * a->d_v) + align256(T * 4);
    return b;
}

hstu_status hstu_layer_workspace_size(const hstu_layer_desc *desc, size_t *bytes)
{
    HSTU_TRY(check_layer_desc(desc));
    if (!bytes)
        return HSTU_ERR_INVALID_ARG;
    *bytes = layer_ws(desc, false, false);
    return HSTU_OK;
}

hstu_status hstu_layer_fwd(const hstu_layer_desc *desc, const void *x, const void *w1, const void *b1,
                           const void *w2, const void *b2, const float *ln_gamma, const float *ln_beta,
                           const int64_t *seq_offsets, const int64_t *timestamps,
                           const int32_t *num_targets, const float *rab_pos, const float *rab_time,
                           void *y, void *saved_uvqk, void *saved_o, void *workspace,
                           size_t workspace_bytes, void *stream)
{
    HSTU_TRY(check_layer_desc(desc));
    const hstu_attn_desc *a = &desc->attn;
    if (!seq_offsets || !rab_pos || !rab_time || !w1 || !w2 || !ln_gamma || !ln_beta)
        return HSTU_ERR_INVALID_ARG;
    if (a->total_tokens > 0 && (!x || !y || !timestamps))
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w1) || !aligned16(w2) || !aligned16(y) || !aligned16(saved_uvqk) ||
        !aligned16(saved_o))
        return HSTU_ERR_INVALID_ARG;
    const size_t need = layer_ws(desc, saved_uvqk != nullptr, saved_o != nullptr);
    HSTU_TRY(check_ws(workspace, workspace_bytes, need));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf16 = a->dtype == HSTU_BF16;
    const size_t eb = elem_bytes(a), T = (size_t)a->total_tokens;
    const int W = layer_width(a), hv = a->num_heads * a->d_v, hq = a->num_heads * a->d_qk;
    const int D = desc->d_model;

    char *cur = static_cast<char *>(workspace) + attn_ws(a, 0);
    char *uvqk = static_cast<char *>(saved_uvqk);
    if (!uvqk) {
        uvqk = cur;
        cur += align256(T * W * eb);
    }
    char *o = static_cast<char *>(saved_o);
    if (!o) {
        o = cur;
        cur += align256(T * hv * eb);
    }
    char *g = cur;

    WsHeader *hdr = static_cast<WsHeader *>(workspace);
    if (desc->fp8_projections) {
        // X and G quantised per row; W1, W2 are E4M3 packs [N][K] + scales
        char *xq = g + align256(T * hv * eb);
        float *sx = reinterpret_cast<float *>(xq + align256(T * D));
        char *gq = reinterpret_cast<char *>(sx) + align256(T * 4);
        float *sg = reinterpret_cast<float *>(gq + align256(T * hv));
        const float *s1 = reinterpret_cast<const float *>(static_cast<const char *>(w1) + align256((size_t)W * D));
        const float *s2 = reinterpret_cast<const float *>(static_cast<const char *>(w2) + align256((size_t)D * hv));
        if (!gemm_e4m3_ok(xq, D, w1, D, uvqk, W, (int64_t)T, W, D) ||
            !gemm_e4m3_ok(gq, hv, w2, hv, y, D, (int64_t)T, D, hv))
            return HSTU_ERR_UNSUPPORTED;
        HSTU_CUDA(launch_quantize_rows_e4m3(x, D, (int64_t)T, D, xq, D, sx, st));
        HSTU_CUDA(launch_gemm_e4m3(xq, D, sx, w1, D, s1, b1, uvqk, W, (int64_t)T, W, D, true, hdr, st));
        HSTU_TRY(attn_fwd_strided(a, uvqk + (size_t)2 * hv * eb, W, uvqk + (size_t)(2 * hv + hq) * eb, W,
                                  uvqk + (size_t)hv * eb, W, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                                  o, hv, workspace, st));
        HSTU_CUDA(launch_norm_gate(true, o, hv, uvqk, W, ln_gamma, ln_beta, desc->ln_eps, g, hv, (int64_t)T, hv, st));
        HSTU_CUDA(launch_quantize_rows_e4m3(g, hv, (int64_t)T, hv, gq, hv, sg, st));
        return cuda_status(launch_gemm_e4m3(gq, hv, sg, w2, hv, s2, b2, y, D, (int64_t)T, D, hv, false, hdr, st));
    }
    // bf16 projections run on the tcgen05 GEMM only: every shape is checked
    // before the first launch.  Y = [U | O | G] W2 + b2 reads its three blocks
    // from their buffers.
    GemmOperands cat_op{};
    cat_op.A = uvqk;
    cat_op.lda = W;
    cat_op.A1 = o;
    cat_op.lda1 = hv;
    cat_op.A2 = g;
    cat_op.lda2 = hv;
    cat_op.a_seg = hv;
    cat_op.B = w2;
    cat_op.ldb = D;
    cat_op.bias = b2;
    cat_op.C = y;
    cat_op.ldc = D;
    if (bf16 && T > 0 &&
        (!gemm_tc_supported(x, D, w1, uvqk, W, (int64_t)T, W, D) ||
         (desc->output_concat ? !gemm_tc_ok(cat_op, (int64_t)T, D, 3 * hv)
                              : !gemm_tc_supported(g, hv, w2, y, D, (int64_t)T, D, hv))))
        return HSTU_ERR_UNSUPPORTED;
    if (bf16)
        HSTU_CUDA(launch_gemm_tc(x, D, w1, b1, uvqk, W, (int64_t)T, W, D, true, hdr, st));
    else
        HSTU_CUDA(launch_gemm_f32(static_cast<const float *>(x), D, static_cast<const float *>(w1),
                                  static_cast<const float *>(b1), reinterpret_cast<float *>(uvqk), W,
                                  (int64_t)T, W, D, true, st));
    HSTU_TRY(attn_fwd_strided(a, uvqk + (size_t)2 * hv * eb, W, uvqk + (size_t)(2 * hv + hq) * eb, W,
                              uvqk + (size_t)hv * eb, W, seq_offsets, timestamps, num_targets,
                              rab_pos, rab_time, o, hv, workspace, st));
    HSTU_CUDA(launch_norm_gate(bf16, o, hv, uvqk, W, ln_gamma, ln_beta, desc->ln_eps, g, hv,
                               (int64_t)T, hv, st));
    if (desc->output_concat) {
        // Y = [U | O | G] W2 + b2
        const int F = 3 * hv;
        if (!layer_cat_copy(desc))
            return cuda_status(launch_gemm_tc_ex(cat_op, (int64_t)T, D, F, GEMM_ACT, false, 1, hdr, st));
        char *cat = g + align256(T * hv * eb);
        HSTU_CUDA(launch_concat3(uvqk, (int64_t)W * eb, o, (int64_t)hv * eb, g, (int64_t)hv * eb, cat,
                                 (int64_t)T, (int64_t)hv * eb, st));
        return cuda_status(launch_gemm_f32(reinterpret_cast<const float *>(cat), F,
                                           static_cast<const float *>(w2), static_cast<const float *>(b2),
                                           static_cast<float *>(y), D, (int64_t)T, D, F, false, st));
    }
    if (bf16)
        return cuda_status(launch_gemm_tc(g, hv, w2, b2, y, D, (int64_t)T, D, hv, false, hdr, st));
    return cuda_status(launch_gemm_f32(reinterpret_cast<const float *>(g), hv,
                                       static_cast<const float *>(w2), static_cast<const float *>(b2),
                                       static_cast<float *>(y), D, (int64_t)T, D, hv, false, st));
}

static size_t layer_bwd_ws(const hstu_layer_desc *d)
{
    const hstu_attn_desc *a = &d->attn;
    const size_t T = (size_t)a->total_tokens, W = layer_width(a), hv = (size_t)a->num_heads * a->d_v;
    const size_t F = (d->output_concat ? 3 : 1) * hv;
    // attention backward scratch, then G [T, H d_v], dcat [T, F], dO [T, H d_v] and dA, dZ [T, W] (bf16)
    return attn_ws(a, 1) + 2 * align256(T * hv * 2) + align256(T * F * 2) + 2 * align256(T * W * 2);
}

static bool layer_bwd_supported(const hstu_layer_desc *d)
{
    const hstu_attn_desc *a = &d->attn;
    const int hv = a->num_heads * a->d_v, W = layer_width(a);
    return a->dtype == HSTU_BF16 && d->d_model % 128 == 0 && hv % 128 == 0 && W % 128 == 0;
}

hstu_status hstu_layer_bwd_workspace_size(const hstu_layer_desc *desc, size_t *bytes)
{
    HSTU_TRY(check_layer_desc(desc));
    if (!bytes)
        return HSTU_ERR_INVALID_ARG;
    *bytes = layer_bwd_ws(desc);
    return HSTU_OK;
}

hstu_status hstu_layer_bwd(const hstu_layer_desc *desc, const void *x, const void *w1, const void *b1,
                           const void *w2, const float *ln_gamma, const float *ln_beta,
                           const int64_t *seq_offsets, const int64_t *timestamps, const int32_t *num_targets,
                           const float *rab_pos, const float *rab_time, const void *saved_uvqk,
                           const void *saved_o, const void *dy, void *dx, float *dw1, float *db1, float *dw2,
                           float *db2, float *d_ln_gamma, float *d_ln_beta, float *d_rab_pos,
                           float *d_rab_time, void *workspace, size_t workspace_bytes, void *stream)
{
    HSTU_TRY(check_layer_desc(desc));
    if (!layer_bwd_supported(desc))
        return HSTU_ERR_UNSUPPORTED;
    const hstu_attn_desc *a = &desc->attn;
    if (!seq_offsets || !rab_pos || !rab_time || !w1 || !w2 || !ln_gamma || !ln_beta || !dw1 || !db1 || !dw2 ||
        !db2 || !d_ln_gamma || !d_ln_beta || !d_rab_pos || !d_rab_time)
        return HSTU_ERR_INVALID_ARG;
    if (a->total_tokens > 0 && (!x || !dx || !dy || !saved_uvqk || !saved_o || !timestamps))
        return HSTU_ERR_INVALID_ARG;
    const void *ptrs[] = {x, w1, b1, w2, saved_uvqk, saved_o, dy, dx, dw1, db1, dw2, db2};
    for (const void *q : ptrs)
        if (!aligned16(q))
            return HSTU_ERR_INVALID_ARG;
    HSTU_TRY(check_ws(workspace, workspace_bytes, layer_bwd_ws(desc)));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t T = a->total_tokens;
    const int W = layer_width(a), hv = a->num_heads * a->d_v, hq = a->num_heads * a->d_qk;
    const int D = desc->d_model;
    const bool cat = desc->output_concat != 0;
    const int F = cat ? 3 * hv : hv;  // width of the output projection's input
    WsHeader *hdr = static_cast<WsHeader *>(workspace);

    HSTU_CUDA(cudaMemsetAsync(dw1, 0, sizeof(float) * (size_t)D * W, st));
    HSTU_CUDA(cudaMemsetAsync(db1, 0, sizeof(float) * W, st));
    HSTU_CUDA(cudaMemsetAsync(dw2, 0, sizeof(float) * (size_t)F * D, st));
    HSTU_CUDA(cudaMemsetAsync(db2, 0, sizeof(float) * D, st));
    HSTU_CUDA(cudaMemsetAsync(d_ln_gamma, 0, sizeof(float) * hv, st));
    HSTU_CUDA(cudaMemsetAsync(d_ln_beta, 0, sizeof(float) * hv, st));
    if (T == 0) {
        return zero_table_grads(a, d_rab_pos, d_rab_time, st);
    }
    char *cur = static_cast<char *>(workspace) + attn_ws(a, 1);
    auto take = [&](size_t bytes) {
        char *p = cur;
        cur += align256(bytes);
        return p;
    };
    char *g = take((size_t)T * hv * 2), *dcat = take((size_t)T * F * 2), *dout = take((size_t)T * hv * 2);
    char *dg = dcat + (size_t)(F - hv) * 2;  // the G block of dcat
    char *da = take((size_t)T * W * 2), *dz = take((size_t)T * W * 2);
    const char *uvqk = static_cast<const char *>(saved_uvqk);
    const int sms = device_info().sms;
    auto splits_for = [&](int64_t M, int N) {
        const int64_t tiles = ((M + 127) / 128) * (N / 128);
        return (int)std::max<int64_t>(1, std::min<int64_t>((2 * sms + tiles - 1) / tiles, (T + 63) / 64));
    };

    // G = LayerNorm(O) U, recomputed from the saved attention output
    HSTU_CUDA(launch_norm_gate(true, saved_o, hv, uvqk, W, ln_gamma, ln_beta, desc->ln_eps, g, hv, T, hv, st));
    // output projection over cat = G or [U | O | G]: dcat = dy W2^T, dW2 = cat^T dy, db2 = sum dy
    GemmOperands op{};
    op.A = dy;
    op.lda = D;
    op.B = w2;
    op.ldb = D;
    op.b_k = true;
    op.C = dcat;
    op.ldc = F;
    if (!gemm_tc_ok(op, T, F, D))
        return HSTU_ERR_UNSUPPORTED;
    HSTU_CUDA(launch_gemm_tc_ex(op, T, F, D, GEMM_ACT, false, 1, hdr, st));
    op = GemmOperands{};
    op.A = g;
    op.lda = hv;
    if (cat) {  // the rows of cat^T come from three buffers
        op.A = uvqk;
        op.lda = W;
        op.A1 = saved_o;
        op.lda1 = hv;
        op.A2 = g;
        op.lda2 = hv;
        op.a_seg = hv;
    }
    op.a_mn = true;
    op.B = dy;
    op.ldb = D;
    op.C32 = dw2;
    op.ldc = D;
    if (!gemm_tc_ok(op, F, D, (int)T))
        return HSTU_ERR_UNSUPPORTED;
    HSTU_CUDA(launch_gemm_tc_ex(op, F, D, (int)T, GEMM_RED_F32, false, splits_for(F, D), hdr, st));
    HSTU_CUDA(launch_colsum_bf16(dy, D, T, D, db2, st));
    // gate: dO and dU (into the U block of dA; plus dcat's U and O blocks), dgamma, dbeta
    HSTU_CUDA(launch_norm_gate_bwd(dg, F, saved_o, hv, uvqk, W, ln_gamma, ln_beta, desc->ln_eps, dout, hv, da, W,
                                   d_ln_gamma, d_ln_beta, T, hv, cat, st));
    // attention: dV, dQ, dK into their blocks of dA, bias-table gradients
    HSTU_TRY(attn_bwd_strided(a, uvqk + (size_t)2 * hv * 2, W, uvqk + (size_t)(2 * hv + hq) * 2, W,
                              uvqk + (size_t)hv * 2, W, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                              dout, hv, da + (size_t)2 * hv * 2, W, da + (size_t)(2 * hv + hq) * 2, W,
                              da + (size_t)hv * 2, W, d_rab_pos, d_rab_time, workspace, st));
    // projection: dZ = dA SiLU'(X W1 + b1) (recomputed in the GEMM), db1, dX = dZ W1^T, dW1 = X^T dZ
    op = GemmOperands{};
    op.A = x;
    op.lda = D;
    op.B = w1;
    op.ldb = W;
    op.bias = b1;
    op.aux = da;
    op.ldaux = W;
    op.C = dz;
    op.ldc = W;
    if (!gemm_tc_ok(op, T, W, D))
        return HSTU_ERR_UNSUPPORTED;
    HSTU_CUDA(launch_gemm_tc_ex(op, T, W, D, GEMM_DSILU, false, 1, hdr, st));
    HSTU_CUDA(launch_colsum_bf16(dz, W, T, W, db1, st));
    op = GemmOperands{};
    op.A = dz;
    op.lda = W;
    op.B = w1;
    op.ldb = W;
    op.b_k = true;
    op.C = dx;
    op.ldc = D;
    if (!gemm_tc_ok(op, T, D, W))
        return HSTU_ERR_UNSUPPORTED;
    HSTU_CUDA(launch_gemm_tc_ex(op, T, D, W, GEMM_ACT, false, 1, hdr, st));
    op = GemmOperands{};
    op.A = x;
    op.lda = D;
    op.a_mn = true;
    op.B = dz;
    op.ldb = W;
    op.C32 = dw1;
    op.ldc = W;
    if (!gemm_tc_ok(op, D, W, (int)T))
        return HSTU_ERR_UNSUPPORTED;
    return cuda_status(launch_gemm_tc_ex(op, D, W, (int)T, GEMM_RED_F32, false, splits_for(D, W), hdr, st));
}

hstu_status hstu_jagged_truncate(int32_t num_seqs, int64_t total_tokens, int32_t keep,
                                 const int64_t *seq_offsets, const int32_t *num_targets, const void *in,
                                 int64_t row_bytes, void *out, int64_t *out_offsets, void *stream)
{
    if (num_seqs < 0 || total_tokens < 0 || keep < 0 || row_bytes <= 0 || row_bytes % 4 != 0 ||
        !seq_offsets || !out_offsets)
        return HSTU_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!in || !out))
        return HSTU_ERR_INVALID_ARG;
    if (num_seqs > kTruncateMaxSeqs)
        return HSTU_ERR_UNSUPPORTED;
    const uintptr_t align = row_bytes % 16 == 0 ? 15u : 3u;
    if ((reinterpret_cast<uintptr_t>(in) & align) || (reinterpret_cast<uintptr_t>(out) & align))
        return HSTU_ERR_INVALID_ARG;
    return cuda_status(launch_jagged_truncate(seq_offsets, num_targets, num_seqs, total_tokens, keep, row_bytes,
                                              in, out, out_offsets, static_cast<cudaStream_t>(stream)));
}

size_t hstu_e4m3_weight_bytes(int32_t K, int32_t N)
{
    if (K < 0 || N < 0)
        return 0;
    return align256((size_t)K * N) + (size_t)N * 4;
}

hstu_status hstu_quantize_weight_e4m3(const void *w, int32_t K, int32_t N, void *pack, void *stream)
{
    if (K <= 0 || N <= 0 || K % 16 || !w || !pack || !aligned16(w) || !aligned16(pack))
        return HSTU_ERR_INVALID_ARG;
    float *scales = reinterpret_cast<float *>(static_cast<char *>(pack) + align256((size_t)K * N));
    return cuda_status(launch_quantize_cols_e4m3(w, K, N, pack, scales, static_cast<cudaStream_t>(stream)));
}

hstu_status hstu_quantize_rows_e4m3(const void *x, int64_t rows, int32_t K, void *codes, float *scales,
                                    void *stream)
{
    if (rows < 0 || K <= 0 || K % 16)
        return HSTU_ERR_INVALID_ARG;
    if (rows > 0 && (!x || !codes || !scales || !aligned16(x) || !aligned16(codes)))
        return HSTU_ERR_INVALID_ARG;
    return cuda_status(launch_quantize_rows_e4m3(x, K, rows, K, codes, K, scales, static_cast<cudaStream_t>(stream)));
}

hstu_status hstu_gemm_e4m3(const void *codes, const float *scales, int64_t M, int32_t K, const void *wpack,
                           int32_t N, const void *bias, int32_t apply_silu, void *y, void *workspace,
                           size_t workspace_bytes, void *stream)
{
    if (M < 0 || K <= 0 || N <= 0 || !wpack)
        return HSTU_ERR_INVALID_ARG;
    HSTU_TRY(check_ws(workspace, workspace_bytes, sizeof(WsHeader)));
    if (M == 0)
        return HSTU_OK;
    if (!codes || !scales || !y)
        return HSTU_ERR_INVALID_ARG;
    if (!gemm_e4m3_ok(codes, K, wpack, K, y, N, M, N, K))
        return (aligned16(codes) && aligned16(wpack) && aligned16(y)) ? HSTU_ERR_UNSUPPORTED : HSTU_ERR_INVALID_ARG;
    const float *ws = reinterpret_cast<const float *>(static_cast<const char *>(wpack) + align256((size_t)K * N));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    HSTU_CUDA(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st));
    return cuda_status(launch_gemm_e4m3(codes, K, scales, wpack, K, ws, bias, y, N, M, N, K, apply_silu != 0,
                                        static_cast<WsHeader *>(workspace), st));
}

hstu_status hstu_check_device_flag(const void *workspace, int32_t *bits, void *stream)
{
    if (!workspace)
        return HSTU_ERR_WORKSPACE;
    int32_t flag = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    HSTU_CUDA(cudaMemcpyAsync(&flag, workspace, sizeof(flag), cudaMemcpyDeviceToHost, st));
    HSTU_CUDA(cudaStreamSynchronize(st));
    if (bits)
        *bits = flag;
    return flag ? HSTU_ERR_DEVICE_CHECK : HSTU_OK;
}

hstu_status hstu_debug_bias_indices(const hstu_attn_desc *desc, const int64_t *seq_offsets,
                                    const int64_t *timestamps, const int32_t *num_targets,
                                    const int64_t *rows, int64_t n, int32_t *pos_index,
                                    int32_t *bucket, void *stream)
{
    HSTU_TRY(check_attn_desc(desc));
    if (n < 0 || (n > 0 && (!seq_offsets || !timestamps || !rows || !pos_index || !bucket)))
        return HSTU_ERR_INVALID_ARG;
    return cuda_status(launch_debug_indices(seq_offsets, timestamps, num_targets, desc->num_seqs,
                                            desc->pos_lo, desc->pos_hi, desc->num_time_buckets,
                                            desc->cand_positions != 0, rows, n, pos_index, bucket,
                                            static_cast<cudaStream_t>(stream)));
}

hstu_status hstu_debug_schedule(const hstu_attn_desc *desc, const int64_t *seq_offsets,
                                const int32_t *num_targets, int is_bwd, int32_t tile_rows,
                                int32_t *items, int32_t max_items_cap, int32_t *count, int32_t *flag,
                                void *stream)
{
    HSTU_TRY(check_attn_desc(desc));
    if (!seq_offsets || !items || !count || !flag || tile_rows < 1)
        return HSTU_ERR_INVALID_ARG;
    if (max_items_cap < max_items(desc->total_tokens, desc->num_seqs, tile_rows))
        return HSTU_ERR_WORKSPACE;
    // the header lives in caller memory: `flag` must point at 256 writable bytes
    return cuda_status(launch_schedule(seq_offsets, num_targets, desc->num_seqs, desc->total_tokens,
                                       desc->max_seq_len, tile_rows, is_bwd,
                                       reinterpret_cast<int2 *>(items), max_items_cap,
                                       reinterpret_cast<WsHeader *>(flag), count,
                                       static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
