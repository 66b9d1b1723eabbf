// Shared device helpers for the HSTU kernels (sm_100a).
//
// The index functions here are the single definition every kernel and the
// debug entry use for the relative-bias gathers of the HSTU attention
// ("DLRMv4 Brings Sequence-Based Recommendation Training to MLPerf", section
// "Model Architecture": a bias from positional and temporal distance).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu.h"

namespace hstu {

// Workspace header (first 256 bytes of every attention workspace).
struct WsHeader {
    int flag;      // device input-check bits of the last call
    int n_items;   // work items written by the scheduler
    int cursor;    // work-stealing counter of persistent kernels
    int pad[61];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

enum : int {
    FLAG_OFFSET0 = 1,
    FLAG_SEQ_RANGE = 2,
    FLAG_SEQ_TOO_LONG = 4,
    FLAG_TARGETS = 8,
    FLAG_TOTAL = 16,
};

// A pipeline wait that runs out records FLAG_TIMEOUT in the header's flag.
enum : int { FLAG_TIMEOUT = 32 };
constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at 2 GHz
// the limit under the bounded-wait test hook (HSTU_DEBUG_WAIT_TEST): ~1 ms, far
// above any wait of a working pipeline (a few tile times), short for a test
constexpr long long kTestWaitLimitCycles = 2000000LL;

// Everything an attention kernel reads; strides are in elements between rows.
struct AttnParams {
    const void *q, *k, *v;
    void *o;
    int64_t sq, sk, sv, so;
    const int64_t *seq_offsets;
    const int64_t *timestamps;
    const int32_t *num_targets;
    const float *rab_pos, *rab_time;
    int B, H, dqk, dv, max_seq_len;
    int64_t T;
    float inv_n;
    int pos_lo, pos_hi, nb;
    int lw, gw;  // semi-local windows (lw = 0: full mask)
    // FP8 scores (forward): E4M3 codes of q and k, [T, H, d] bytes, and their
    // per-(token, head) scales [T, H]; null for bf16 scores
    const void *q8, *k8;
    const float *sq8, *sk8;
    const int2 *items;
    WsHeader *hdr;
    // clock cycles after which a pipeline wait gives up (FLAG_TIMEOUT), and the
    // test hook of the bounded waits: the forward's first CTA withholds the load
    // of its first key tile
    long long wait_limit;
    int withhold_first_k;
    // backward only
    const void *dout;
    int64_t sdo;
    void *dq, *dk, *dvv;
    int64_t sdq, sdk, sdv;
    float *dq_acc;  // fp32 [T, H, dqk] accumulator (bf16 mode)
    float *d_rab_pos, *d_rab_time;
    int cand_own;  // candidates at their own index (else at the slot after the history)
    // head strides of the bias tables and their gradients: 0 when the heads share
    // one pair of tables, the table sizes when each head has its own
    int64_t pos_hstride, time_hstride;
};

// floor(log2(1 + max(dt, 0))) capped at nb - 1, exact on int64 seconds.
__device__ __forceinline__ int time_bucket(int64_t t_i, int64_t t_j, int nb)
{
    int64_t dt = t_i - t_j;
    dt = dt < 0 ? 0 : dt;
    int b = 63 - __clzll((long long)(dt + 1));
    return b < nb - 1 ? b : nb - 1;
}

__device__ __forceinline__ int pos_index(int p_i, int p_j, int lo, int hi)
{
    int d = p_i - p_j;
    d = d < lo ? lo : (d > hi ? hi : d);
    return d - lo;
}

// Local position of token i: candidates share the slot after the history, or
// (own) keep their own index.
__device__ __forceinline__ int token_pos(int i, int hist, bool own) { return (i < hist || own) ? i : hist; }

__device__ __forceinline__ bool visible(int i, int j, int hist)
{
    return i < hist ? (j <= i) : (j < hist || j == i);
}

// visible() restricted to the semi-local windows: with lw > 0 the query must
// be fewer than lw positions after the key, or the key among the first gw
// tokens of the sequence.
__device__ __forceinline__ bool visible_w(int i, int j, int hist, int lw, int gw, bool own)
{
    return visible(i, j, hist) && (lw <= 0 || token_pos(i, hist, own) - token_pos(j, hist, own) < lw || j < gw);
}

// SiLU and its derivative on the fp32 path (IEEE division, expf).
__device__ __forceinline__ float silu_precise(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ float silu_grad_precise(float x)
{
    float s = 1.0f / (1.0f + expf(-x));
    return s * (1.0f + x * (1.0f - s));
}

// ---- shared-memory addresses and bf16 packing -------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---- host helpers -----------------------------------------------------------

inline int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

// Upper bound on the work items of a schedule with tiles of `tile` rows.
inline int64_t max_items(int64_t T, int B, int tile) { return (T + tile - 1) / tile + B; }

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace hstu
