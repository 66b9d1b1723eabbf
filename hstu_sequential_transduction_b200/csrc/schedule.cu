// Jagged tile scheduler.
//
// The HSTU attention is evaluated only on the lower triangle of each
// sequence's (query, key) grid ("DLRMv4 Brings Sequence-Based Recommendation
// Training to MLPerf", text under Table 7).  The scheduler turns seq_offsets
// (and num_targets) into a list of (sequence, tile) work items, longest first
// (an LPT order), without any host synchronization:
//   forward:  item (b, qt) owns query rows [qt*tile, (qt+1)*tile) of sequence
//             b and walks the key tiles that row block can see; its cost is
//             about qt + 1 key tiles;
//   backward: item (b, kt) owns key rows of tile kt and walks the query tiles
//             that see it; its cost is about ntiles_b - kt.
// Items are grouped by "level" l (cost l + 1 tiles) in descending order and,
// inside a level, by sequence index.  One CTA per level computes its start
// offset (the number of items on higher levels) and compacts its sequences
// with a block scan, so the list is deterministic.
//
// Sequences whose offsets or targets are inconsistent are dropped (they get
// no items) and recorded in the workspace flag; nothing is read out of range.
#include "common.cuh"
#include "internal.h"

namespace hstu {

namespace {

constexpr int kSchedThreads = 256;

struct SeqCheck {
    int ntiles;  // 0 for empty or dropped sequences
    int bits;    // flag bits raised by this sequence
};

__device__ __forceinline__ SeqCheck check_seq(const int64_t *off, const int32_t *nt, int b,
                                              int64_t T, int max_len, int tile)
{
    SeqCheck c{0, 0};
    int64_t s0 = off[b], s1 = off[b + 1];
    if (s0 < 0 || s1 < s0 || s1 > T) {
        c.bits |= FLAG_SEQ_RANGE;
        return c;
    }
    int64_t L = s1 - s0;
    if (L > (int64_t)max_len) {
        c.bits |= FLAG_SEQ_TOO_LONG;
        return c;
    }
    if (nt) {
        int n = nt[b];
        if (n < 0 || (int64_t)n > L) {
            c.bits |= FLAG_TARGETS;
            return c;
        }
    }
    c.ntiles = (int)((L + tile - 1) / tile);
    return c;
}

// Exclusive scan of one int per thread across the block; returns the total.
__device__ int block_exclusive_scan(int v, int *excl, int *warp_sums)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o)
            x += y;
    }
    if (lane == 31)
        warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < (kSchedThreads / 32) ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o)
                w += y;
        }
        if (lane < kSchedThreads / 32)
            warp_sums[lane] = w;  // inclusive per-warp prefix
    }
    __syncthreads();
    int before = warp ? warp_sums[warp - 1] : 0;
    int total = warp_sums[kSchedThreads / 32 - 1];
    *excl = before + x - v;
    __syncthreads();
    return total;
}

__device__ int block_sum(int v, int *warp_sums)
{
    int ex;
    return block_exclusive_scan(v, &ex, warp_sums);
}

__global__ void __launch_bounds__(kSchedThreads)
schedule_kernel(const int64_t *__restrict__ off, const int32_t *__restrict__ nt, int B, int64_t T,
                int max_len, int tile, int is_bwd, int2 *__restrict__ items, int capacity,
                WsHeader *__restrict__ hdr, int32_t *__restrict__ count_out)
{
    __shared__ int warp_sums[kSchedThreads / 32];
    const int level = blockIdx.x;

    // items on higher levels: sum_b max(0, ntiles_b - level - 1)
    int part = 0, bits = 0;
    for (int b = threadIdx.x; b < B; b += kSchedThreads) {
        SeqCheck c = check_seq(off, nt, b, T, max_len, tile);
        part += max(0, c.ntiles - level - 1);
        bits |= c.bits;
    }
    int start = block_sum(part, warp_sums);

    if (level == 0) {
        // flag bits of this call, written by the level-0 block only
        __shared__ int sbits;
        if (threadIdx.x == 0)
            sbits = 0;
        __syncthreads();
        if (bits)
            atomicOr(&sbits, bits);
        __syncthreads();
        if (threadIdx.x == 0) {
            int f = sbits;
            if (off[0] != 0)
                f |= FLAG_OFFSET0;
            if (off[B] != T)
                f |= FLAG_TOTAL;
            hdr->flag = f;
            hdr->cursor = 0;
        }
    }

    // compact the sequences present on this level, in sequence order
    int running = start;
    for (int base = 0; base < B; base += kSchedThreads) {
        int b = base + threadIdx.x;
        int present = 0, ntl = 0;
        if (b < B) {
            ntl = check_seq(off, nt, b, T, max_len, tile).ntiles;
            present = ntl > level;
        }
        int ex;
        int total = block_exclusive_scan(present, &ex, warp_sums);
        if (present) {
            int pos = running + ex;
            if (pos < capacity)
                items[pos] = make_int2(b, is_bwd ? (ntl - 1 - level) : level);
        }
        running += total;
    }
    if (level == 0 && threadIdx.x == 0) {
        int n = min(running, capacity);
        hdr->n_items = n;
        if (count_out)
            *count_out = n;
    }
}

__global__ void debug_indices_kernel(const int64_t *__restrict__ off, const int64_t *__restrict__ ts,
                                     const int32_t *__restrict__ nt, int B, int lo, int hi, int nb, bool own,
                                     const int64_t *__restrict__ rows, int64_t n,
                                     int32_t *__restrict__ pos_out, int32_t *__restrict__ bkt_out)
{
    int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= n)
        return;
    int64_t gi = rows[2 * e], gj = rows[2 * e + 1];
    if (B <= 0) {
        pos_out[e] = -1;
        bkt_out[e] = -1;
        return;
    }
    // sequence of gi by binary search over the non-decreasing offsets
    int a = 0, z = B;  // find largest b with off[b] <= gi
    while (z - a > 1) {
        int m = (a + z) / 2;
        if (off[m] <= gi)
            a = m;
        else
            z = m;
    }
    int b = a;
    int64_t s0 = off[b], s1 = off[b + 1];
    if (gi < s0 || gi >= s1 || gj < s0 || gj >= s1) {
        pos_out[e] = -1;
        bkt_out[e] = -1;
        return;
    }
    int L = (int)(s1 - s0);
    int hist = L - (nt ? nt[b] : 0);
    int i = (int)(gi - s0), j = (int)(gj - s0);
    pos_out[e] = pos_index(token_pos(i, hist, own), token_pos(j, hist, own), lo, hi);
    bkt_out[e] = time_bucket(ts[gi], ts[gj], nb);
}

}  // namespace

cudaError_t launch_schedule(const int64_t *off, const int32_t *nt, int B, int64_t T, int max_len,
                            int tile, int is_bwd, int2 *items, int capacity, WsHeader *hdr,
                            int32_t *count_out, cudaStream_t stream)
{
    int levels = max(1, ceil_div(max(max_len, 1), tile));
    schedule_kernel<<<levels, kSchedThreads, 0, stream>>>(off, nt, B, T, max_len, tile, is_bwd,
                                                          items, capacity, hdr, count_out);
    return cudaGetLastError();
}

cudaError_t launch_debug_indices(const int64_t *off, const int64_t *ts, const int32_t *nt, int B,
                                 int lo, int hi, int nb, bool own, const int64_t *rows, int64_t n,
                                 int32_t *pos_out, int32_t *bkt_out, cudaStream_t stream)
{
    if (n == 0)
        return cudaSuccess;
    int threads = 256;
    int64_t blocks = (n + threads - 1) / threads;
    debug_indices_kernel<<<(unsigned)blocks, threads, 0, stream>>>(off, ts, nt, B, lo, hi, nb, own, rows,
                                                                   n, pos_out, bkt_out);
    return cudaGetLastError();
}

}  // namespace hstu
