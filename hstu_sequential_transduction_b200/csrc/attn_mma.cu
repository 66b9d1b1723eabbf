// HSTU jagged attention, bf16 on the legacy warp-level tensor-core path
// (mma.sync m16n8k16, fp32 accumulate).  This is the correctness baseline the
// tcgen05 kernels are measured against; it is also the fallback for head dims
// the tcgen05 kernels do not take.
//
// Forward, per work item (sequence b, 64-row query tile) and head:
//   for each visible 64-row key tile:  S = Q K^T (registers),
//   P = SiLU(S + rab_pos + rab_time) * inv_n on visible pairs (the pointwise
//   attention of the "HSTU Architecture" section: no softmax, no running max),
//   O += P V with P kept in registers as the A operand.  No score matrix
//   touches global memory.
// Backward, per (sequence, 64-row key tile) and head (key-stationary):
//   recompute S and P for every query tile that sees the key tile,
//   dV += P^T dO;  dP^T = V dO^T;  dS = dP * SiLU'(S) * inv_n;
//   dK += dS^T Q;  dQ += dS K (fp32 atomics into an accumulator);
//   the bias-table gradients collect dS per positional index and time bucket
//   in shared memory and are flushed with one global atomic per touched bin.
#include "common.cuh"
#include "internal.h"

namespace hstu {

namespace {

constexpr int BM = 64;        // query rows per tile
constexpr int BN = 64;        // key rows per tile
constexpr int kThreads = 128; // 4 warps, 16 query rows each
// bias tables go to shared memory when they are at most this many floats
constexpr int kSmemTableMax = 2560;

template <int D>
struct Tiles {
    static constexpr int LD = D + 8;                 // padded row, bf16 elements
    static constexpr int TILE = BM * LD;             // elements per tile
    static constexpr size_t bytes = 5 * TILE * 2 + 2 * BN * sizeof(int64_t);
};

struct SeqView {
    int64_t s0;
    int L, hist;
};

__device__ __forceinline__ SeqView seq_view(const AttnParams &p, int b)
{
    SeqView s;
    s.s0 = p.seq_offsets[b];
    s.L = (int)(p.seq_offsets[b + 1] - s.s0);
    s.hist = s.L - (p.num_targets ? p.num_targets[b] : 0);
    return s;
}

// Copy rows [r0, r0 + 64) of a jagged [T, H, D] bf16 tensor (head h) into a
// padded shared tile; rows at or past L are zero-filled.
template <int D>
__device__ __forceinline__ void load_tile(__nv_bfloat16 *dst, const __nv_bfloat16 *src,
                                          int64_t stride, const SeqView &s, int r0, int h)
{
    constexpr int CH = D / 8;
    for (int c = threadIdx.x; c < BM * CH; c += kThreads) {
        int r = c / CH, ch = c % CH;
        bool ok = r0 + r < s.L;
        const __nv_bfloat16 *g = ok ? src + (s.s0 + r0 + r) * stride + (int64_t)h * D + ch * 8 : src;
        cp_async16(dst + r * Tiles<D>::LD + ch * 8, g, ok ? 16 : 0);
    }
}

__device__ __forceinline__ void load_ts(int64_t *dst, const int64_t *ts, const SeqView &s, int r0)
{
    if (threadIdx.x < BN) {
        int r = r0 + threadIdx.x;
        dst[threadIdx.x] = r < s.L ? ts[s.s0 + r] : 0;
    }
}

// Key tiles seen by query tile qt: every tile holding history keys up to
// the tile itself, plus the diagonal tile for candidate-only query tiles.
__device__ __forceinline__ int fwd_num_tiles(int qt, const SeqView &s)
{
    int nh = (s.hist + BN - 1) / BN;
    int n = min(qt + 1, nh);
    return n + (qt >= nh ? 1 : 0);
}

__device__ __forceinline__ int fwd_tile(int idx, int qt, const SeqView &s)
{
    int nh = (s.hist + BN - 1) / BN;
    return idx < min(qt + 1, nh) ? idx : qt;
}

template <int D>
__global__ void __launch_bounds__(kThreads)
attn_fwd_mma_kernel(const AttnParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    using TL = Tiles<D>;
    __nv_bfloat16 *sQ = reinterpret_cast<__nv_bfloat16 *>(smem);
    __nv_bfloat16 *sK = sQ + TL::TILE;      // 2 buffers
    __nv_bfloat16 *sV = sK + 2 * TL::TILE;  // 2 buffers
    int64_t *sT = reinterpret_cast<int64_t *>(sV + 2 * TL::TILE);  // 2 x BN
    float *sTab = reinterpret_cast<float *>(sT + 2 * BN);

    const int item = blockIdx.x / p.H, h = blockIdx.x % p.H;
    if (item >= p.hdr->n_items)
        return;
    const int2 it = p.items[item];
    const SeqView s = seq_view(p, it.x);
    const int qt = it.y, i0 = qt * BM;

    const int npos = p.pos_hi - p.pos_lo + 1;
    const bool tab_in_smem = npos + p.nb <= kSmemTableMax;
    const float *tpos = p.rab_pos, *ttime = p.rab_time;
    if (tab_in_smem) {
        for (int e = threadIdx.x; e < npos; e += kThreads)
            sTab[e] = p.rab_pos[e];
        for (int e = threadIdx.x; e < p.nb; e += kThreads)
            sTab[npos + e] = p.rab_time[e];
        tpos = sTab;
        ttime = sTab + npos;
    }

    const __nv_bfloat16 *gq = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *gk = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *gv = static_cast<const __nv_bfloat16 *>(p.v);
    const int ntiles = fwd_num_tiles(qt, s);

    load_tile<D>(sQ, gq, p.sq, s, i0, h);
    load_tile<D>(sK, gk, p.sk, s, fwd_tile(0, qt, s) * BN, h);
    load_tile<D>(sV, gv, p.sv, s, fwd_tile(0, qt, s) * BN, h);
    cp_async_commit();
    load_ts(sT, p.timestamps, s, fwd_tile(0, qt, s) * BN);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    // the two query rows this thread owns
    int ri[2] = {i0 + warp * 16 + g, i0 + warp * 16 + g + 8};
    int pi[2];
    int64_t ti[2];
#pragma unroll
    for (int a = 0; a < 2; a++) {
        pi[a] = token_pos(ri[a], s.hist);
        ti[a] = ri[a] < s.L ? p.timestamps[s.s0 + ri[a]] : 0;
    }

    float oacc[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; n++)
#pragma unroll
        for (int e = 0; e < 4; e++)
            oacc[n][e] = 0.f;
    uint32_t qf[D / 16][4];

    for (int idx = 0; idx < ntiles; idx++) {
        const int buf = idx & 1;
        if (idx + 1 < ntiles) {
            const int r0 = fwd_tile(idx + 1, qt, s) * BN;
            load_tile<D>(sK + (buf ^ 1) * TL::TILE, gk, p.sk, s, r0, h);
            load_tile<D>(sV + (buf ^ 1) * TL::TILE, gv, p.sv, s, r0, h);
            cp_async_commit();
            load_ts(sT + (buf ^ 1) * BN, p.timestamps, s, r0);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (idx == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; kk++) {
                const int m = lane >> 3;
                const __nv_bfloat16 *a =
                    sQ + (warp * 16 + (lane & 7) + 8 * (m & 1)) * TL::LD + kk * 16 + 8 * (m >> 1);
                ldmatrix_x4(qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], a);
            }
        }
        const __nv_bfloat16 *cK = sK + buf * TL::TILE;
        const __nv_bfloat16 *cV = sV + buf * TL::TILE;
        const int64_t *cT = sT + buf * BN;
        const int j0 = fwd_tile(idx, qt, s) * BN;

        float sacc[BN / 8][4];
#pragma unroll
        for (int n = 0; n < BN / 8; n++)
#pragma unroll
            for (int e = 0; e < 4; e++)
                sacc[n][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; kk++) {
#pragma unroll
            for (int np = 0; np < BN / 16; np++) {
                const int m = lane >> 3;
                const __nv_bfloat16 *b =
                    cK + (np * 16 + (lane & 7) + 8 * (m >> 1)) * TL::LD + kk * 16 + 8 * (m & 1);
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4(r0, r1, r2, r3, b);
                mma_bf16_16816(sacc[2 * np], qf[kk], r0, r1);
                mma_bf16_16816(sacc[2 * np + 1], qf[kk], r2, r3);
            }
        }
        // score epilogue: bias gather, mask, SiLU, 1/N
#pragma unroll
        for (int n = 0; n < BN / 8; n++) {
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int a = e >> 1;
                const int c = n * 8 + 2 * t4 + (e & 1);
                const int j = j0 + c;
                const bool vis = ri[a] < s.L && j < s.L && visible_w(ri[a], j, s.hist, p.lw, p.gw);
                float x = sacc[n][e] + tpos[pos_index(pi[a], token_pos(j, s.hist), p.pos_lo, p.pos_hi)] +
                          ttime[time_bucket(ti[a], cT[c], p.nb)];
                sacc[n][e] = vis ? silu_fast(x) * p.inv_n : 0.f;
            }
        }
        // O += P V, P from registers
#pragma unroll
        for (int kk = 0; kk < BN / 16; kk++) {
            uint32_t af[4];
            af[0] = pack_bf16(sacc[2 * kk][0], sacc[2 * kk][1]);
            af[1] = pack_bf16(sacc[2 * kk][2], sacc[2 * kk][3]);
            af[2] = pack_bf16(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
            af[3] = pack_bf16(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
#pragma unroll
            for (int np = 0; np < D / 16; np++) {
                const int m = lane >> 3;
                const __nv_bfloat16 *b =
                    cV + (kk * 16 + (lane & 7) + 8 * (m & 1)) * TL::LD + np * 16 + 8 * (m >> 1);
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(r0, r1, r2, r3, b);
                mma_bf16_16816(oacc[2 * np], af, r0, r1);
                mma_bf16_16816(oacc[2 * np + 1], af, r2, r3);
            }
        }
        __syncthreads();
    }

    __nv_bfloat16 *go = static_cast<__nv_bfloat16 *>(p.o);
#pragma unroll
    for (int a = 0; a < 2; a++) {
        if (ri[a] >= s.L)
            continue;
        __nv_bfloat16 *row = go + (s.s0 + ri[a]) * p.so + (int64_t)h * D;
#pragma unroll
        for (int n = 0; n < D / 8; n++) {
            *reinterpret_cast<uint32_t *>(row + n * 8 + 2 * t4) =
                pack_bf16(oacc[n][2 * a], oacc[n][2 * a + 1]);
        }
    }
}

// ---------------------------------------------------------------------------
// Backward (key-stationary).  Query tiles are 32 rows here.
constexpr int BQ = 32;
// bias-gradient bins live in shared memory when they fit
constexpr int kSmemBinMax = 10240;

template <int D>
struct BwdTiles {
    static constexpr int LD = D + 8;
    static constexpr int KT = BN * LD;   // key/value tile elements
    static constexpr int QT = BQ * LD;   // query/dout tile elements
    static constexpr int LDS = BQ + 8;   // dS^T row (bf16)
    static constexpr size_t bytes =
        (2 * KT + 4 * QT + BN * LDS) * 2 + 2 * BQ * sizeof(int64_t);
};

template <int D>
__device__ __forceinline__ void load_rows(__nv_bfloat16 *dst, int ld, const __nv_bfloat16 *src,
                                          int64_t stride, const SeqView &s, int r0, int rows, int h)
{
    constexpr int CH = D / 8;
    for (int c = threadIdx.x; c < rows * CH; c += kThreads) {
        int r = c / CH, ch = c % CH;
        bool ok = r0 + r < s.L;
        const __nv_bfloat16 *g = ok ? src + (s.s0 + r0 + r) * stride + (int64_t)h * D + ch * 8 : src;
        cp_async16(dst + r * ld + ch * 8, g, ok ? 16 : 0);
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads)
attn_bwd_mma_kernel(const AttnParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    using TL = BwdTiles<D>;
    __nv_bfloat16 *sK = reinterpret_cast<__nv_bfloat16 *>(smem);
    __nv_bfloat16 *sV = sK + TL::KT;
    __nv_bfloat16 *sQ = sV + TL::KT;       // 2 buffers
    __nv_bfloat16 *sO = sQ + 2 * TL::QT;   // dO, 2 buffers
    __nv_bfloat16 *sS = sO + 2 * TL::QT;   // dS^T [BN][LDS]
    int64_t *sTq = reinterpret_cast<int64_t *>(sS + BN * TL::LDS);  // 2 x BQ
    float *sBin = reinterpret_cast<float *>(sTq + 2 * BQ);

    const int item = blockIdx.x / p.H, h = blockIdx.x % p.H;
    if (item >= p.hdr->n_items)
        return;
    const int2 it = p.items[item];
    const SeqView s = seq_view(p, it.x);
    const int kt = it.y, j0 = kt * BN;
    const int npos = p.pos_hi - p.pos_lo + 1;
    const bool bins_in_smem = npos + p.nb <= kSmemBinMax;
    float *bpos = p.d_rab_pos, *btime = p.d_rab_time;
    const float *tpos = p.rab_pos, *ttime = p.rab_time;
    if (bins_in_smem) {
        for (int e = threadIdx.x; e < npos + p.nb; e += kThreads)
            sBin[e] = 0.f;
        bpos = sBin;
        btime = sBin + npos;
    }

    // query rows that see this key tile
    const int q_begin = j0;
    const int q_end = j0 < s.hist ? s.L : min(j0 + BN, s.L);
    const int nq = (q_end - q_begin + BQ - 1) / BQ;

    const __nv_bfloat16 *gq = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *gk = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *gv = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *gdo = static_cast<const __nv_bfloat16 *>(p.dout);

    load_rows<D>(sK, TL::LD, gk, p.sk, s, j0, BN, h);
    load_rows<D>(sV, TL::LD, gv, p.sv, s, j0, BN, h);
    load_rows<D>(sQ, TL::LD, gq, p.sq, s, q_begin, BQ, h);
    load_rows<D>(sO, TL::LD, gdo, p.sdo, s, q_begin, BQ, h);
    cp_async_commit();
    if (threadIdx.x < BQ) {
        int r = q_begin + threadIdx.x;
        sTq[threadIdx.x] = r < s.L ? p.timestamps[s.s0 + r] : 0;
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3, m = lane >> 3;
    // the two key rows this thread owns in the S^T fragments
    int rj[2] = {j0 + warp * 16 + g, j0 + warp * 16 + g + 8};
    int pj[2];
    int64_t tj[2];
#pragma unroll
    for (int a = 0; a < 2; a++) {
        pj[a] = token_pos(rj[a], s.hist);
        tj[a] = rj[a] < s.L ? p.timestamps[s.s0 + rj[a]] : 0;
    }

    float dkacc[D / 8][4], dvacc[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; n++)
#pragma unroll
        for (int e = 0; e < 4; e++) {
            dkacc[n][e] = 0.f;
            dvacc[n][e] = 0.f;
        }

    for (int iq = 0; iq < nq; iq++) {
        const int buf = iq & 1;
        const int i0 = q_begin + iq * BQ;
        if (iq + 1 < nq) {
            load_rows<D>(sQ + (buf ^ 1) * TL::QT, TL::LD, gq, p.sq, s, i0 + BQ, BQ, h);
            load_rows<D>(sO + (buf ^ 1) * TL::QT, TL::LD, gdo, p.sdo, s, i0 + BQ, BQ, h);
            cp_async_commit();
            if (threadIdx.x < BQ) {
                int r = i0 + BQ + threadIdx.x;
                sTq[(buf ^ 1) * BQ + threadIdx.x] = r < s.L ? p.timestamps[s.s0 + r] : 0;
            }
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const __nv_bfloat16 *cQ = sQ + buf * TL::QT;
        const __nv_bfloat16 *cO = sO + buf * TL::QT;
        const int64_t *cT = sTq + buf * BQ;

        // S^T = K Q^T and dP^T = V dO^T for this warp's 16 key rows
        float sacc[BQ / 8][4], pacc[BQ / 8][4];
#pragma unroll
        for (int n = 0; n < BQ / 8; n++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                sacc[n][e] = 0.f;
                pacc[n][e] = 0.f;
            }
#pragma unroll
        for (int kk = 0; kk < D / 16; kk++) {
            uint32_t ka[4], va[4];
            const int arow = (warp * 16 + (lane & 7) + 8 * (m & 1)) * TL::LD + kk * 16 + 8 * (m >> 1);
            ldmatrix_x4(ka[0], ka[1], ka[2], ka[3], sK + arow);
            ldmatrix_x4(va[0], va[1], va[2], va[3], sV + arow);
#pragma unroll
            for (int np = 0; np < BQ / 16; np++) {
                const int brow = (np * 16 + (lane & 7) + 8 * (m >> 1)) * TL::LD + kk * 16 + 8 * (m & 1);
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4(r0, r1, r2, r3, cQ + brow);
                mma_bf16_16816(sacc[2 * np], ka, r0, r1);
                mma_bf16_16816(sacc[2 * np + 1], ka, r2, r3);
                ldmatrix_x4(r0, r1, r2, r3, cO + brow);
                mma_bf16_16816(pacc[2 * np], va, r0, r1);
                mma_bf16_16816(pacc[2 * np + 1], va, r2, r3);
            }
        }
        // elementwise: P, dS, bias-table gradients
#pragma unroll
        for (int n = 0; n < BQ / 8; n++) {
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int a = e >> 1;
                const int c = n * 8 + 2 * t4 + (e & 1);
                const int i = i0 + c;
                const bool vis = i < s.L && rj[a] < s.L && visible_w(i, rj[a], s.hist, p.lw, p.gw);
                const int pidx = pos_index(token_pos(i, s.hist), pj[a], p.pos_lo, p.pos_hi);
                const int bkt = time_bucket(cT[c], tj[a], p.nb);
                float x = sacc[n][e] + tpos[pidx] + ttime[bkt];
                float sg = 1.0f / (1.0f + __expf(-x));
                float pv = vis ? x * sg * p.inv_n : 0.f;
                float ds = vis ? pacc[n][e] * sg * (1.0f + x * (1.0f - sg)) * p.inv_n : 0.f;
                sacc[n][e] = pv;
                pacc[n][e] = ds;
                if (vis) {
                    atomicAdd(bpos + pidx, ds);
                    atomicAdd(btime + bkt, ds);
                }
            }
        }
        // dV += P^T dO ; dK += dS^T Q
#pragma unroll
        for (int kk = 0; kk < BQ / 16; kk++) {
            uint32_t pa[4], sa[4];
            pa[0] = pack_bf16(sacc[2 * kk][0], sacc[2 * kk][1]);
            pa[1] = pack_bf16(sacc[2 * kk][2], sacc[2 * kk][3]);
            pa[2] = pack_bf16(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
            pa[3] = pack_bf16(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
            sa[0] = pack_bf16(pacc[2 * kk][0], pacc[2 * kk][1]);
            sa[1] = pack_bf16(pacc[2 * kk][2], pacc[2 * kk][3]);
            sa[2] = pack_bf16(pacc[2 * kk + 1][0], pacc[2 * kk + 1][1]);
            sa[3] = pack_bf16(pacc[2 * kk + 1][2], pacc[2 * kk + 1][3]);
#pragma unroll
            for (int np = 0; np < D / 16; np++) {
                const int brow = (kk * 16 + (lane & 7) + 8 * (m & 1)) * TL::LD + np * 16 + 8 * (m >> 1);
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(r0, r1, r2, r3, cO + brow);
                mma_bf16_16816(dvacc[2 * np], pa, r0, r1);
                mma_bf16_16816(dvacc[2 * np + 1], pa, r2, r3);
                ldmatrix_x4_trans(r0, r1, r2, r3, cQ + brow);
                mma_bf16_16816(dkacc[2 * np], sa, r0, r1);
                mma_bf16_16816(dkacc[2 * np + 1], sa, r2, r3);
            }
            // dS^T rows (keys) x cols (queries) to shared memory for dQ
#pragma unroll
            for (int half = 0; half < 2; half++) {
                const int n = 2 * kk + half;
                const int col = n * 8 + 2 * t4;
                *reinterpret_cast<uint32_t *>(sS + (warp * 16 + g) * TL::LDS + col) =
                    pack_bf16(pacc[n][0], pacc[n][1]);
                *reinterpret_cast<uint32_t *>(sS + (warp * 16 + g + 8) * TL::LDS + col) =
                    pack_bf16(pacc[n][2], pacc[n][3]);
            }
        }
        __syncthreads();
        // dQ[i, c] += sum_j dS[i, j] K[j, c]; warp: 16 query rows x D/2 columns
        {
            const int ib = (warp & 1) * 16, cb = (warp >> 1) * (D / 2);
            float qacc[D / 16][4];
#pragma unroll
            for (int n = 0; n < D / 16; n++)
#pragma unroll
                for (int e = 0; e < 4; e++)
                    qacc[n][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < BN / 16; kk++) {
                uint32_t af[4];
                ldmatrix_x4_trans(af[0], af[1], af[2], af[3],
                                  sS + (kk * 16 + (lane & 7) + 8 * (m >> 1)) * TL::LDS + ib + 8 * (m & 1));
#pragma unroll
                for (int np = 0; np < D / 32; np++) {
                    uint32_t r0, r1, r2, r3;
                    ldmatrix_x4_trans(r0, r1, r2, r3,
                                      sK + (kk * 16 + (lane & 7) + 8 * (m & 1)) * TL::LD + cb + np * 16 +
                                          8 * (m >> 1));
                    mma_bf16_16816(qacc[2 * np], af, r0, r1);
                    mma_bf16_16816(qacc[2 * np + 1], af, r2, r3);
                }
            }
#pragma unroll
            for (int a = 0; a < 2; a++) {
                const int i = i0 + ib + g + 8 * a;
                if (i >= s.L)
                    continue;
                float *row = p.dq_acc + ((s.s0 + i) * p.H + h) * (int64_t)D + cb;
#pragma unroll
                for (int n = 0; n < D / 16; n++) {
                    atomicAdd(row + n * 8 + 2 * t4, qacc[n][2 * a]);
                    atomicAdd(row + n * 8 + 2 * t4 + 1, qacc[n][2 * a + 1]);
                }
            }
        }
        __syncthreads();
    }

    // dK, dV rows of this key tile
    __nv_bfloat16 *gdk = static_cast<__nv_bfloat16 *>(p.dk);
    __nv_bfloat16 *gdv = static_cast<__nv_bfloat16 *>(p.dvv);
#pragma unroll
    for (int a = 0; a < 2; a++) {
        if (rj[a] >= s.L)
            continue;
        __nv_bfloat16 *rk = gdk + (s.s0 + rj[a]) * p.sdk + (int64_t)h * D;
        __nv_bfloat16 *rv = gdv + (s.s0 + rj[a]) * p.sdv + (int64_t)h * D;
#pragma unroll
        for (int n = 0; n < D / 8; n++) {
            *reinterpret_cast<uint32_t *>(rk + n * 8 + 2 * t4) = pack_bf16(dkacc[n][2 * a], dkacc[n][2 * a + 1]);
            *reinterpret_cast<uint32_t *>(rv + n * 8 + 2 * t4) = pack_bf16(dvacc[n][2 * a], dvacc[n][2 * a + 1]);
        }
    }
    if (bins_in_smem) {
        __syncthreads();
        for (int e = threadIdx.x; e < npos + p.nb; e += kThreads) {
            float v = sBin[e];
            if (v != 0.f)
                atomicAdd(e < npos ? p.d_rab_pos + e : p.d_rab_time + (e - npos), v);
        }
    }
}

__global__ void convert_dq_kernel(const float *__restrict__ acc, __nv_bfloat16 *__restrict__ dq,
                                  int64_t T, int H, int d, int64_t sdq, float scale)
{
    const int64_t n = T * H * d;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * blockDim.x) {
        int64_t t = e / ((int64_t)H * d);
        int64_t r = e % ((int64_t)H * d);
        dq[t * sdq + r] = __float2bfloat16_rn(acc[e] * scale);
    }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D>
cudaError_t fwd_launch(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    const int npos = p.pos_hi - p.pos_lo + 1;
    size_t bytes = Tiles<D>::bytes + (npos + p.nb <= kSmemTableMax ? (npos + p.nb) * sizeof(float) : 0);
    cudaError_t e = set_smem(attn_fwd_mma_kernel<D>, bytes);
    if (e != cudaSuccess)
        return e;
    attn_fwd_mma_kernel<D><<<(unsigned)grid_items * p.H, kThreads, bytes, stream>>>(p);
    return cudaGetLastError();
}

template <int D>
cudaError_t bwd_launch(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    const int npos = p.pos_hi - p.pos_lo + 1;
    size_t bytes = BwdTiles<D>::bytes + (npos + p.nb <= kSmemBinMax ? (npos + p.nb) * sizeof(float) : 0);
    cudaError_t e = set_smem(attn_bwd_mma_kernel<D>, bytes);
    if (e != cudaSuccess)
        return e;
    attn_bwd_mma_kernel<D><<<(unsigned)grid_items * p.H, kThreads, bytes, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_mma(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    if (grid_items <= 0)
        return cudaSuccess;
    switch (p.dqk) {
    case 32: return fwd_launch<32>(p, grid_items, stream);
    case 64: return fwd_launch<64>(p, grid_items, stream);
    case 128: return fwd_launch<128>(p, grid_items, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attn_bwd_mma(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    if (grid_items <= 0)
        return cudaSuccess;
    switch (p.dqk) {
    case 32: return bwd_launch<32>(p, grid_items, stream);
    case 64: return bwd_launch<64>(p, grid_items, stream);
    case 128: return bwd_launch<128>(p, grid_items, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_convert_dq(const float *acc, void *dq, int64_t T, int H, int d, int64_t sdq,
                              float scale, cudaStream_t stream)
{
    if (T == 0)
        return cudaSuccess;
    int64_t n = T * H * d;
    int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
    convert_dq_kernel<<<blocks, 256, 0, stream>>>(acc, static_cast<__nv_bfloat16 *>(dq), T, H, d, sdq,
                                                  scale);
    return cudaGetLastError();
}

}  // namespace hstu
