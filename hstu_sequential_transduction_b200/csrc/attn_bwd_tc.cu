// HSTU jagged attention backward on sm_100a: TMA + tcgen05 (TMEM), head dims 64
// and 128.
//
// Exact derivatives of the forward (the DLRMv4 page, text under Table 7: the
// backward produces dQ, dK and dV through about five GEMMs), plus the
// gradients of the relative-bias tables.  Per work item (sequence, 128-row key
// tile, head) the CTA keeps K and V resident and walks the query rows that see
// the tile in steps of 64:
//   S^T  = K Q^T,  dP^T = V dO^T               (TMEM, 64 columns each)
//   P = SiLU(s), dS' = dP * 2 SiLU'(s)          (epilogue, s = score + bias)
//   dV += P^T dO,  dK += dS'^T Q                (TMEM accumulators, 128 cols each)
//   dQ^T = K^T dS'^T                            (TMEM) -> shared staging ->
//        TMA bulk reduce-add into an fp32 dQ accumulator in global memory
// The constant factors (inv_n for P, inv_n / 2 for dS) are applied once at
// the end.  With h = s / 2 and t = tanh(h):
//   SiLU(s) = h (1 + t),  2 SiLU'(s) = (1 + t)(1 + h (1 - t)) = 1 + t + h (1 - t^2).
// Bias-table gradients without per-pair atomics: the positional index of a
// pair is query - key, constant along diagonals, so each warp reduces its
// 32 x 32 block of dS' along the 63 diagonals with one shuffle per column and
// adds each diagonal sum to the table with one global reduction; the two
// clamped entries, which most far blocks land on, are summed in registers per
// thread and reduced once per warp and CTA.  Time buckets are monotone along a
// key row of sorted stamps: lane k of a warp holds the warp's sum for bucket
// k; blocks within two adjacent buckets add to per-thread carries, reduced
// across the warp only when the bucket moves; other blocks write their rows'
// bucket runs to a lane-private shared row that lane k sums by column.
// Candidate rows, unsorted stamps and stamps spanning more than 2^24 s take an
// exact per-pair path.
//
// Warp roles (320 threads): warp 0 TMA, warp 1 TMEM owner + MMA issuer,
// warps 2-9 epilogue (lane quarter = warp % 4 selects the TMEM rows, the two
// groups of four warps split each step's 64 query columns).
// TMEM columns: dK [0,128), dV [128,256), S^T [256,320), dP^T [320,384),
// dQ^T [384,448), and the bf16 P^T [448,480) and dS'^T [480,512) of a step,
// which the dV and dK MMAs read as their A operands straight from TMEM.
#include "internal.h"
#include "tc_common.cuh"

namespace hstu {

namespace {

constexpr int KB = 128;  // key rows per CTA
constexpr int QB = 64;   // query rows per step
constexpr int kEpiWarpsB = 8;                   // 2 per TMEM lane quarter
constexpr int kEpiThreadsB = kEpiWarpsB * 32;
constexpr int kThreadsB = kEpiThreadsB + 64;
constexpr int kGroupsB = kEpiWarpsB / 4;         // column groups of a step
constexpr int NC = QB / kGroupsB;                // query columns per epilogue thread
constexpr uint32_t kTmemColsB = 512;
constexpr int kRegK = 16384;  // 128 rows x 128 B
constexpr int kRegQ = 8192;   // 64 rows x 128 B
constexpr int COL_DK = 0, COL_DV = 128, COL_S = 256, COL_DP = 320, COL_DQ = 384, COL_PT = 448, COL_DST = 480;

constexpr int QS = 3;  // Q / dO ring stages
enum BBars { KV_FULL = 0, Q_FULL = 1, Q_EMPTY = Q_FULL + QS, S_FULL = Q_EMPTY + QS, S_FREE, P_FULL, P_FREE,
             DQ_FULL, DQ_FREE, ACC_FULL, NBARS_B };

// Shared-memory layout for head dim DH (64 or 128): NR = DH / 64 swizzled
// 128-byte-wide regions per tile.  V directly follows K, so that for DH = 64 the
// dQ^T MMA can run with M = 128: its second 64 rows read V^T and are discarded.
template <int DH>
struct BL {
    static constexpr int NR = DH / 64;
    static constexpr int K = 0;
    static constexpr int V = K + NR * kRegK;
    static constexpr int Q0 = V + NR * kRegK;       // QS stages x NR regions
    static constexpr int O0 = Q0 + QS * NR * kRegQ;  // dO, QS stages x NR regions
    static constexpr int DST = O0 + QS * NR * kRegQ;  // dS'^T [128 keys x 64 queries] (B operand of dQ^T)
    // per warp, 4 KB used in turn: dQ staging, fp32 [NC x 32], and 32 lanes x 32
    // time-bucket partial sums
    static constexpr int DQS = DST + kRegK;
    static constexpr int E = DQS + QB * 128 * 4;   // time bias by exponent (512)
    static constexpr int PW = E + 512 * 4;         // per warp: NC query stamps + 64 bias window
    static constexpr int PW_FLOATS = NC + 64;
    static constexpr int BAR = PW + kEpiWarpsB * PW_FLOATS * 4;
    static constexpr int MISC = BAR + NBARS_B * 8;
    static constexpr int BYTES = MISC + 64;
    static_assert(BYTES + 1024 <= 227 * 1024, "backward tile does not fit in shared memory");
};

__device__ __forceinline__ uint32_t exp_offset(float ti1, float tj)
{
    return (__float_as_uint(__fsub_rz(ti1, tj)) >> 21) & 0x7FCu;
}

__device__ __forceinline__ int exp_bucket(int e, int nb)
{
    return (e >= 256 || e < 127) ? 0 : min(e - 127, nb - 1);
}

// Block classes (uniform across one warp's 32 keys x NC queries of a step).
//   CLAMPED  every pair visible and on one clamped positional index;
//   WINDOW   no candidate queries: positional index = query - key, read from
//            and reduced along the block's diagonals (masked when not full);
//   GENERAL  candidate queries, unsorted stamps or stamps outside the
//            fast-bucket range: exact per-pair path.
enum StepClass { CLS_GENERAL = 0, CLS_WINDOW = 1, CLS_WINDOW_MASKED = 2, CLS_CLAMPED = 3 };

// NC consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld_nc(uint32_t taddr, float *v)
{
    if constexpr (NC == 16)
        tmem_ld16(taddr, v);
    else
        tmem_ld32(taddr, v);
}

// Result of the elementwise pass over one thread's NC query columns.
struct RowOut {
    uint32_t b0, b1;  // exponent offsets of the first and last visible column
    float all, hi;    // sum of dS' over the row segment, and over columns in bucket b1
    bool mid;         // a visible column falls in a bucket other than b0 and b1
};

// Time-bucket modes of a 32 x NC block (decided per warp from the extreme
// stamp differences of its sorted rows and columns).
enum BucketMode { BK_ANY = 0, BK_ONE = 1, BK_TWO = 2 };

// Elementwise backward of the NC query columns one thread owns (one key row):
// P = SiLU, dS' = dP (1+t)(1+h(1-t)); dS' replaces dP in dv[], P is packed.
// Columns outside [c_lo, c_hi) are masked when MASK.  The time bucket of a
// column: BK_ONE, the whole block is in one bucket, whose bias the caller has
// already added to the positional term (wrow / bconst); BK_TWO, every row spans
// at most two buckets, so the bucket is one compare of the exact
// round-toward-zero difference against the upper bucket's power of two;
// BK_ANY, looked up per column.  No atomics, no data-dependent branches.
// Written as three passes over the columns (biased half-scores, tanh,
// products) so that the independent per-column chains are issued back to
// back instead of one after the other.
template <bool MASK, bool WINDOW, int MODE>
__device__ __forceinline__ RowOut bwd_row(float *sv, float *dv, const float *ti, float tjf, const char *Eb,
                                          const float *wrow, float bconst, int c_lo, int c_hi, uint32_t *pk)
{
    RowOut o;
    const int f = MASK ? min(max(c_lo, 0), NC - 1) : 0, l = MASK ? min(max(c_hi - 1, 0), NC - 1) : NC - 1;
    o.b0 = exp_offset(ti[f], tjf);
    o.b1 = MODE == BK_ONE ? o.b0 : exp_offset(ti[l], tjf);
    const float E0 = MODE == BK_ONE ? 0.f : *reinterpret_cast<const float *>(Eb + o.b0);
    const float E1 = MODE == BK_ONE ? 0.f : *reinterpret_cast<const float *>(Eb + o.b1);
    // BK_TWO: a column is in bucket b1 when RZ(ti - tj) >= 2^(bucket of b1); the
    // stamps are integers and the threshold a power of two, so that is ti >= tj + 2^k
    // in exact arithmetic, i.e. ti >= RU(tj + 2^k): one compare per column
    const float lim = __fadd_ru(tjf, __uint_as_float(o.b1 << 21));
    o.mid = false;
    float upf[NC];  // 1 where the column is in bucket b1
#pragma unroll
    for (int u = 0; u < NC / 4; u++) {
        float tv[4];
        if (MODE != BK_ONE) {
            const float4 t4 = *reinterpret_cast<const float4 *>(ti + 4 * u);  // stamps are shared by the warp
            tv[0] = t4.x;
            tv[1] = t4.y;
            tv[2] = t4.z;
            tv[3] = t4.w;
        }
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int c = 4 * u + e;
            float bt;
            if (MODE == BK_ONE) {
                bt = 0.f;  // the block's one time bias is folded into bp by the caller
                upf[c] = 0.f;
            } else if (MODE == BK_TWO) {
                const bool up = tv[e] >= lim;
                upf[c] = up ? 1.f : 0.f;
                bt = up ? E1 : E0;
            } else {
                const uint32_t off = exp_offset(tv[e], tjf);
                bt = *reinterpret_cast<const float *>(Eb + off);
                upf[c] = off == o.b1 ? 1.f : 0.f;
                o.mid |= (!MASK || (c >= c_lo && c < c_hi)) && (off != o.b0) && (off != o.b1);
            }
            const float bp = WINDOW ? wrow[c] : bconst;
            sv[c] = MODE == BK_ONE ? fmaf(sv[c], 0.5f, bp) : fmaf(sv[c], 0.5f, bp) + bt;
        }
    }
    float th[NC];
#pragma unroll
    for (int c = 0; c < NC; c++)
        th[c] = tanh_approx(sv[c]);
    // four partial sums each, so that the additions do not form one serial chain
    float all[4] = {0.f, 0.f, 0.f, 0.f}, hi[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < NC; c += 2) {
        float pv[2];
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int cc = c + e;
            const float hh = sv[cc], t = th[cc];
            float pval = fmaf(hh, t, hh);
            // (1 + t)(1 + h (1 - t)) = 1 + t + h (1 - t^2)
            const float y = fmaf(hh, fmaf(-t, t, 1.f), t);
            float ds = fmaf(dv[cc], y, dv[cc]);
            if (MASK) {
                const bool vis = cc >= c_lo && cc < c_hi;
                pval = vis ? pval : 0.f;
                ds = vis ? ds : 0.f;
            }
            dv[cc] = ds;
            pv[e] = pval;
            all[cc & 3] += ds;
            if (MODE != BK_ONE)
                hi[cc & 3] = fmaf(upf[cc], ds, hi[cc & 3]);
        }
        pk[c >> 1] = pack_bf16(pv[0], pv[1]);
    }
    o.all = (all[0] + all[1]) + (all[2] + all[3]);
    o.hi = (hi[0] + hi[1]) + (hi[2] + hi[3]);
    return o;
}

// Sums of dS' along the diagonals of a warp's 32 x NC block (lanes are key
// rows, registers query columns): lane l returns diagonal l in accP (zero for
// l >= NC) and diagonal l - 32 in accN, with one shuffle per column.
__device__ __forceinline__ void warp_diagonals(const float *ds, int lane, float &accP, float &accN)
{
    float p2[2] = {0.f, 0.f}, n2[2] = {0.f, 0.f};  // two chains each
#pragma unroll
    for (int k = 0; k < NC; k++) {
        // the source lane is taken modulo 32: k - lane wraps to the row on diagonal lane or lane - 32
        const float y = __shfl_sync(0xffffffffu, ds[k], k - lane);
        if (k >= lane)
            p2[k & 1] += y;
        else
            n2[k & 1] += y;
    }
    accP = p2[0] + p2[1];
    accN = n2[0] + n2[1];
}

// DH: head dim (64 or 128); SL: semi-local windows in use (otherwise every
// window test compiles away)
template <int DH, bool SL, bool XB = false>
__global__ void __launch_bounds__(kThreadsB, 1)
attn_bwd_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmDQ, int head_major,
                   const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV, int kv_tma)
{
    using BL = hstu::BL<DH>;
    constexpr int NR = BL::NR;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);

    // Block order over the schedule's longest-first tile list: the heads of a
    // tile side by side, or head-major (every tile for head 0, then head 1, ...)
    // when the launch asks for it, so that the tiles in flight share one head's
    // Q, dO and dQ accumulator rows in L2
    const int grid_items = gridDim.x / p.H;
    const int item = head_major ? blockIdx.x % grid_items : blockIdx.x / p.H;
    const int h = head_major ? blockIdx.x / grid_items : blockIdx.x % p.H;
    if (item >= p.hdr->n_items)
        return;
    const int2 it = p.items[item];
    const int64_t s0 = p.seq_offsets[it.x];
    const int L = (int)(p.seq_offsets[it.x + 1] - s0);
    const int hist = L - (p.num_targets ? p.num_targets[it.x] : 0);
    const int j0 = it.y * KB;
    const int lw = SL ? p.lw : 0, gw = SL ? p.gw : 0;
    int q_end = j0 < hist ? L : min(j0 + KB, L);
    // Semi-local windows: without global keys in the tile, history queries past
    // the local window of its last key see nothing, and candidates (position
    // hist) see it only if hist is within the window of that key
    if (lw > 0 && j0 >= gw && j0 < hist) {
        const int last = min(j0 + KB, hist) - 1;
        if (hist - last >= lw)
            q_end = min(q_end, min(hist, last + lw));
    }
    const int nq = (q_end - j0 + QB - 1) / QB;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) { return base + BL::BAR + 8u * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + BL::MISC + 8);
    float *E = reinterpret_cast<float *>(sm + BL::E);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBARS_B; i++) {
            const bool epi = (i == S_FREE || i == P_FULL || i == DQ_FREE);
            mbar_init(bar(i), epi ? kEpiWarpsB : 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tmK);
        tma_prefetch(&tmV);
        tma_prefetch(&tmQ);
        tma_prefetch(&tmO);
        tma_prefetch(&tmDQ);
    }
    if (warp == 1)
        tmem_alloc(base + BL::MISC, kTmemColsB);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + BL::MISC);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            mbar_expect_tx(bar(KV_FULL), 2 * NR * kRegK);
            for (int r = 0; r < NR; r++) {
                tma_load_2d(base + BL::K + r * kRegK, &tmK, h * DH + 64 * r, (int)(s0 + j0), bar(KV_FULL));
                tma_load_2d(base + BL::V + r * kRegK, &tmV, h * DH + 64 * r, (int)(s0 + j0), bar(KV_FULL));
            }
            for (int i = 0; i < nq; i++) {
                const int s = i % QS;
                const int y = (int)(s0 + j0 + i * QB);
                if (i >= QS && !mbar_wait(bar(Q_EMPTY + s), ((i - QS) / QS) & 1, abort_flag, p.hdr))
                    break;
                mbar_expect_tx(bar(Q_FULL + s), 2 * NR * kRegQ);
                for (int r = 0; r < NR; r++) {
                    tma_load_2d(base + BL::Q0 + s * NR * kRegQ + r * kRegQ, &tmQ, h * DH + 64 * r, y, bar(Q_FULL + s));
                    tma_load_2d(base + BL::O0 + s * NR * kRegQ + r * kRegQ, &tmO, h * DH + 64 * r, y, bar(Q_FULL + s));
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idSdP = idesc_bf16(KB, QB, 0, 0);
            constexpr uint32_t idGrad = idesc_bf16(KB, DH, 0, 1);
            constexpr uint32_t idDQ = idesc_bf16(128, QB, 1, 1);  // DH = 64: rows 64-127 are discarded
            auto issue_SdP = [&](int i) {
                const int s = i % QS;
                for (int ks = 0; ks < DH / 16; ks++) {
                    const uint32_t ok_ = (ks >> 2) * kRegK + (ks & 3) * 32;
                    const uint32_t oq = s * NR * kRegQ + (ks >> 2) * kRegQ + (ks & 3) * 32;
                    umma_bf16(tmem + COL_S, smem_desc_sw128(base + BL::K + ok_, 16, 1024),
                              smem_desc_sw128(base + BL::Q0 + oq, 16, 1024), idSdP, ks > 0);
                    umma_bf16(tmem + COL_DP, smem_desc_sw128(base + BL::V + ok_, 16, 1024),
                              smem_desc_sw128(base + BL::O0 + oq, 16, 1024), idSdP, ks > 0);
                }
                umma_commit(bar(S_FULL));
            };
            auto issue_grads = [&](int i) {
                const int s = i % QS;
                // A = P^T / dS'^T from TMEM (lane = key, column = query pair)
                for (int ks = 0; ks < QB / 16; ks++) {
                    const uint32_t acc = (i > 0 || ks > 0);
                    umma_bf16_ts(tmem + COL_DV, tmem + COL_PT + 8 * ks,
                                 smem_desc_sw128(base + BL::O0 + s * NR * kRegQ + ks * 2048, kRegQ, 1024), idGrad, acc);
                    umma_bf16_ts(tmem + COL_DK, tmem + COL_DST + 8 * ks,
                                 smem_desc_sw128(base + BL::Q0 + s * NR * kRegQ + ks * 2048, kRegQ, 1024), idGrad, acc);
                }
            };
            auto issue_dq = [&]() {
                for (int ks = 0; ks < KB / 16; ks++)
                    umma_bf16(tmem + COL_DQ, smem_desc_sw128(base + BL::K + ks * 2048, kRegK, 1024),
                              smem_desc_sw128(base + BL::DST + ks * 2048, kRegK, 1024), idDQ, ks > 0);
            };
            bool ok = mbar_wait(bar(KV_FULL), 0, abort_flag, p.hdr) &&
                      mbar_wait(bar(Q_FULL), 0, abort_flag, p.hdr);
            if (ok) {
                tc_fence_after();
                issue_SdP(0);
            }
            for (int i = 0; ok && i < nq; i++) {
                if (i + 1 < nq) {
                    ok = mbar_wait(bar(S_FREE), i & 1, abort_flag, p.hdr) &&
                         mbar_wait(bar(Q_FULL + (i + 1) % QS), ((i + 1) / QS) & 1, abort_flag, p.hdr);
                    if (!ok)
                        break;
                    tc_fence_after();
                    issue_SdP(i + 1);
                }
                if (!(ok = mbar_wait(bar(P_FULL), i & 1, abort_flag, p.hdr)))
                    break;
                tc_fence_after();
                issue_grads(i);
                if (i > 0) {
                    if (!(ok = mbar_wait(bar(DQ_FREE), (i - 1) & 1, abort_flag, p.hdr)))
                        break;
                    tc_fence_after();
                }
                issue_dq();
                umma_commit(bar(Q_EMPTY + i % QS));
                umma_commit(bar(P_FREE));
                umma_commit(bar(DQ_FULL));
            }
            umma_commit(bar(ACC_FULL));
        }
    } else {
        // ---------------- epilogue ----------------
        // time tables, filled while the first tiles load; only the epilogue warps use them
        // offsets of this CTA's head's rows in per-head tables and their gradients
        // (zero with shared tables)
        const int hp = XB ? h * (int)p.pos_hstride : 0, ht = XB ? h * (int)p.time_hstride : 0;
        const bool own = XB && p.cand_own != 0;
        for (int e = threadIdx.x - 64; e < 512; e += kEpiThreadsB)
            E[e] = 0.5f * p.rab_time[ht + exp_bucket(e, p.nb)];
        named_bar(1, kEpiThreadsB);
        // Every warp handles a 32-key x NC-query block of each step on its own:
        // stamps, bias window, class and bias-table gradients are per warp, so
        // the loop has no CTA-wide barrier.
        const int ew = warp - 2, g = ew >> 2, quarter = warp & 3;
        const uint32_t full = 0xffffffffu;
        const int r = quarter * 32 + lane;  // key row of the tile (TMEM lane); d index for dQ^T
        const int j = j0 + r;
        const bool krow_ok = j < L;
        const int lo = p.pos_lo, hi = p.pos_hi;
        const int64_t tb = p.timestamps[s0 + j0];
        const int64_t tj = krow_ok ? p.timestamps[s0 + j] : tb;
        const int pj = token_pos(j, hist, own);
        const int64_t lim = (int64_t)1 << 24;
        const float tjf = (float)(tj - tb);
        const float gscale = 0.5f * p.inv_n;
        const int jw0 = j0 + quarter * 32;                 // first key row of the warp
        const int jw_n = max(0, min(32, L - jw0));         // valid key rows of the warp
        const int64_t tj_up = __shfl_up_sync(full, tj, 1);
        const bool rows_bad = __any_sync(full, krow_ok && ((tj - tb >= lim) || (tj - tb <= -lim) ||
                                                           (lane > 0 && tj_up > tj)));
        const float tjf_first = __shfl_sync(full, tjf, 0);
        const float tjf_last = __shfl_sync(full, tjf, max(jw_n - 1, 0));
        float *TIw = reinterpret_cast<float *>(sm + BL::PW) + ew * BL::PW_FLOATS;  // NC stamps
        float *Ww = TIw + NC;  // Ww[m]: positional bias / 2 at diagonal (query - key) = D_w + m - 31
        float *DQW = reinterpret_cast<float *>(sm + BL::DQS) + ew * NC * 32;  // this warp's [NC x 32]
        const uint32_t dqw_addr = base + BL::DQS + ew * NC * 128;
        const char *Eb = reinterpret_cast<const char *>(E);
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        auto clamp_idx = [&](int d) { return (d < lo ? lo : (d > hi ? hi : d)) - lo; };

        // Time-bias gradient.  Outside the exact path every stamp difference lies
        // in (-2^25, 2^25), so its exponent bucket k = e - 127 (e the biased
        // exponent of the float difference; k = 0 for e < 127 or a negative
        // difference, which the bucketisation also sends to bucket 0) is below 26:
        // lane k of the warp holds the warp's running sum for k in hacc, and
        // the global table gets one reduction per lane when the CTA ends.
        // Blocks whose pairs span at most two adjacent buckets (klo, klo + 1 for
        // the whole warp) add to per-thread carries c0 / c1, summed across the
        // warp only when klo moves, which it does a few dozen times per CTA
        // since buckets only grow along a key row of sorted stamps.  Other blocks
        // go through TGw: each thread writes the sums of its row's bucket runs
        // to its own 32-float row (groups of four XOR-swizzled by the lane, so
        // the zeroing and the column reads are conflict free) and lane k then
        // adds up column k.
        float hacc = 0.f, c0 = 0.f, c1 = 0.f;
        int kc = -1;
        // Gradient of the two clamped positional entries (distance >= pos_hi and
        // <= pos_lo), summed per thread over the whole CTA and reduced once at the
        // end: every far block lands on them, and adding each step's small partial
        // sums straight into their large global totals would round most of them away.
        float cl_hi = 0.f, cl_lo = 0.f;
        float *TGw = reinterpret_cast<float *>(sm + BL::DQS) + ew * 32 * 32;  // shares the dQ staging
        float *tgr = TGw + lane * 32;
        auto tg_slot = [&](uint32_t k, int row) { return (((k >> 2) ^ (uint32_t)(row & 7)) << 2) | (k & 3); };
        auto k_of = [](uint32_t off) {  // exp_offset -> bucket k
            const uint32_t k = (off >> 2) - 127u;
            return k < 32u ? k : 0u;
        };
        auto warp_sum = [&](float v) {
#pragma unroll
            for (int o = 16; o; o >>= 1)
                v += __shfl_xor_sync(full, v, o);
            return v;
        };
        auto carry_flush = [&](int klo) {  // warp-uniform
            if (kc >= 0) {
                const float r0 = warp_sum(c0);
                if (lane == kc)
                    hacc += r0;
                if (klo == kc + 1) {
                    c0 = c1;
                } else {
                    const float r1 = warp_sum(c1);
                    if (lane == kc + 1)
                        hacc += r1;
                    c0 = 0.f;
                }
            }
            c1 = 0.f;
            kc = klo;
        };

        // dQ'^T of step k for this warp: TMEM -> [NC queries x 32 d] staging ->
        // bulk reduce-add (each warp its own box)
        auto handle_dq = [&](int k) -> bool {
            if (!mbar_wait(bar(DQ_FULL), k & 1, abort_flag, p.hdr))
                return false;
            tc_fence_after();
            if (32 * quarter >= DH) {  // rows past the head dim (DH = 64): nothing to add
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bar(DQ_FREE));
                return true;
            }
            float qv[NC];
            tmem_ld_nc(trow + COL_DQ + NC * g, qv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(DQ_FREE));
                bulk_wait_read0();
            }
            __syncwarp();
#pragma unroll
            for (int c = 0; c < NC; c++)
                DQW[c * 32 + lane] = qv[c];
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_reduce_add_2d(&tmDQ, h * DH + 32 * quarter, (int)(s0 + j0 + k * QB + NC * g), dqw_addr);
                bulk_commit();
            }
            return true;
        };

        // per-warp inputs of step i, prefetched one step ahead
        int64_t tq = tb;
        float wlo = 0.f, whi = 0.f;
        auto prefetch = [&](int i) {
            const int iw0 = j0 + i * QB + NC * g;
            const int dw = iw0 - jw0;
            wlo = 0.5f * p.rab_pos[hp + clamp_idx(dw + lane - 31)];
            whi = 0.5f * p.rab_pos[hp + clamp_idx(dw + lane + 1)];
            if (lane < NC)
                tq = iw0 + lane < L ? p.timestamps[s0 + iw0 + lane] : tb;
        };
        prefetch(0);
        bool ok = true;
        for (int i = 0; i < nq; i++) {
            const int i0 = j0 + i * QB;
            const int iw0 = i0 + NC * g;  // first query of this warp's block
            const int dw = iw0 - jw0;     // query - key offset of the block's diagonal 0
            const int64_t tq_up = __shfl_up_sync(full, tq, 1);
            const bool q_ok = lane < NC && iw0 + lane < L;
            const bool cols_bad = __any_sync(full, q_ok && ((tq - tb + 1 >= lim) || (tq - tb + 1 <= -lim) ||
                                                            (lane > 0 && tq_up > tq)));
            const float tqf = (float)(tq - tb + 1);

            const int q_last = min(iw0 + NC, L) - 1;  // last valid query of the block
            // every pair of the block inside the local window, or every key global
            const bool band_w = lw <= 0 || iw0 + NC - 1 - jw0 < lw || jw0 + 32 <= gw;
            const bool full_w = (iw0 >= jw0 + 31) && (jw0 + 32 <= hist) && (iw0 + NC <= L) && (iw0 + NC <= hist) &&
                                band_w;
            const int dmin_w = dw - 31, dmax_w = dw + NC - 1;
            int cls = CLS_GENERAL;
            if (!rows_bad && !cols_bad) {
                if (full_w && (dmin_w >= hi || dmax_w <= lo))
                    cls = CLS_CLAMPED;
                else if (q_last < hist)
                    cls = full_w ? CLS_WINDOW : CLS_WINDOW_MASKED;
            }
            int mode = BK_ANY;
            int klo = 0;  // bucket of the block's smallest stamp difference (BK_ONE, BK_TWO)
            const float dlo = __fsub_rz(__shfl_sync(full, tqf, 0), tjf_last);
            const float dhi = __fsub_rz(__shfl_sync(full, tqf, max(0, q_last - iw0)), tjf_first);
            float e_one = 0.f;  // BK_ONE: the block's time bias / 2, folded into the window
            if (cls != CLS_GENERAL && q_last >= iw0 && jw_n > 0) {
                const uint32_t de = (__float_as_uint(dhi) >> 23) - (__float_as_uint(dlo) >> 23);
                if (dlo >= 1.f)
                    mode = de == 0 ? BK_ONE : (de == 1 ? BK_TWO : BK_ANY);
                klo = (int)(__float_as_uint(dlo) >> 23) - 127;
                // (a masked block runs the per-column variant, which adds the bias itself)
                if (mode == BK_ONE && cls != CLS_WINDOW_MASKED)
                    e_one = *reinterpret_cast<const float *>(Eb + ((__float_as_uint(dlo) >> 21) & 0x7FCu));
            }
            __syncwarp();
            if (lane < NC)
                TIw[lane] = tqf;
            Ww[lane] = wlo + e_one;
            Ww[lane + 32] = whi + e_one;
            __syncwarp();
            if (i + 1 < nq)
                prefetch(i + 1);

            if (!(ok = mbar_wait(bar(S_FULL), i & 1, abort_flag, p.hdr)))
                break;
            tc_fence_after();
            float sv[NC], dv[NC];
            tmem_ld_nc(trow + COL_S + NC * g, sv);
            tmem_ld_nc(trow + COL_DP + NC * g, dv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(S_FREE));

            uint32_t pk[NC / 2], dk[NC / 2];
            if (cls != CLS_GENERAL) {
                RowOut o;
                if (cls == CLS_CLAMPED) {
                    if (mode == BK_ONE)
                        o = bwd_row<false, false, BK_ONE>(sv, dv, TIw, tjf, Eb, nullptr, Ww[0], 0, NC, pk);
                    else if (mode == BK_TWO)
                        o = bwd_row<false, false, BK_TWO>(sv, dv, TIw, tjf, Eb, nullptr, Ww[0], 0, NC, pk);
                    else
                        o = bwd_row<false, false, BK_ANY>(sv, dv, TIw, tjf, Eb, nullptr, Ww[0], 0, NC, pk);
                    if (dmin_w >= hi)
                        cl_hi += o.all;
                    else
                        cl_lo += o.all;
                } else {
                    const float *wrow = Ww + 31 - lane;  // wrow[c]: diagonal c - lane
                    if (cls == CLS_WINDOW)
                        o = mode == BK_ONE   ? bwd_row<false, true, BK_ONE>(sv, dv, TIw, tjf, Eb, wrow, 0.f, 0, NC, pk)
                            : mode == BK_TWO ? bwd_row<false, true, BK_TWO>(sv, dv, TIw, tjf, Eb, wrow, 0.f, 0, NC, pk)
                                             : bwd_row<false, true, BK_ANY>(sv, dv, TIw, tjf, Eb, wrow, 0.f, 0, NC, pk);
                    else {
                        // this key row sees queries [j, L), cut at j + local_window
                        // unless the key is global
                        const int c_hi = (lw > 0 && j >= gw) ? min(NC, min(L, j + lw) - iw0) : min(NC, L - iw0);
                        o = bwd_row<true, true, BK_ANY>(sv, dv, TIw, tjf, Eb, wrow, 0.f, j - iw0,
                                                       krow_ok ? c_hi : 0, pk);
                    }
                    float accP, accN;
                    warp_diagonals(dv, lane, accP, accN);
                    // diagonal sums: past either clamp into the CTA's accumulators,
                    // otherwise straight to the table
                    auto diag_add = [&](int dd, float v) {
                        if (dd >= hi)
                            cl_hi += v;
                        else if (dd <= lo)
                            cl_lo += v;
                        else if (v != 0.f)
                            red_add_global(p.d_rab_pos + hp + (dd - lo), v * gscale);
                    };
                    diag_add(dw + lane, accP);
                    diag_add(dw + lane - 32, accN);
                }
                const bool two = o.b1 != o.b0;
                const float v0 = two ? o.all - o.hi : o.all, v1 = two ? o.hi : 0.f;
                if (mode != BK_ANY) {
                    // every visible pair of the block is in bucket klo or klo + 1
                    if (klo != kc)
                        carry_flush(klo);
                    const bool up0 = (int)k_of(o.b0) != kc, up1 = (int)k_of(o.b1) != kc;
                    c0 += (up0 ? 0.f : v0) + (up1 ? 0.f : v1);
                    c1 += (up0 ? v0 : 0.f) + (up1 ? v1 : 0.f);
                } else {
                    // the bulk reduction of the previous dQ has read the staging, and
                    // the lanes have read the rows of the previous block
                    if (lane == 0)
                        bulk_wait_read0();
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < 8; u++)
                        *reinterpret_cast<float4 *>(tgr + ((u ^ (lane & 7)) << 2)) = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (!o.mid) {
                        // at most two runs, b0 then b1 (distinct offsets below 2 share bucket 0)
                        const uint32_t k0 = k_of(o.b0), k1 = k_of(o.b1);
                        tgr[tg_slot(k0, lane)] = k1 == k0 ? v0 + v1 : v0;
                        if (k1 != k0)
                            tgr[tg_slot(k1, lane)] = v1;
                    } else {
                        // buckets never decrease along the row, so each run is one store
                        uint32_t kcur = 32u;
                        float racc = 0.f;
#pragma unroll
                        for (int c = 0; c < NC; c++) {
                            if (dv[c] != 0.f) {
                                const uint32_t k = k_of(exp_offset(TIw[c], tjf));
                                if (k != kcur) {
                                    if (kcur < 32u)
                                        tgr[tg_slot(kcur, lane)] = racc;
                                    kcur = k;
                                    racc = 0.f;
                                }
                                racc += dv[c];
                            }
                        }
                        if (kcur < 32u)
                            tgr[tg_slot(kcur, lane)] = racc;
                    }
                    __syncwarp();
                    float sum = 0.f;
#pragma unroll
                    for (int l = 0; l < 32; l++)
                        sum += TGw[l * 32 + tg_slot((uint32_t)lane, l)];
                    hacc += sum;
                }
#pragma unroll
                for (int c = 0; c < NC; c += 2)
                    dk[c >> 1] = pack_bf16(dv[c], dv[c + 1]);
            } else {
                // exact per-pair path: candidates, unsorted or far-apart stamps
#pragma unroll
                for (int c = 0; c < NC; c += 2) {
                    float pv[2], dsv[2];
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const int ii = iw0 + c + e;
                        pv[e] = 0.f;
                        dsv[e] = 0.f;
                        if (krow_ok && ii < L && visible_w(ii, j, hist, lw, gw, own)) {
                            const int idx = pos_index(token_pos(ii, hist, own), pj, lo, hi);
                            const int b = time_bucket(p.timestamps[s0 + ii], tj, p.nb);
                            const float hh = 0.5f * (sv[c + e] + p.rab_pos[hp + idx] + p.rab_time[ht + b]);
                            const float t = tanh_approx(hh);
                            pv[e] = fmaf(hh, t, hh);
                            const float ds = fmaf(dv[c + e], fmaf(hh, fmaf(-t, t, 1.f), t), dv[c + e]);
                            dsv[e] = ds;
                            red_add_global(p.d_rab_pos + hp + idx, ds * gscale);
                            red_add_global(p.d_rab_time + ht + b, ds * gscale);
                        }
                    }
                    pk[c >> 1] = pack_bf16(pv[0], pv[1]);
                    dk[c >> 1] = pack_bf16(dsv[0], dsv[1]);
                }
            }

            // the previous step's dQ, deferred so the gradient MMAs overlap this step's math
            if (i > 0 && !(ok = handle_dq(i - 1)))
                break;
            // P^T and dS'^T of this thread's row to TMEM, dS'^T also to shared
            // memory (K-major, 128B swizzle), once the previous step's gradient
            // and dQ MMAs have finished reading them
            if (i > 0 && !(ok = mbar_wait(bar(P_FREE), (i - 1) & 1, abort_flag, p.hdr)))
                break;
            tmem_st16(trow + COL_PT + (NC / 2) * g, pk);
            tmem_st16(trow + COL_DST + (NC / 2) * g, dk);
            unsigned char *drow = sm + BL::DST + r * 128;
#pragma unroll
            for (int u = 0; u < NC / 8; u++) {
                const int sw = ((NC / 8 * g + u) ^ (r & 7)) << 4;
                *reinterpret_cast<uint4 *>(drow + sw) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
            }
            tmem_wait_st();
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(P_FULL));
        }
        if (ok)
            ok = handle_dq(nq - 1);
        carry_flush(-1);
        if (hacc != 0.f)
            red_add_global(p.d_rab_time + ht + min(lane, p.nb - 1), hacc * gscale);
        {
            const float sh = warp_sum(cl_hi), sl = warp_sum(cl_lo);
            if (lane == 0 && sh != 0.f)
                red_add_global(p.d_rab_pos + hp + (hi - lo), sh * gscale);
            if (lane == 0 && sl != 0.f)
                red_add_global(p.d_rab_pos + hp, sl * gscale);
        }
        if (ok && mbar_wait(bar(ACC_FULL), 0, abort_flag, p.hdr)) {
            tc_fence_after();
            constexpr int DC = DH / kGroupsB;  // dK / dV columns per thread
            __nv_bfloat16 *gdk = static_cast<__nv_bfloat16 *>(p.dk) + (s0 + j) * p.sdk + (int64_t)h * DH + DC * g;
            __nv_bfloat16 *gdv = static_cast<__nv_bfloat16 *>(p.dvv) + (s0 + j) * p.sdv + (int64_t)h * DH + DC * g;
            if (kv_tma && j0 + 32 * quarter + 32 <= L) {
                // every key row of this warp in the sequence: [32 x 32] boxes staged
                // in the (now idle) Q / dO ring and written by TMA stores, instead
                // of 16-byte stores from every row
                unsigned char *stg = sm + BL::Q0 + ew * (2 * DC / 32) * 2048;
#pragma unroll
                for (int which = 0; which < 2; which++) {
                    const uint32_t col = (which ? COL_DV : COL_DK) + DC * g;
                    const float scale = which ? p.inv_n : gscale;
#pragma unroll
                    for (int cc = 0; cc < DC; cc += 32) {
                        float v[32];
                        tmem_ld32(trow + col + cc, v);
                        tmem_wait_ld();
                        unsigned char *box = stg + (which * (DC / 32) + cc / 32) * 2048;
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            uint4 w;
                            w.x = pack_bf16(v[8 * u] * scale, v[8 * u + 1] * scale);
                            w.y = pack_bf16(v[8 * u + 2] * scale, v[8 * u + 3] * scale);
                            w.z = pack_bf16(v[8 * u + 4] * scale, v[8 * u + 5] * scale);
                            w.w = pack_bf16(v[8 * u + 6] * scale, v[8 * u + 7] * scale);
                            *reinterpret_cast<uint4 *>(box + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) = w;
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int which = 0; which < 2; which++)
#pragma unroll
                        for (int cc = 0; cc < DC; cc += 32)
                            tma_store_2d(which ? &tmDV : &tmDK, h * DH + DC * g + cc, (int)(s0 + j0 + 32 * quarter),
                                         smem_u32(stg + (which * (DC / 32) + cc / 32) * 2048));
                    bulk_commit();
                }
            } else {
#pragma unroll
            for (int which = 0; which < 2; which++) {
                const uint32_t col = (which ? COL_DV : COL_DK) + DC * g;
                const float scale = which ? p.inv_n : gscale;
                __nv_bfloat16 *dst = which ? gdv : gdk;
#pragma unroll
                for (int cc = 0; cc < DC; cc += 32) {
                    float v[32];
                    tmem_ld32(trow + col + cc, v);
                    tmem_wait_ld();
                    if (krow_ok) {
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            uint4 w;
                            w.x = pack_bf16(v[8 * u] * scale, v[8 * u + 1] * scale);
                            w.y = pack_bf16(v[8 * u + 2] * scale, v[8 * u + 3] * scale);
                            w.z = pack_bf16(v[8 * u + 4] * scale, v[8 * u + 5] * scale);
                            w.w = pack_bf16(v[8 * u + 6] * scale, v[8 * u + 7] * scale);
                            *reinterpret_cast<uint4 *>(dst + cc + 8 * u) = w;
                        }
                    }
                }
            }
            }
        }
        if (lane == 0)
            bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemColsB);
}

// dQ (bf16, row stride sdq) = scale * the fp32 accumulator [T, H d]: eight
// elements per thread and iteration (two 16-byte loads, one 16-byte store);
// H d is a multiple of 64, so a group of eight never crosses a row.
__global__ void __launch_bounds__(256)
convert_dq_kernel(const float4 *__restrict__ acc, __nv_bfloat16 *__restrict__ dq, int64_t T, int hd, int64_t sdq,
                  float scale)
{
    const int64_t groups = T * (hd / 8);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < groups;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = e / (hd / 8);
        const int c = (int)(e - t * (hd / 8)) * 8;
        const float4 a = acc[2 * e], b = acc[2 * e + 1];
        uint4 w;
        w.x = pack_bf16(a.x * scale, a.y * scale);
        w.y = pack_bf16(a.z * scale, a.w * scale);
        w.z = pack_bf16(b.x * scale, b.y * scale);
        w.w = pack_bf16(b.z * scale, b.w * scale);
        *reinterpret_cast<uint4 *>(dq + t * sdq + c) = w;
    }
}

template <int DH>
cudaError_t bwd_tc_launch(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    CUtensorMap mk, mv, mq, mo, mdq;
    const int cols = p.H * DH;
    cudaError_t e = make_row_tensor_map(&mk, p.k, p.T, cols, p.sk);
    if (e == cudaSuccess)
        e = make_row_tensor_map(&mv, p.v, p.T, cols, p.sv);
    if (e == cudaSuccess)
        e = make_tensor_map_2d(&mq, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.T, cols, p.sq * 2, 64, QB,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_tensor_map_2d(&mo, p.dout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.T, cols, p.sdo * 2, 64, QB,
                               CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_tensor_map_2d(&mdq, p.dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.T, cols, (int64_t)cols * 4,
                               32, NC, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess)
        return e;
    const size_t bytes = BL<DH>::BYTES + 1024;
    // the extended bias readings (candidates at their own index, per-head tables)
    // are separate instantiations, so that the common case compiles without them
    const bool xb = (p.num_targets && p.cand_own) || p.pos_hstride;
    auto kern = xb ? (p.lw > 0 ? attn_bwd_tc_kernel<DH, true, true> : attn_bwd_tc_kernel<DH, false, true>)
                   : (p.lw > 0 ? attn_bwd_tc_kernel<DH, true> : attn_bwd_tc_kernel<DH, false>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess)
        return e;
    // Head-major order pays where a key tile's Q / dO / dQ rows leave L2 before
    // the sequence's next tile reads them: one sequence's tiles over all heads
    // do not fit one wave of CTAs, and the batch's rows (8 d bytes per token
    // and head) exceed twice the L2.  Windowed masks keep each tile's rows near
    // its keys, and short or few rows stay in L2 in tile order, where the heads
    // side by side balance better (same-process timings: head-major 10-34 %
    // faster on long-history batches, 3-19 % slower on short, Zipf and
    // windowed ones).
    const DeviceInfo info = device_info();
    const int sms = info.sms;
    const int64_t l2 = info.l2_bytes;
    const int64_t max_tiles = ((int64_t)p.max_seq_len + KB - 1) / KB;
    const int head_major = p.lw == 0 && max_tiles * p.H > sms && p.T * p.H * 8 * DH > 2 * l2;
    // dK and dV by TMA stores of [32 x 32] boxes where their rows are 16-byte aligned
    CUtensorMap mdk, mdv;
    memset(&mdk, 0, sizeof(mdk));
    memset(&mdv, 0, sizeof(mdv));
    int kv_tma = reinterpret_cast<uintptr_t>(p.dk) % 16 == 0 && reinterpret_cast<uintptr_t>(p.dvv) % 16 == 0 &&
                 (p.sdk * 2) % 16 == 0 && (p.sdv * 2) % 16 == 0;
    if (kv_tma && (make_tensor_map_2d(&mdk, p.dk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.T, cols, p.sdk * 2, 32, 32,
                                      CU_TENSOR_MAP_SWIZZLE_64B) != cudaSuccess ||
                   make_tensor_map_2d(&mdv, p.dvv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.T, cols, p.sdv * 2, 32, 32,
                                      CU_TENSOR_MAP_SWIZZLE_64B) != cudaSuccess))
        kv_tma = 0;
    kern<<<(unsigned)grid_items * p.H, kThreadsB, bytes, stream>>>(p, mk, mv, mq, mo, mdq, head_major, mdk, mdv,
                                                                     kv_tma);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_tc(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    if (grid_items <= 0 || p.T == 0)
        return cudaSuccess;
    return p.dqk == 64 ? bwd_tc_launch<64>(p, grid_items, stream) : bwd_tc_launch<128>(p, grid_items, stream);
}

cudaError_t launch_convert_dq(const float *acc, void *dq, int64_t T, int H, int d, int64_t sdq,
                              float scale, cudaStream_t stream)
{
    if (T == 0)
        return cudaSuccess;
    // 16-byte stores: the caller's dq rows start on 16-byte boundaries
    if ((H * d) % 8 || sdq % 8 || (reinterpret_cast<uintptr_t>(dq) & 15u))
        return cudaErrorInvalidValue;
    const int64_t groups = T * (H * d / 8);
    const int blocks = (int)std::min<int64_t>((groups + 255) / 256, (int64_t)device_info().sms * 8);
    convert_dq_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4 *>(acc),
                                                  static_cast<__nv_bfloat16 *>(dq), T, H * d, sdq, scale);
    return cudaGetLastError();
}

}  // namespace hstu
