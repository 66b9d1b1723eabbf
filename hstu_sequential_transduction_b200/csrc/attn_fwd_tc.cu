// HSTU jagged attention forward on sm_100a: TMA + tcgen05 (TMEM) kernel.
//
// Computes, per (sequence, 128-row query tile, head) work unit,
//   O = inv_n * sum_j SiLU(Q K_j^T + rab_pos + rab_time) V_j
// over the visible 128-row key tiles j (the pointwise attention of the
// "HSTU Architecture" section; causal block with appended candidates of the
// DLRMv4 page's "Model Architecture" section).  No score matrix reaches HBM.
// Persistent: one CTA per SM walks a share of the units, so the next unit's
// query and first key tiles load and its first S MMAs run while the epilogue
// still writes out the previous unit's O.
//
// Warp roles (320 threads):
//   warp 0     TMA producer: Q of each unit into one of two buffers, then K_j
//              and V_j into two-stage rings (separate K and V rings, so K_{j+2}
//              loads as soon as S_j is done);
//   warp 1     owns TMEM (512 columns) and issues every tcgen05.mma from one
//              thread: S_j = Q K_j^T into one of two S buffers, O += P_j V_j;
//   warps 2-9  epilogue: two groups of four warps (one per TMEM lane quarter),
//              each taking 64 of the 128 key columns of every S tile:
//              tcgen05.ld, relative bias, SiLU, bf16 pack, and tcgen05.st of P
//              over the first 32 of its own S columns, where the P V MMA reads
//              it as its A operand; at the end of a unit they read O from TMEM
//              and write it out.
// TMEM columns: S buffers [0,128) and [128,256), O [256, 256 + D).  S_{j+2}
// reuses buffer j % 2 once P_j V_j has completed.
//
// Epilogue arithmetic (stamps rebased to the query tile's first stamp, within
// 2^24 s, and sorted within the warp's key columns):
//   h = s/2 + rab_pos/2 + rab_time/2       (tables pre-halved, exact)
//   SiLU(x) = x sigma(x) = h (1 + tanh h)  (one MUFU tanh per score)
// The positional term reads the warp's 96-entry window of the clamped table
// (index p_i - p_j, contiguous along a row), or one constant when every
// column of the block is past a clamp.  The temporal bucket
// floor(log2(1 + dt)) is the exponent of the fp32 difference (t_i + 1) - t_j,
// computed with round-toward-zero so the exponent is exact; a row whose
// columns fall in one bucket adds that bucket's bias, a row spanning two picks
// one of two by comparing the key stamp against a per-row limit, and any other
// row maps the exponent through a 512-entry table to rab_time/2.  Diagonal and
// ragged tiles without candidate rows keep this arithmetic under a per-column
// mask; candidate rows (their own tile, and tiles mixing them with history
// rows), unsorted stamps and stamps more than 2^24 s apart take out-of-line
// exact per-pair paths (int64 bucket).  The candidate-position and per-head
// table options compile into separate instantiations.
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.h"
#include "tc_common.cuh"

namespace hstu {

namespace {

constexpr int TBM = 128, TBN = 128;
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreadsTc = kEpiThreads + 64;
constexpr uint32_t kTmemCols = 512;
constexpr int kRegion = 16384;  // one 128-row x 128-byte swizzled region

// Every barrier that can be waited on more than once per work item comes in
// pairs, one per buffer, so that no wait ever sees its barrier two phases on.
// Q_FULL / Q_EMPTY + b: query buffer b loaded / read by its last S MMA;
// K_*, V_*, S_FULL, P_FULL + b: the tile in stage / S buffer b;
// P_FREE + b: P V of the tile in S buffer b has completed (buffer b is free);
// O_FULL: a work item's O is complete in TMEM; O_FREE: the epilogue has read it.
// E_DONE / E_READY: with per-head tables, every epilogue warp is done with the
// previous head's time table / has filled its part of the next one.
enum Bars { Q_FULL = 0, Q_EMPTY = 2, K_FULL = 4, K_EMPTY = 6, V_FULL = 8, V_EMPTY = 10, S_FULL = 12,
            P_FULL = 14, P_FREE = 16, O_FULL = 18, O_FREE = 19, E_DONE = 20, E_READY = 21, NBARS = 22 };

// F8: Q and K tiles are E4M3 codes (one 128-byte region for D = 128)
template <int D, bool F8 = false, bool CAND = false>
struct FwdLayout {
    static constexpr int NREG = D / 64;
    static constexpr int TILE = NREG * kRegion;       // a bf16 tile (V; Q and K unless F8)
    static constexpr int QKT = F8 ? kRegion : TILE;   // a Q or K tile
    static constexpr int Q = 0;                 // two query buffers
    static constexpr int K0 = Q + 2 * QKT;
    static constexpr int V0 = K0 + 2 * QKT;
    // CAND: per epilogue warp, a [32 rows x 32 columns] bf16 box of O (64-byte
    // swizzle) on its way to a TMA store
    static constexpr int OST = V0 + 2 * TILE;
    static constexpr int E = OST + (CAND ? kEpiWarps * 2048 : 0);
    // per epilogue warp: 64 key stamps + 96-entry positional-bias window of a tile
    // (+ 64 key scales / 2 with F8)
    static constexpr int PW = E + 512 * 4;
    static constexpr int PW_FLOATS = 64 + 96 + (F8 ? 64 : 0);
    static constexpr int BAR = PW + kEpiWarps * PW_FLOATS * 4;
    static constexpr int MISC = BAR + NBARS * 8;
    static constexpr int BYTES = MISC + 64;
    static_assert(BYTES + 1024 <= 227 * 1024, "forward tile does not fit in shared memory");
};

__device__ __forceinline__ float time_bias_fast(float ti1, float tj, const float *E)
{
    const float d = __fsub_rz(ti1, tj);
    const uint32_t off = (__float_as_uint(d) >> 21) & 0x7FCu;
    return *reinterpret_cast<const float *>(reinterpret_cast<const char *>(E) + off);
}

// P for the 64 key columns one thread owns (one query row), packed to bf16.
// wr[-c]: positional bias / 2 of column c; tj[c]: rebased key stamp.
// MASK: only columns c_lo <= c < c_lim are visible.
// MODE: 0 time bucket looked up per column, 1 one bucket for the whole row
// (e_hi), 2 two buckets: e_hi for the columns whose key stamp is at most klim
// (those whose difference reaches the upper bucket), e_lo for the others.  CONSTB: the positional index is clamped
// for every column, so the positional bias is wr[0].
// F8: the raw score is dec(q) . dec(k) without the row scales; column c's half
// scale is ks[c] and the row's scale rsq, so h = s rsq ks[c] + bias / 2.
template <bool MASK, int MODE, bool CONSTB, bool F8 = false>
__device__ __forceinline__ void fwd_row(float *sv, const float *wr, const float *tj, float ti1,
                                        const float *E, float e_hi, float e_lo, float klim, int c_lo, int c_lim,
                                        uint32_t *pk, const float *ks = nullptr, float rsq = 0.f)
{
    const float bconst = CONSTB ? wr[0] + (MODE == 1 ? e_hi : 0.f) : 0.f;
    // three passes per 32 columns (biased half-scores, tanh, products) so the
    // independent per-column chains issue back to back
#pragma unroll
    for (int hb = 0; hb < 64; hb += 32) {
#pragma unroll
        for (int u = 0; u < 8; u++) {
            float tv[4], kf[4];
            if (F8) {
                const float4 k4 = *reinterpret_cast<const float4 *>(ks + hb + 4 * u);  // shared by the warp
                kf[0] = rsq * k4.x;
                kf[1] = rsq * k4.y;
                kf[2] = rsq * k4.z;
                kf[3] = rsq * k4.w;
            }
            if (MODE != 1) {
                const float4 t4 = *reinterpret_cast<const float4 *>(tj + hb + 4 * u);  // shared by the warp
                tv[0] = t4.x;
                tv[1] = t4.y;
                tv[2] = t4.z;
                tv[3] = t4.w;
            }
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int cc = hb + 4 * u + e;
                const float sc = F8 ? kf[e] : 0.5f;
                if (CONSTB && MODE == 1) {
                    sv[cc] = fmaf(sv[cc], sc, bconst);
                    continue;
                }
                float bt;
                if (MODE == 1)
                    bt = e_hi;
                else if (MODE == 2)
                    bt = tv[e] <= klim ? e_hi : e_lo;
                else
                    bt = time_bias_fast(ti1, tv[e], E);
                sv[cc] = fmaf(sv[cc], sc, CONSTB ? wr[0] : wr[-cc]) + bt;
            }
        }
        float th[32];
#pragma unroll
        for (int c = 0; c < 32; c++)
            th[c] = tanh_approx(sv[hb + c]);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
            float pv[2];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int cc = hb + c + e;
                float v = fmaf(sv[cc], th[c + e], sv[cc]);
                if (MASK)
                    v = (cc >= c_lo && cc < c_lim) ? v : 0.f;
                pv[e] = v;
            }
            pk[(hb + c) >> 1] = pack_bf16(pv[0], pv[1]);
        }
    }
}

// The two rare tile kinds, kept out of line so that the common tile loop stays
// small.  Both read this thread's 64 S columns from TMEM at taddr and write P
// (bf16) back over the first 32 of them.
//
// Exact per-pair rule: candidate rows, unsorted or far-apart stamps.  ts points
// at the sequence's stamps; jc0 is the key index of the thread's first column.
template <bool F8>
__device__ __noinline__ void p_tile_exact(uint32_t taddr, int i, bool row_ok, int jc0, int L, int hist, int lw,
                                          int gw, bool own, int pi, int64_t ti, const int64_t *ts, const float *rab_pos,
                                          const float *rab_time, int pos_lo, int pos_hi, int nb, float rsq,
                                          const float *KSw)
{
    float sv[64];
    tmem_ld32(taddr, sv);
    tmem_ld32(taddr + 32, sv + 32);
    tmem_wait_ld();
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 64; c += 2) {
        float pv[2];
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int j = jc0 + c + e;
            pv[e] = 0.f;
            if (row_ok && j < L && visible_w(i, j, hist, lw, gw, own)) {
                const float bp = rab_pos[pos_index(pi, token_pos(j, hist, own), pos_lo, pos_hi)];
                const float bt = rab_time[time_bucket(ti, ts[j], nb)];
                const float sr = F8 ? sv[c + e] * (2.f * rsq * KSw[c + e]) : sv[c + e];
                const float hh = 0.5f * (sr + bp + bt);
                pv[e] = fmaf(hh, tanh_approx(hh), hh);
            }
        }
        pk[c >> 1] = pack_bf16(pv[0], pv[1]);
    }
    tmem_st16(taddr, pk);
    tmem_st16(taddr + 16, pk + 16);
}

// The candidates' own tile: a candidate sees only itself, at position and time
// difference 0, so every row has the same bias bself; cd is the row's own column
// among the thread's 64 (outside [0, 64): none).
template <bool F8>
__device__ __noinline__ void p_tile_own(uint32_t taddr, int cd, bool row_ok, float bself, float rsq,
                                        const float *KSw)
{
    float sv[64];
    tmem_ld32(taddr, sv);
    tmem_ld32(taddr + 32, sv + 32);
    tmem_wait_ld();
    float sd = 0.f;
#pragma unroll
    for (int c = 0; c < 64; c++)
        sd = c == cd ? sv[c] : sd;
    float pd = 0.f;
    if (row_ok && cd >= 0 && cd < 64) {
        const float sr = F8 ? sd * (2.f * rsq * KSw[cd]) : sd;
        const float hh = 0.5f * (sr + bself);
        pd = fmaf(hh, tanh_approx(hh), hh);
    }
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 64; c += 2)
        pk[c >> 1] = pack_bf16(c == cd ? pd : 0.f, c + 1 == cd ? pd : 0.f);
    tmem_st16(taddr, pk);
    tmem_st16(taddr + 16, pk + 16);
}

// SL: semi-local windows in use (otherwise every window test compiles away);
// F8: S = Q K^T on E4M3 codes (tq, tk map the codes), rescaled in the epilogue;
// CAND: the batch has candidate rows (the candidates' own tiles take their own
// path, O leaves through TMA stores); the instantiation without them keeps the
// leaner tile loop
template <int D, bool SL, bool F8 = false, bool CAND = false, bool XB = false>
__global__ void __launch_bounds__(kThreadsTc, 1)
attn_fwd_tc_kernel(const AttnParams p, const __grid_constant__ CUtensorMap tq,
                   const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                   const __grid_constant__ CUtensorMap to, int o_tma)
{
    using LY = FwdLayout<D, F8, CAND>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);

    // Persistent: each CTA takes one unit per round of gridDim.x units of the
    // scheduler's (cost-ordered) list, unit w = (item w / H, head w % H).  Every
    // role walks the same units; `g` below counts K/V/S tiles across them.
    const int n_units = p.hdr->n_items * p.H;
    // the u-th unit of this CTA: rounds of gridDim.x units, alternating direction,
    // so that over the cost-ordered list every CTA gets a similar total
    auto unit_index = [&](int u) {
        const int G = (int)gridDim.x, b = (int)blockIdx.x;
        return u * G + ((u & 1) ? G - 1 - b : b);
    };
    const int lw = SL ? p.lw : 0, gw = SL ? p.gw : 0;
    struct Unit {
        int64_t s0;
        int L, hist, qt, i0, h, gt, lt0, nhist, ntiles;
        __device__ int tile_of(int t) const { return t >= nhist ? qt : (t < gt ? t : t - gt + lt0); }
    };
    auto unit = [&](int w) {
        Unit U;
        const int2 it = p.items[w / p.H];
        U.h = w % p.H;
        U.qt = it.y;
        U.s0 = p.seq_offsets[it.x];
        U.L = (int)(p.seq_offsets[it.x + 1] - U.s0);
        U.hist = U.L - (p.num_targets ? p.num_targets[it.x] : 0);
        U.i0 = U.qt * TBM;
        const int nh = (U.hist + TBN - 1) / TBN;
        const int nfull = min(U.qt + 1, nh);  // history key tiles up to this query tile
        // Semi-local windows: of those, the tiles holding global keys [0, gt) and the
        // tiles reaching into the local window of the tile's first row [lt0, nfull).
        U.gt = nfull;
        U.lt0 = nfull;
        if (lw > 0) {
            U.gt = min(nfull, (gw + TBN - 1) / TBN);
            U.lt0 = min(nfull, max(U.gt, max(0, token_pos(U.i0, U.hist, XB && p.cand_own) - lw + 1) / TBN));
        }
        U.nhist = U.gt + (nfull - U.lt0);
        U.ntiles = U.nhist + (U.qt >= nh ? 1 : 0);  // + the candidates' own tile
        return U;
    };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) { return base + LY::BAR + 8u * i; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + LY::MISC + 8);
    float *E = reinterpret_cast<float *>(sm + LY::E);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBARS; i++) {
            const bool epi = (i == P_FULL || i == P_FULL + 1 || i == O_FREE || i == E_DONE || i == E_READY);
            mbar_init(bar(i), epi ? kEpiWarps : 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch(&tq);
        tma_prefetch(&tk);
        tma_prefetch(&tv);
    }
    if (warp == 1)
        tmem_alloc(base + LY::MISC, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + LY::MISC);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            bool ok = true;
            int g = 0;
            for (int u = 0, w = unit_index(0); ok && w < n_units; u++, w = unit_index(u)) {
                const Unit U = unit(w);
                const int qs = u & 1;
                if (u >= 2 && !(ok = mbar_wait(bar(Q_EMPTY + qs), ((u >> 1) - 1) & 1, abort_flag, p.hdr, p.wait_limit)))
                    break;
                mbar_expect_tx(bar(Q_FULL + qs), LY::QKT);
                for (int r = 0; r < LY::QKT / kRegion; r++)
                    tma_load_2d(base + LY::Q + qs * LY::QKT + r * kRegion, &tq, U.h * D + 64 * r,
                                (int)(U.s0 + U.i0), bar(Q_FULL + qs));
                for (int t = 0; t < U.ntiles; t++, g++) {
                    const int s = g & 1;
                    const int j0 = U.tile_of(t) * TBN;
                    if (g >= 2 && !(ok = mbar_wait(bar(K_EMPTY + s), ((g >> 1) - 1) & 1, abort_flag, p.hdr, p.wait_limit)))
                        break;
                    // test hook: CTA 0 never loads its first key tile, so the waits on
                    // it run out (every load that is issued still completes)
                    if (g == 0 && p.withhold_first_k && blockIdx.x == 0)
                        continue;
                    mbar_expect_tx(bar(K_FULL + s), LY::QKT);
                    for (int r = 0; r < LY::QKT / kRegion; r++)
                        tma_load_2d(base + LY::K0 + s * LY::QKT + r * kRegion, &tk, U.h * D + 64 * r,
                                    (int)(U.s0 + j0), bar(K_FULL + s));
                    if (g >= 2 && !(ok = mbar_wait(bar(V_EMPTY + s), ((g >> 1) - 1) & 1, abort_flag, p.hdr, p.wait_limit)))
                        break;
                    mbar_expect_tx(bar(V_FULL + s), LY::TILE);
                    for (int r = 0; r < LY::NREG; r++)
                        tma_load_2d(base + LY::V0 + s * LY::TILE + r * kRegion, &tv, U.h * D + 64 * r,
                                    (int)(U.s0 + j0), bar(V_FULL + s));
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(TBM, TBN, 0, 0);
            constexpr uint32_t idO = idesc_bf16(TBM, D, 0, 1);
            // S of tile g (query buffer qs) into S buffer g % 2
            auto issue_S = [&](int g, int qs) {
                const int s = g & 1;
                if (F8) {  // E4M3: 32 codes (32 bytes) of K per MMA, one 128-byte region
                    constexpr uint32_t idS8 = idesc_e4m3(TBM, TBN, 0, 0);
                    for (int ks = 0; ks < D / 32; ks++) {
                        const uint64_t a = smem_desc_sw128(base + LY::Q + qs * LY::QKT + ks * 32, 16, 1024);
                        const uint64_t b = smem_desc_sw128(base + LY::K0 + s * LY::QKT + ks * 32, 16, 1024);
                        umma_e4m3(tmem + s * TBN, a, b, idS8, ks > 0);
                    }
                } else {
                    for (int ks = 0; ks < D / 16; ks++) {
                        const uint32_t off = (ks >> 2) * kRegion + (ks & 3) * 32;
                        const uint64_t a = smem_desc_sw128(base + LY::Q + qs * LY::TILE + off, 16, 1024);
                        const uint64_t b = smem_desc_sw128(base + LY::K0 + s * LY::TILE + off, 16, 1024);
                        umma_bf16(tmem + s * TBN, a, b, idS, ks > 0);
                    }
                }
                umma_commit(bar(K_EMPTY + s));
                umma_commit(bar(S_FULL + s));
            };
            // O (+)= P_g V_g; `first` starts a work item's accumulator
            auto issue_PV = [&](int g, bool first) {
                const int s = g & 1;
                // A = P_g from TMEM: keys 16 ks .. sit in S buffer columns 64 (ks / 4) + 8 (ks % 4)
                for (int ks = 0; ks < TBN / 16; ks++) {
                    const uint64_t b = smem_desc_sw128(base + LY::V0 + s * LY::TILE + ks * 2048, kRegion, 1024);
                    umma_bf16_ts(tmem + 2 * TBN, tmem + s * TBN + 64 * (ks >> 2) + 8 * (ks & 3), b, idO,
                                 (!first || ks > 0));
                }
                umma_commit(bar(V_EMPTY + s));
                umma_commit(bar(P_FREE + s));
            };
            // S buffer g % 2 is free once P V of tile g - 2 has completed
            auto s_free = [&](int g) {
                return g < 2 || mbar_wait(bar(P_FREE + (g & 1)), ((g >> 1) - 1) & 1, abort_flag, p.hdr, p.wait_limit);
            };
            bool ok = true;
            int gb = 0;  // first tile of the current unit
            for (int u = 0, w = unit_index(0); ok && w < n_units; u++, w = unit_index(u)) {
                const Unit U = unit(w);
                const int qs = u & 1, nt = U.ntiles;
                if (!(ok = mbar_wait(bar(Q_FULL + qs), (u >> 1) & 1, abort_flag, p.hdr, p.wait_limit)))
                    break;
                for (int t = 0; ok && t < min(2, nt); t++) {
                    const int g = gb + t;
                    ok = s_free(g) && mbar_wait(bar(K_FULL + (g & 1)), (g >> 1) & 1, abort_flag, p.hdr, p.wait_limit);
                    if (ok) {
                        tc_fence_after();
                        issue_S(g, qs);
                    }
                }
                if (ok && nt <= 2)
                    umma_commit(bar(Q_EMPTY + qs));
                // the previous unit's O has been read out of TMEM
                if (ok && u >= 1)
                    ok = mbar_wait(bar(O_FREE), (u - 1) & 1, abort_flag, p.hdr, p.wait_limit);
                for (int j = 0; ok && j < nt; j++) {
                    const int g = gb + j;
                    ok = mbar_wait(bar(P_FULL + (g & 1)), (g >> 1) & 1, abort_flag, p.hdr, p.wait_limit) &&
                         mbar_wait(bar(V_FULL + (g & 1)), (g >> 1) & 1, abort_flag, p.hdr, p.wait_limit);
                    if (!ok)
                        break;
                    tc_fence_after();
                    issue_PV(g, j == 0);
                    if (j + 2 < nt) {
                        ok = s_free(g + 2) &&
                             mbar_wait(bar(K_FULL + (g & 1)), ((g + 2) >> 1) & 1, abort_flag, p.hdr, p.wait_limit);
                        if (!ok)
                            break;
                        tc_fence_after();
                        issue_S(g + 2, qs);
                        if (j + 3 == nt)
                            umma_commit(bar(Q_EMPTY + qs));  // the unit's last S has been issued
                    }
                }
                if (ok)
                    umma_commit(bar(O_FULL));
                gb += nt;
            }
        }
    } else {
        // ---------------- epilogue ----------------
        // expanded time table (index = sign:exponent of the fp32 (1 + dt)), filled
        // while the first tiles load; only the epilogue warps read it
        // per-head tables: the table of the head in E (refilled when the head changes)
        auto fill_e = [&](int hh) {
            const float *rt = p.rab_time + hh * (int)p.time_hstride;
            for (int e = threadIdx.x - 64; e < 512; e += kEpiThreads) {
                const int bkt = (e >= 256 || e < 127) ? 0 : min(e - 127, p.nb - 1);
                E[e] = 0.5f * rt[bkt];
            }
        };
        fill_e(0);
        named_bar(1, kEpiThreads);
        int e_state = 0;  // head in E (bits 1..) and the refill barriers' phase (bit 0)
        const int ew = warp - 2, g = ew >> 2, quarter = warp & 3;
        const int r = quarter * 32 + lane;
        bool ok = true;
        int gtile = 0;  // tiles of this CTA so far (S buffer gtile % 2)
        for (int u = 0, w = unit_index(0); ok && w < n_units; u++, w = unit_index(u)) {
        const Unit U = unit(w);
        const int64_t s0 = U.s0;
        const int L = U.L, hist = U.hist, i0 = U.i0, h = U.h, ntiles = U.ntiles;
        const bool own = XB && p.cand_own != 0;
        // this head's rows of per-head tables (0 if shared)
        const int hp = XB ? h * (int)p.pos_hstride : 0, ht = XB ? h * (int)p.time_hstride : 0;
        if (XB && p.time_hstride && h != (e_state >> 1)) {
            // every epilogue warp reaches this unit: refill E once all are done with
            // it, through bounded waits (a warp that gave up makes the others give up)
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(E_DONE));
            if (!(ok = mbar_wait(bar(E_DONE), e_state & 1, abort_flag, p.hdr, p.wait_limit)))
                break;
            fill_e(h);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(E_READY));
            if (!(ok = mbar_wait(bar(E_READY), e_state & 1, abort_flag, p.hdr, p.wait_limit)))
                break;
            e_state = (h << 1) | (~e_state & 1);
        }
        auto tile_of = [&](int t) { return U.tile_of(t); };
        const int i = i0 + r;
        const bool row_ok = i < L;
        const int64_t tb = p.timestamps[s0 + i0];
        const int64_t ti = row_ok ? p.timestamps[s0 + i] : tb;
        const int pi = token_pos(i, hist, own);
        const int64_t lim = (int64_t)1 << 24;
        const uint32_t full_mask = 0xffffffffu;
        const bool qbad = __any_sync(full_mask, (ti - tb + 1 >= lim) || (ti - tb + 1 <= -lim));
        const float ti1f = (float)(ti - tb + 1);
        // this warp's 32 rows x 64 key columns of a tile: its own stamps and bias
        // window, so the loop needs no barrier wider than a warp
        float *TJw = reinterpret_cast<float *>(sm + LY::PW) + ew * LY::PW_FLOATS;  // key stamp - tb
        // Ww[m]: positional bias / 2 at offset pw - jw - 63 + m, pw = the warp's first row position
        // (positions grow with the row, candidates share one, so a row's pi - pw is in [0, 31])
        float *Ww = TJw + 64;
        float *KSw = Ww + 96;  // F8: half scales of the key columns
        // F8: this row's q scale
        const float rsq = F8 && row_ok ? p.sq8[(s0 + i) * p.H + h] : 0.f;
        const int pw = token_pos(i0 + 32 * quarter, hist, own);
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        auto clamp_idx = [&](int d) { return (d < p.pos_lo ? p.pos_lo : (d > p.pos_hi ? p.pos_hi : d)) - p.pos_lo; };

        // loads of the next tile's inputs; nothing here consumes a loaded value,
        // so the loads stay in flight while this tile is processed
        float w0 = 0.f, w1 = 0.f, w2 = 0.f;
        int64_t ta = tb, tc = tb;  // stamps of key columns 2 lane, 2 lane + 1
        float ka = 0.f, kc = 0.f;  // F8: scales of key columns 2 lane, 2 lane + 1
        auto prep = [&](int t) {
            const int jw = tile_of(t) * TBN + 64 * g;
            const int dbase = pw - jw - 63;
            w0 = p.rab_pos[hp + clamp_idx(dbase + lane)];
            w1 = p.rab_pos[hp + clamp_idx(dbase + lane + 32)];
            w2 = p.rab_pos[hp + clamp_idx(dbase + lane + 64)];
            const int j = jw + 2 * lane;
            ta = tb;
            tc = tb;
            if (j < L)
                ta = p.timestamps[s0 + j];
            if (j + 1 < L)
                tc = p.timestamps[s0 + j + 1];
            if (F8) {
                ka = j < L ? p.sk8[(s0 + j) * p.H + h] : 0.f;
                kc = j + 1 < L ? p.sk8[(s0 + j + 1) * p.H + h] : 0.f;
            }
        };
        prep(0);
        for (int t = 0; t < ntiles; t++, gtile++) {
            const int s = gtile & 1;
            const int j0 = tile_of(t) * TBN;
            const int j = j0 + 64 * g + 2 * lane;
            const int64_t ta_next = __shfl_down_sync(full_mask, ta, 1);
            const bool kbad = (j < L && (ta - tb >= lim || ta - tb <= -lim)) ||
                              (j + 1 < L && (tc - tb >= lim || tc - tb <= -lim));
            const bool kunsorted = (j + 1 < L && ta > tc) || (lane < 31 && j + 2 < L && tc > ta_next);
            const bool slow_time = __any_sync(full_mask, kbad) || qbad;
            const bool tj_sorted = !__any_sync(full_mask, kunsorted);
            __syncwarp();
            *reinterpret_cast<float2 *>(TJw + 2 * lane) = make_float2((float)(ta - tb), (float)(tc - tb));
            Ww[lane] = 0.5f * w0;
            Ww[lane + 32] = 0.5f * w1;
            Ww[lane + 64] = 0.5f * w2;
            if (F8)
                *reinterpret_cast<float2 *>(KSw + 2 * lane) = make_float2(0.5f * ka, 0.5f * kc);
            __syncwarp();
            // every pair of the tile inside the local window (or every key global)?
            const bool band_all = lw <= 0 || token_pos(min(i0 + TBM, L) - 1, hist, own) - j0 < lw ||
                                  j0 + TBN <= gw;
            const bool band_cut = !band_all;
            const bool full = (j0 + TBN <= hist) && (j0 + TBN - 1 <= i0) && band_all;
            if (t + 1 < ntiles)
                prep(t + 1);

            if (!(ok = mbar_wait(bar(S_FULL + s), (gtile >> 1) & 1, abort_flag, p.hdr, p.wait_limit)))
                break;
            tc_fence_after();
            float sv[64];
            tmem_ld32(trow + s * TBN + 64 * g, sv);
            tmem_ld32(trow + s * TBN + 64 * g + 32, sv + 32);
            tmem_wait_ld();

            uint32_t pk[32];
            bool stored = false;  // P already in TMEM (the out-of-line tile kinds)
            // diagonal / ragged tiles without candidate rows keep the fast math
            // with a per-column mask (positions equal indices there)
            // one interval of visible columns per row: no band cut inside global keys
            const bool masked_fast = !full && !slow_time && min(i0 + TBM, L) <= hist && (!band_cut || j0 >= gw);
            if ((full && !slow_time) || masked_fast) {
                const float *wr = Ww + (pi - pw) + 63;  // wr[-c]: key column c of this row
                const float *tj = TJw;
                if (full) {
                    // columns are sorted by time within the tile when the key
                    // stamps are; the row spans at most two buckets if the
                    // first and last differences are one exponent apart
                    const float dh = __fsub_rz(ti1f, tj[0]), dl = __fsub_rz(ti1f, tj[63]);
                    const uint32_t bh = __float_as_uint(dh) >> 23, bl = __float_as_uint(dl) >> 23;
                    const bool srt = tj_sorted && dl >= 1.f;
                    const bool one = __all_sync(0xffffffffu, !row_ok || (srt && bh == bl));
                    const bool two = __all_sync(0xffffffffu, !row_ok || (srt && bh - bl <= 1u));
                    // every column past the positional clamp (full tiles hold history keys only)
                    const int dnear = pi - (j0 + 64 * g + 63), dfar = pi - (j0 + 64 * g);
                    const bool cst = __all_sync(0xffffffffu, !row_ok || dnear >= p.pos_hi || dfar <= p.pos_lo);
                    const float e_hi = time_bias_fast(ti1f, tj[0], E), e_lo = time_bias_fast(ti1f, tj[63], E);
                    // two buckets: a column is in the upper one when RZ(ti - tj) >= 2^k
                    // (k = the bucket of the first column); stamps are integers and
                    // 2^k a power of two, so that is tj <= ti - 2^k exactly, i.e.
                    // tj <= RD(ti - 2^k): one compare per column
                    const float thr = __fsub_rd(ti1f, __uint_as_float(bh << 23));
                    if (one) {
                        if (cst)
                            fwd_row<false, 1, true, F8>(sv, wr, tj, ti1f, E, e_hi, e_lo, thr, 0, 64, pk, KSw, rsq);
                        else
                            fwd_row<false, 1, false, F8>(sv, wr, tj, ti1f, E, e_hi, e_lo, thr, 0, 64, pk, KSw, rsq);
                    } else if (two) {
                        if (cst)
                            fwd_row<false, 2, true, F8>(sv, wr, tj, ti1f, E, e_hi, e_lo, thr, 0, 64, pk, KSw, rsq);
                        else
                            fwd_row<false, 2, false, F8>(sv, wr, tj, ti1f, E, e_hi, e_lo, thr, 0, 64, pk, KSw, rsq);
                    } else {
                        fwd_row<false, 0, false, F8>(sv, wr, tj, ti1f, E, 0.f, 0.f, 0.f, 0, 64, pk, KSw, rsq);
                    }
                } else {
                    // visible: key j <= i, j < L and, when the tile crosses the local
                    // window's edge (no global keys here), j > i - local_window
                    const int c_lim = min(i - j0 - 64 * g + 1, L - j0 - 64 * g);
                    const int c_lo = band_cut ? i - lw + 1 - (j0 + 64 * g) : 0;
                    fwd_row<true, 0, false, F8>(sv, wr, tj, ti1f, E, 0.f, 0.f, 0.f, c_lo, c_lim, pk, KSw, rsq);
                }
            } else if (CAND && i0 >= hist && j0 == i0) {
                p_tile_own<F8>(trow + s * TBN + 64 * g, i - j0 - 64 * g, row_ok,
                               p.rab_pos[hp + pos_index(0, 0, p.pos_lo, p.pos_hi)] + p.rab_time[ht], rsq, KSw);
                stored = true;
            } else if (CAND) {
                p_tile_exact<F8>(trow + s * TBN + 64 * g, i, row_ok, j0 + 64 * g, L, hist, lw, gw, own, pi, ti,
                                 p.timestamps + s0, p.rab_pos + hp, p.rab_time + ht, p.pos_lo, p.pos_hi, p.nb, rsq, KSw);
                stored = true;
            } else {
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    float pv[2];
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const int j = j0 + 64 * g + c + e;
                        pv[e] = 0.f;
                        if (row_ok && j < L && visible_w(i, j, hist, lw, gw, own)) {
                            const float bp = p.rab_pos[hp + pos_index(pi, token_pos(j, hist, own), p.pos_lo, p.pos_hi)];
                            const float bt = p.rab_time[ht + time_bucket(ti, p.timestamps[s0 + j], p.nb)];
                            const float sr = F8 ? sv[c + e] * (2.f * rsq * KSw[c + e]) : sv[c + e];
                            const float hh = 0.5f * (sr + bp + bt);
                            pv[e] = fmaf(hh, tanh_approx(hh), hh);
                        }
                    }
                    pk[c >> 1] = pack_bf16(pv[0], pv[1]);
                }
            }
            // P over the first 32 of this thread's S columns (already read)
            if (!stored) {
                tmem_st16(trow + s * TBN + 64 * g, pk);
                tmem_st16(trow + s * TBN + 64 * g + 16, pk + 16);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(bar(P_FULL + s));
        }
        if (!(ok = ok && mbar_wait(bar(O_FULL), u & 1, abort_flag, p.hdr, p.wait_limit)))
            break;
        if (CAND && o_tma && i0 + 32 * quarter + 32 <= L) {
            // every row of this warp in the sequence: [32 x 32] boxes through shared
            // memory and one TMA store each (coalesced, one instruction per box)
            tc_fence_after();
            unsigned char *stg = sm + LY::OST + ew * 2048;
#pragma unroll
            for (int cc = 0; cc < D / 2; cc += 32) {
                float ov[32];
                tmem_ld32(trow + 2 * TBN + g * (D / 2) + cc, ov);
                tmem_wait_ld();
                uint4 packed[4];
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++)
                    packed[q4] = make_uint4(pack_bf16(ov[8 * q4] * p.inv_n, ov[8 * q4 + 1] * p.inv_n),
                                            pack_bf16(ov[8 * q4 + 2] * p.inv_n, ov[8 * q4 + 3] * p.inv_n),
                                            pack_bf16(ov[8 * q4 + 4] * p.inv_n, ov[8 * q4 + 5] * p.inv_n),
                                            pack_bf16(ov[8 * q4 + 6] * p.inv_n, ov[8 * q4 + 7] * p.inv_n));
                if (lane == 0)
                    bulk_wait_read0();  // the previous box has been read out
                __syncwarp();
#pragma unroll
                for (int q4 = 0; q4 < 4; q4++)
                    *reinterpret_cast<uint4 *>(stg + lane * 64 + ((q4 ^ ((lane >> 1) & 3)) << 4)) = packed[q4];
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&to, h * D + g * (D / 2) + cc, (int)(s0 + i0 + 32 * quarter), smem_u32(stg));
                    bulk_commit();
                }
            }
        } else {
            tc_fence_after();
            __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(p.o) + (s0 + i) * p.so + (int64_t)h * D + g * (D / 2);
#pragma unroll
            for (int cc = 0; cc < D / 2; cc += 32) {
                float ov[32];
                tmem_ld32(trow + 2 * TBN + g * (D / 2) + cc, ov);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; q4++) {
                        uint4 v;
                        v.x = pack_bf16(ov[8 * q4] * p.inv_n, ov[8 * q4 + 1] * p.inv_n);
                        v.y = pack_bf16(ov[8 * q4 + 2] * p.inv_n, ov[8 * q4 + 3] * p.inv_n);
                        v.z = pack_bf16(ov[8 * q4 + 4] * p.inv_n, ov[8 * q4 + 5] * p.inv_n);
                        v.w = pack_bf16(ov[8 * q4 + 6] * p.inv_n, ov[8 * q4 + 7] * p.inv_n);
                        *reinterpret_cast<uint4 *>(orow + cc + 8 * q4) = v;
                    }
                }
            }
        }
        // O has been read out of TMEM: the next unit's first P V may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(bar(O_FREE));
        }
        if (lane == 0)
            bulk_wait0();  // the O boxes have left shared memory
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    // looked up once per process (a function-local static: thread-safe)
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    return fn;
}

template <int D, bool SL, bool F8 = false, bool CAND = false, bool XB = false>
cudaError_t fwd_tc_launch(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    CUtensorMap maps[3];
    const void *ptrs[3] = {p.q, p.k, p.v};
    const int64_t strides[3] = {p.sq, p.sk, p.sv};
    cudaError_t e;
    if (F8) {  // E4M3 codes [T, H D] bytes: boxes of 128 codes x 128 rows
        e = make_tensor_map_2d(&maps[0], p.q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.T, p.H * D, (int64_t)p.H * D, 128,
                               128, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e == cudaSuccess)
            e = make_tensor_map_2d(&maps[1], p.k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.T, p.H * D, (int64_t)p.H * D,
                                   128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        e = make_row_tensor_map(&maps[0], ptrs[0], p.T, p.H * D, strides[0]);
        if (e == cudaSuccess)
            e = make_row_tensor_map(&maps[1], ptrs[1], p.T, p.H * D, strides[1]);
    }
    if (e == cudaSuccess)
        e = make_row_tensor_map(&maps[2], ptrs[2], p.T, p.H * D, strides[2]);
    if (e != cudaSuccess)
        return e;
    // O by TMA stores of [32 x 32] boxes where its rows are 16-byte aligned;
    // otherwise (and for warps whose rows run past the sequence) plain stores
    CUtensorMap mo;
    memset(&mo, 0, sizeof(mo));
    int o_tma = CAND && (reinterpret_cast<uintptr_t>(p.o) % 16 == 0) && (p.so * 2) % 16 == 0;
    if (o_tma && make_tensor_map_2d(&mo, p.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.T, p.H * D, p.so * 2, 32, 32,
                                    CU_TENSOR_MAP_SWIZZLE_64B) != cudaSuccess)
        o_tma = 0;
    const size_t bytes = FwdLayout<D, F8, CAND>::BYTES + 1024;
    e = cudaFuncSetAttribute(attn_fwd_tc_kernel<D, SL, F8, CAND, XB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)bytes);
    if (e != cudaSuccess)
        return e;
    // persistent: at most one CTA per SM, each walking its share of the work units
    const int sms = device_info().sms;
    const int64_t units = (int64_t)grid_items * p.H;
    const unsigned grid = (unsigned)std::min<int64_t>(units, sms);
    attn_fwd_tc_kernel<D, SL, F8, CAND, XB><<<grid, kThreadsTc, bytes, stream>>>(p, maps[0], maps[1], maps[2], mo, o_tma);
    return cudaGetLastError();
}

// The semi-local windows and the extended bias readings (candidates at their own
// index, per-head tables) are separate instantiations, so that the common case
// compiles without their bookkeeping.
template <int D, bool F8, bool CAND>
cudaError_t fwd_tc_pick(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    if ((CAND && p.cand_own) || p.pos_hstride)
        return p.lw > 0 ? fwd_tc_launch<D, true, F8, CAND, true>(p, grid_items, stream)
                        : fwd_tc_launch<D, false, F8, CAND, true>(p, grid_items, stream);
    return p.lw > 0 ? fwd_tc_launch<D, true, F8, CAND>(p, grid_items, stream)
                    : fwd_tc_launch<D, false, F8, CAND>(p, grid_items, stream);
}

}  // namespace

cudaError_t make_tensor_map_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype,
                               int64_t rows, int64_t cols, int64_t row_stride_bytes, int box_cols,
                               int box_rows, CUtensorMapSwizzle swizzle)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc)
        return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_row_tensor_map(CUtensorMap *map, const void *base, int64_t rows, int cols,
                                int64_t row_stride_elems)
{
    return make_tensor_map_2d(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rows, cols, row_stride_elems * 2,
                              64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool tensor_maps_available() { return tensor_map_encoder() != nullptr; }

bool attn_tc_supported(const AttnParams &p)
{
    return (p.dqk == 64 || p.dqk == 128) && p.dv == p.dqk && p.T >= 0 && p.T < ((int64_t)1 << 31) - 256;
}

cudaError_t launch_attn_fwd_tc(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    if (grid_items <= 0 || p.T == 0)
        return cudaSuccess;
    const bool cand = p.num_targets != nullptr;  // FP8 scores keep the one instantiation
    switch (p.dqk) {
    case 64:
        return cand ? fwd_tc_pick<64, false, true>(p, grid_items, stream)
                    : fwd_tc_pick<64, false, false>(p, grid_items, stream);
    case 128:
        if (p.q8)  // FP8 scores
            return fwd_tc_pick<128, true, false>(p, grid_items, stream);
        return cand ? fwd_tc_pick<128, false, true>(p, grid_items, stream)
                    : fwd_tc_pick<128, false, false>(p, grid_items, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace hstu
