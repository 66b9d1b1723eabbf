// HSTU jagged attention in fp32 on CUDA cores (the small fp32 workloads).
//
// Same definition as the bf16 kernels ("HSTU Architecture": SiLU weighting,
// relative positional + temporal bias, causal/candidate mask, 1/N), computed
// with IEEE fp32 arithmetic and the precise exponential.  One thread owns one
// query row; key/value tiles are staged in shared memory and read as
// broadcasts.  The backward uses the query-tile schedule and scatters dK, dV
// and the bias-table gradients with fp32 atomics.
#include "common.cuh"
#include "internal.h"

namespace hstu {

namespace {

constexpr int TR = kF32Tile;  // rows per tile (query and key)

struct SeqV {
    int64_t s0;
    int L, hist;
};

__device__ __forceinline__ SeqV seqv(const AttnParams &p, int b)
{
    SeqV s;
    s.s0 = p.seq_offsets[b];
    s.L = (int)(p.seq_offsets[b + 1] - s.s0);
    s.hist = s.L - (p.num_targets ? p.num_targets[b] : 0);
    return s;
}

__device__ __forceinline__ int ntiles_fwd(int qt, const SeqV &s)
{
    int nh = (s.hist + TR - 1) / TR;
    return min(qt + 1, nh) + (qt >= nh ? 1 : 0);
}

__device__ __forceinline__ int tile_fwd(int idx, int qt, const SeqV &s)
{
    int nh = (s.hist + TR - 1) / TR;
    return idx < min(qt + 1, nh) ? idx : qt;
}

template <int D>
__device__ __forceinline__ void stage(float *dst, const float *src, int64_t stride, const SeqV &s,
                                      int r0, int h)
{
    for (int e = threadIdx.x; e < TR * D; e += TR) {
        int r = e / D, c = e % D;
        dst[e] = r0 + r < s.L ? src[(s.s0 + r0 + r) * stride + (int64_t)h * D + c] : 0.f;
    }
}

template <int D>
__global__ void __launch_bounds__(TR) attn_fwd_f32_kernel(const AttnParams p)
{
    __shared__ float sK[TR * D], sV[TR * D];
    __shared__ int64_t sT[TR];
    const int item = blockIdx.x / p.H, h = blockIdx.x % p.H;
    if (item >= p.hdr->n_items)
        return;
    const int2 it = p.items[item];
    const SeqV s = seqv(p, it.x);
    const int qt = it.y;
    const int i = qt * TR + threadIdx.x;
    const bool row_ok = i < s.L;
    const float *gq = static_cast<const float *>(p.q);
    float q[D], o[D];
#pragma unroll
    for (int c = 0; c < D; c++) {
        q[c] = row_ok ? gq[(s.s0 + i) * p.sq + (int64_t)h * D + c] : 0.f;
        o[c] = 0.f;
    }
    const bool own = p.cand_own;
    const float *rab_pos = p.rab_pos + h * p.pos_hstride, *rab_time = p.rab_time + h * p.time_hstride;
    const int pi = token_pos(i, s.hist, own);
    const int64_t ti = row_ok ? p.timestamps[s.s0 + i] : 0;
    const int n = ntiles_fwd(qt, s);
    for (int idx = 0; idx < n; idx++) {
        const int j0 = tile_fwd(idx, qt, s) * TR;
        __syncthreads();
        stage<D>(sK, static_cast<const float *>(p.k), p.sk, s, j0, h);
        stage<D>(sV, static_cast<const float *>(p.v), p.sv, s, j0, h);
        sT[threadIdx.x] = j0 + (int)threadIdx.x < s.L ? p.timestamps[s.s0 + j0 + threadIdx.x] : 0;
        __syncthreads();
        for (int jj = 0; jj < TR; jj++) {
            const int j = j0 + jj;
            if (!row_ok || j >= s.L || !visible_w(i, j, s.hist, p.lw, p.gw, own))
                continue;
            float x = 0.f;
#pragma unroll
            for (int c = 0; c < D; c++)
                x = fmaf(q[c], sK[jj * D + c], x);
            x += rab_pos[pos_index(pi, token_pos(j, s.hist, own), p.pos_lo, p.pos_hi)] +
                 rab_time[time_bucket(ti, sT[jj], p.nb)];
            const float w = silu_precise(x) * p.inv_n;
#pragma unroll
            for (int c = 0; c < D; c++)
                o[c] = fmaf(w, sV[jj * D + c], o[c]);
        }
    }
    if (row_ok) {
        float *go = static_cast<float *>(p.o) + (s.s0 + i) * p.so + (int64_t)h * D;
#pragma unroll
        for (int c = 0; c < D; c++)
            go[c] = o[c];
    }
}

// dq written directly; dk, dv, d_rab_* accumulated with atomics (zeroed first).
template <int D>
__global__ void __launch_bounds__(TR) attn_bwd_f32_kernel(const AttnParams p)
{
    __shared__ float sK[TR * D], sV[TR * D];
    __shared__ int64_t sT[TR];
    const int item = blockIdx.x / p.H, h = blockIdx.x % p.H;
    if (item >= p.hdr->n_items)
        return;
    const int2 it = p.items[item];
    const SeqV s = seqv(p, it.x);
    const int qt = it.y;
    const int i = qt * TR + threadIdx.x;
    const bool row_ok = i < s.L;
    const float *gq = static_cast<const float *>(p.q);
    const float *gdo = static_cast<const float *>(p.dout);
    float *gdk = static_cast<float *>(p.dk);
    float *gdv = static_cast<float *>(p.dvv);
    float q[D], dq[D], dout[D];
#pragma unroll
    for (int c = 0; c < D; c++) {
        q[c] = row_ok ? gq[(s.s0 + i) * p.sq + (int64_t)h * D + c] : 0.f;
        dout[c] = row_ok ? gdo[(s.s0 + i) * p.sdo + (int64_t)h * D + c] : 0.f;
        dq[c] = 0.f;
    }
    const bool own = p.cand_own;
    const float *rab_pos = p.rab_pos + h * p.pos_hstride, *rab_time = p.rab_time + h * p.time_hstride;
    const int pi = token_pos(i, s.hist, own);
    const int64_t ti = row_ok ? p.timestamps[s.s0 + i] : 0;
    const int n = ntiles_fwd(qt, s);
    for (int idx = 0; idx < n; idx++) {
        const int j0 = tile_fwd(idx, qt, s) * TR;
        __syncthreads();
        stage<D>(sK, static_cast<const float *>(p.k), p.sk, s, j0, h);
        stage<D>(sV, static_cast<const float *>(p.v), p.sv, s, j0, h);
        sT[threadIdx.x] = j0 + (int)threadIdx.x < s.L ? p.timestamps[s.s0 + j0 + threadIdx.x] : 0;
        __syncthreads();
        for (int jj = 0; jj < TR; jj++) {
            const int j = j0 + jj;
            if (!row_ok || j >= s.L || !visible_w(i, j, s.hist, p.lw, p.gw, own))
                continue;
            float x = 0.f, dp = 0.f;
#pragma unroll
            for (int c = 0; c < D; c++) {
                x = fmaf(q[c], sK[jj * D + c], x);
                dp = fmaf(dout[c], sV[jj * D + c], dp);
            }
            const int pidx = pos_index(pi, token_pos(j, s.hist, own), p.pos_lo, p.pos_hi);
            const int bkt = time_bucket(ti, sT[jj], p.nb);
            x += rab_pos[pidx] + rab_time[bkt];
            const float w = silu_precise(x) * p.inv_n;
            const float ds = dp * silu_grad_precise(x) * p.inv_n;
            float *dkr = gdk + (s.s0 + j) * p.sdk + (int64_t)h * D;
            float *dvr = gdv + (s.s0 + j) * p.sdv + (int64_t)h * D;
#pragma unroll
            for (int c = 0; c < D; c++) {
                dq[c] = fmaf(ds, sK[jj * D + c], dq[c]);
                atomicAdd(dkr + c, ds * q[c]);
                atomicAdd(dvr + c, w * dout[c]);
            }
            atomicAdd(p.d_rab_pos + h * p.pos_hstride + pidx, ds);
            atomicAdd(p.d_rab_time + h * p.time_hstride + bkt, ds);
        }
    }
    if (row_ok) {
        float *gdq = static_cast<float *>(p.dq) + (s.s0 + i) * p.sdq + (int64_t)h * D;
#pragma unroll
        for (int c = 0; c < D; c++)
            gdq[c] = dq[c];
    }
}

}  // namespace

cudaError_t launch_attn_fwd_f32(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    if (grid_items <= 0)
        return cudaSuccess;
    const unsigned grid = (unsigned)grid_items * p.H;
    switch (p.dqk) {
    case 32: attn_fwd_f32_kernel<32><<<grid, TR, 0, stream>>>(p); break;
    case 64: attn_fwd_f32_kernel<64><<<grid, TR, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_attn_bwd_f32(const AttnParams &p, int grid_items, cudaStream_t stream)
{
    if (grid_items <= 0)
        return cudaSuccess;
    const unsigned grid = (unsigned)grid_items * p.H;
    switch (p.dqk) {
    case 32: attn_bwd_f32_kernel<32><<<grid, TR, 0, stream>>>(p); break;
    case 64: attn_bwd_f32_kernel<64><<<grid, TR, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace hstu
