// Attention forward for callers that cannot allocate device memory.
//
// hstu_attn_fwd needs a caller-provided workspace for its jagged tile
// scheduler (a 256-byte header plus the work list).  Some callers cannot
// provide one: a plugin running inside a host framework that owns every
// device allocation and hands the plugin nothing but its input and output
// buffers, or a latency-critical path where cudaMalloc is not allowed because
// it can synchronize the whole device.  For them, hstu_attn_fwd_noalloc keeps
// that scratch in one fixed, file-scope device array instead.
//
// The array is a static __device__ symbol: every GPU that loads this library
// holds it (kNoAllocScratchBytes, about 512 KiB) until the process exits.  Host
// code cannot use the symbol's name as a device address, so the first call on
// each device looks the address up with cudaGetSymbolAddress (with that device
// current) and caches it; that first call should come before any stream
// capture.  Every call shares the array and the array keeps the previous
// call's contents; nothing in it has to start at zero, because the scheduler
// rewrites the header and the work list before the attention kernel reads
// them.  Calls that overlap on the GPU (different streams, or different host
// threads on one device) race on the array and must be serialized by the
// caller.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

// Largest work list the static scratch holds: ceil(T / 64) + B items.
constexpr int kNoAllocMaxItems = 65536;
constexpr size_t kNoAllocScratchBytes = sizeof(hstu::WsHeader) + sizeof(int2) * kNoAllocMaxItems;
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
hstu_status scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return HSTU_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices)
        return HSTU_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return HSTU_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HSTU_OK;
}

}  // namespace

extern "C" hstu_status hstu_attn_fwd_noalloc(const hstu_attn_desc *desc, const void *q,
                                              const void *k, const void *v,
                                              const int64_t *seq_offsets,
                                              const int64_t *timestamps,
                                              const int32_t *num_targets, const float *rab_pos,
                                              const float *rab_time, void *out, void *stream)
{
    size_t need = 0;
    hstu_status st = hstu_attn_workspace_size(desc, 0, &need);
    if (st != HSTU_OK)
        return st;
    if (desc->fp8_qk)  // the FP8 codes need a caller's workspace
        return HSTU_ERR_UNSUPPORTED;
    if (need > kNoAllocScratchBytes)
        return HSTU_ERR_UNSUPPORTED;  // problem larger than the static scratch
    void *scratch = nullptr;
    st = scratch_address(&scratch);
    if (st != HSTU_OK)
        return st;
    return hstu_attn_fwd(desc, q, k, v, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                         out, scratch, kNoAllocScratchBytes, stream);
}
