// Per-device attributes the launchers size their grids by, cached per device.
#include <mutex>

#include "internal.h"

namespace hstu {

namespace {

constexpr int kMaxDevices = 128;
std::mutex g_info_mutex;
DeviceInfo g_info[kMaxDevices];
bool g_info_valid[kMaxDevices] = {};

}  // namespace

DeviceInfo device_info()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0)
        dev = 0;
    DeviceInfo d;
    if (dev < kMaxDevices) {
        std::lock_guard<std::mutex> lock(g_info_mutex);
        if (g_info_valid[dev])
            return g_info[dev];
    }
    int sms = 0, l2 = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0)
        l2 = 126 << 20;
    d.sms = sms;
    d.l2_bytes = l2;
    if (dev < kMaxDevices) {
        std::lock_guard<std::mutex> lock(g_info_mutex);
        g_info[dev] = d;
        g_info_valid[dev] = true;
    }
    return d;
}

}  // namespace hstu
