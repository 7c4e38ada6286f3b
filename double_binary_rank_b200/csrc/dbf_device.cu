// Launch state shared by the launchers: the current device's SM count, the
// one-time kernel attributes (dynamic shared-memory limit, carve-out), and
// the grid-barrier time limit of the decode kernels. Both are properties of a device, so they are kept per device
// (a process may drive several GPUs, one host thread each), looked up under
// a lock and cached after the first call on each device.
#include "dbf_internal.cuh"

#include <atomic>
#include <map>
#include <mutex>
#include <utility>

namespace dbf {
namespace {

constexpr int kMaxDevices = 64;

std::mutex g_lock;
int g_sms[kMaxDevices] = {};
std::map<std::pair<int, const void *>, int> g_smem_set;   // (device, kernel) -> bytes already allowed

int current_device()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

std::atomic<unsigned long long> g_decode_wait_ns{0};   // 0: the default limit
constexpr unsigned long long kDecodeDefaultWaitNs = 2000000000ull;   // 2 s

}  // namespace

unsigned long long decode_wait_ns()
{
    const unsigned long long v = g_decode_wait_ns.load(std::memory_order_relaxed);
    return v ? v : kDecodeDefaultWaitNs;
}

void set_decode_wait_ns(unsigned long long ns) { g_decode_wait_ns.store(ns, std::memory_order_relaxed); }

int device_sms()
{
    const int dev = current_device();
    if (dev < 0) return 148;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_sms[dev]) {
        int v = 0;
        g_sms[dev] = (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) ? v : 148;
    }
    return g_sms[dev];
}

cudaError_t allow_smem(const void *kernel, int bytes, bool max_shared_carveout)
{
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> guard(g_lock);
    int &have = g_smem_set[std::make_pair(dev, kernel)];
    if (bytes <= have) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (max_shared_carveout) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
    }
    have = bytes;
    return cudaSuccess;
}

}  // namespace dbf
