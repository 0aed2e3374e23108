// Per-device host state of the launchers: the SM count, the opt-in dynamic
// shared-memory size and carveout of each kernel, and the driver's tensor-map
// encoder.
// A process may drive several GPUs, from several host threads: the SM count
// and the kernel attribute are kept per device (a function attribute set with
// one device current does not carry over to another), under one mutex.
#include <mutex>

#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kMaxDevices = 64;

std::mutex g_device_mutex;
int g_sms[kMaxDevices] = {};

// (kernel, device) pairs whose opt-in shared-memory limit has been raised,
// with the size it was raised to.
struct SmemAttr {
    const void* func;
    int device;
    int bytes;
};
constexpr int kMaxAttrs = 1024;
SmemAttr g_attrs[kMaxAttrs];
int g_nattrs = 0;

EncodeTiledFn lookup_encode() {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<EncodeTiledFn>(ptr);
    return nullptr;
}

}  // namespace

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lock(g_device_mutex);
    if (g_sms[dev] <= 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
        g_sms[dev] = sms;
    }
    return g_sms[dev];
}

cudaError_t ensure_dynamic_smem(const void* func, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_device_mutex);
    for (int i = 0; i < g_nattrs; ++i)
        if (g_attrs[i].func == func && g_attrs[i].device == dev && g_attrs[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    // Every kernel of the library asks for the largest shared-memory carveout,
    // so that an SM never has to change its L1 / shared split between two of
    // them (it can only do so when idle): a call's CTAs can then start on an
    // SM while the previous call's CTAs still run there.
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    for (int i = 0; i < g_nattrs; ++i)
        if (g_attrs[i].func == func && g_attrs[i].device == dev) {
            g_attrs[i].bytes = bytes;
            return cudaSuccess;
        }
    if (g_nattrs < kMaxAttrs) g_attrs[g_nattrs++] = SmemAttr{func, dev, bytes};
    return cudaSuccess;
}

EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = lookup_encode();  // (initialised once, thread-safe)
    return fn;
}

}  // namespace bq
