// noalloc.cu -- pararnn_linear_scan_noalloc: the diagonal / 2x2-block linear scan of
// pararnn_linear_scan without a context and without any device allocation.
//
// Some callers cannot call cudaMalloc: a host program whose device memory is owned by
// another allocator (a framework's caching pool, a pre-sized arena), a loop where the
// implicit synchronisation of cudaMalloc/cudaFree would stall the device, or a
// service that must not meet an out-of-memory error after start-up.  For them the
// scan's scratch (its control block and the look-back words) lives in one static
// device array below, which every device that loads this library holds until exit.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pararnn.h"
#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)16 << 20;  // PARARNN_NOALLOC_SCRATCH_BYTES
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a stand-in for the symbol: the
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
// Per device: the array's device address as last resolved and the next free epoch.
// A primary context that was torn down and created again (cudaDeviceReset) reloads the
// module, and the array may then sit elsewhere with new contents: every call resolves
// the address again, and a changed address restarts the epochs, which clears the array.
void *g_addr[kMaxDevices] = {};
unsigned long long g_epoch[kMaxDevices] = {};

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

extern "C" int pararnn_linear_scan_noalloc(int kind, const float *J, const float *b, const float *h0,
                                           float *h_out, int B, int T, int N, int reverse, int *status_out,
                                           void *cuda_stream) {
    if (!J || !b || !h_out || !status_out || B < 1 || T < 1 || N < 1 || (reverse != 0 && reverse != 1))
        return PARARNN_EINVAL;
    if (kind != PARARNN_SCAN_DIAG && kind != PARARNN_SCAN_BLOCK2) return PARARNN_EINVAL;
    auto mis = [](const void *p) { return p && ((uintptr_t)p & 15u); };
    if (mis(J) || mis(b) || mis(h0) || mis(h_out) || ((uintptr_t)status_out & 3u)) return PARARNN_EALIGN;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return PARARNN_ECUDA;
    }
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    prn::ScanReq r{kind, B, T, N, reverse, J, b, h0, h_out};
    prn::Plan plan;
    if (prn::scan_diag_plan(r, nsm, &plan)) return PARARNN_ECUDA;
    const size_t ctl_b = up256(sizeof(prn::Ctl));
    const size_t ag_b = up256(plan.agg_words * 8), in_b = up256(plan.inc_words * 8);
    if (ctl_b + ag_b + in_b > kScratchBytes) return PARARNN_ESCRATCH;

    std::lock_guard<std::mutex> lock(g_mu);
    // The array's device address on the current device (no allocation; cheap after the
    // module is loaded).
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) {
        cudaGetLastError();
        return PARARNN_ECUDA;
    }
    if (addr != g_addr[dev]) {
        g_addr[dev] = addr;
        g_epoch[dev] = 0;  // a new array (first call, or a re-created context): clear it below
    }
    char *base = static_cast<char *>(g_addr[dev]);
    prn::Work w;
    w.ctl = reinterpret_cast<prn::Ctl *>(base);
    w.sticky = status_out;
    w.agg = reinterpret_cast<unsigned long long *>(base + ctl_b);
    w.inc = reinterpret_cast<unsigned long long *>(base + ctl_b + ag_b);
    w.side = nullptr;
    // Look-back words persist from call to call and carry the epoch that wrote them.
    // A fresh epoch range per call keeps stale words from matching; the first call on
    // a device and every wrap of the 32-bit range clear them.
    if (g_epoch[dev] == 0 || g_epoch[dev] + plan.epochs + 2 >= 0xffffffffull) {
        if (cudaMemsetAsync(base + ctl_b, 0, kScratchBytes - ctl_b, st) != cudaSuccess)
            return PARARNN_ECUDA;
        g_epoch[dev] = 1;
    }
    w.epoch0 = (unsigned)g_epoch[dev];
    g_epoch[dev] += plan.epochs;
    if (cudaMemsetAsync(base, 0, ctl_b, st) != cudaSuccess) return PARARNN_ECUDA;
    if (cudaMemsetAsync(status_out, 0, sizeof(int), st) != cudaSuccess) return PARARNN_ECUDA;
    prn::DbgHost dbg;
    if (prn::scan_diag_launch(r, plan, w, dbg, st) != cudaSuccess) {
        cudaGetLastError();
        return PARARNN_ECUDA;
    }
    return PARARNN_OK;
}
