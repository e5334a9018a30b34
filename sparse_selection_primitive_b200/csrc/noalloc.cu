// lapsum_backward_noalloc: the backward pass for callers that cannot hand the
// library a device workspace.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they need the gradient: code running while a CUDA graph is being captured
// with a strict no-allocation policy, real-time or embedded hosts whose
// memory is all reserved up front, and plugin hosts that own every device
// allocation themselves.  For them this entry point keeps its scratch memory
// in a fixed array that is part of the library image on every GPU that loads
// it, and so needs no workspace argument at all.
//
// The long-row backward (n > 4096) needs per-CTA partial sums, one ratio per
// row and one counter per row; those live in the array below.  Rows of up to
// 4096 scores use the on-chip kernel, which needs no scratch.
#include <cmath>
#include <mutex>

#include "lapsum_common.cuh"
#include "lapsum_kernels.h"

namespace lapsum {
namespace {

constexpr int kNoAllocRows = 1024;        // most rows per call
constexpr int kNoAllocRecords = 4096;     // most per-CTA partial records per call
constexpr int kNoAllocMaxDevices = 64;
constexpr size_t kPartialBytes = (size_t)kNoAllocRecords * 4 * sizeof(double);
constexpr size_t kRowBytes = (size_t)kNoAllocRows * sizeof(double);
constexpr size_t kTicketBytes = (size_t)kNoAllocRows * sizeof(uint32_t);
constexpr size_t kScratchBytes = kPartialBytes + kRowBytes + kTicketBytes;  // 140 KiB

// Shared by every call on a device; it keeps the contents of the last call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kNoAllocMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  Host code
// cannot use the symbol itself as a device pointer.  The address is looked up
// on every call made outside a stream capture (so that a device reset, which
// reloads the module and may move the array, leaves no stale address behind)
// and kept per device for calls made while a capture records the stream.
cudaError_t scratch_address(cudaStream_t st, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(g_mu);
    if (cap == cudaStreamCaptureStatusNone || g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace lapsum

using namespace lapsum;

extern "C" int lapsum_backward_noalloc(const float* r, int64_t ld, const double* b, const float* v,
                                       float* g, int64_t B, int64_t n, double t, void* stream) {
    if (r == nullptr || b == nullptr || v == nullptr || g == nullptr) return LAPSUM_EINVAL;
    if (B < 1 || n < 1 || ld < n) return LAPSUM_EINVAL;
    if (!(t > 0.0) || !std::isfinite(t)) return LAPSUM_EINVAL;
    if (B > kNoAllocRows) return LAPSUM_EINVAL;
    cudaStream_t st = (cudaStream_t)stream;
    const bool vec = ((reinterpret_cast<uintptr_t>(r) | reinterpret_cast<uintptr_t>(v) |
                       reinterpret_cast<uintptr_t>(g)) & 15u) == 0 && (ld % 4) == 0;
    if (n <= 4096)  // on-chip rows: no scratch at all
        return launch_onchip_backward(r, ld, b, v, g, B, (int)n, t, vec ? 1 : 0, st) == cudaSuccess
                   ? LAPSUM_OK
                   : LAPSUM_ECUDA;
    // The long-row reduction runs about 8 CTAs per SM over all rows; each CTA
    // leaves one record, and every record must fit in the array.
    // (the same per-device SM count sizes the launch's grid)
    if ((int64_t)device_sm_count() * 8 + B > kNoAllocRecords) return LAPSUM_EINVAL;
    void* base = nullptr;
    if (scratch_address(st, &base) != cudaSuccess) return LAPSUM_ECUDA;
    char* s = static_cast<char*>(base);
    double* partials = reinterpret_cast<double*>(s);
    double* row_R = reinterpret_cast<double*>(s + kPartialBytes);
    uint32_t* tickets = reinterpret_cast<uint32_t*>(s + kPartialBytes + kRowBytes);
    // the per-row last-CTA counters must start at zero
    if (cudaMemsetAsync(tickets, 0, (size_t)B * sizeof(uint32_t), st) != cudaSuccess)
        return LAPSUM_ECUDA;
    return launch_backward_stream(r, ld, b, v, g, B, n, t, partials, row_R, tickets, vec ? 1 : 0,
                                  st) == cudaSuccess
               ? LAPSUM_OK
               : LAPSUM_ECUDA;
}
