// noalloc.cu -- sgq_gemv_thresh_noalloc: the fused threshold + sparse GEMV for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all, or cannot at the moment they
// run the GEMV: code running under an allocator that must not be re-entered,
// a plugin inside a host framework that owns all device memory, a path that
// must never fail for lack of memory in the middle of a decode step. For them
// the split-K partial sums live in a fixed-size array compiled into this
// library instead of a caller-provided workspace. Inputs and outputs are still
// the caller's.
//
// The array, g_noalloc_scratch, is a file-scope __device__ variable: every GPU
// that loads the library holds SGQ_NOALLOC_MAX_N floats (256 KB) for it until
// the process exits. In host code its name is only a host-side stand-in for
// the variable, not a device address, so the first call on each device (with
// that device current) looks up the real address with cudaGetSymbolAddress,
// once, under std::call_once, and caches it; later calls reuse the cached
// address. That first call makes a runtime query and should come before any
// stream capture. The address stays valid until the process exits or the
// device is reset (cudaDeviceReset): do not use this entry point across a
// reset.
//
// Every call first clears the N floats it uses with cudaMemsetAsync on the
// caller's stream (so the sums start from zero whatever an earlier call left
// behind, in stream order with the GEMV), then runs the GEMV, whose epilogue
// kernel leaves them at zero again. All calls on a device share the one
// array: calls that overlap on the GPU (two streams, or two host threads on
// one device without ordering between them) race on it.
#include "sgq_launch.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

static __device__ __align__(256) float g_noalloc_scratch[SGQ_NOALLOC_MAX_N];

namespace {

constexpr int kMaxDevices = 64;
std::once_flag g_setup_once[kMaxDevices];
float *g_scratch_addr[kMaxDevices];   // device address per device (set once)
cudaError_t g_setup_err[kMaxDevices]; // result of that device's set-up

// The host-side checks that sgq_gemv_thresh makes before it launches anything,
// so that the clear below is enqueued only for a call that will run.
bool launchable(const void *qweight, const void *sz, int N, int K, int group, const void *x,
                const void *y, const float *y_f32)
{
    auto a16 = [](const void *p) { return ((uintptr_t)p & 15u) == 0; };
    return (group == 32 || group == 64 || group == 128) && N > 0 && K > 0 && N % 32 == 0 &&
           K % group == 0 && K % 8 == 0 && qweight && sz && x && y && a16(qweight) &&
           a16(sz) && a16(x) && a16(y) && (!y_f32 || a16(y_f32));
}

} // namespace

extern "C" int sgq_gemv_thresh_noalloc(const void *qweight, const void *sz, int N, int K,
                                       int group, const void *x, float t, void *y,
                                       float *y_f32, int32_t *status, void *stream)
{
    if (N > SGQ_NOALLOC_MAX_N)
        return SGQ_ERR_TOO_LARGE;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return sgq::record_cuda_error(e);
    if (dev < 0 || dev >= kMaxDevices)
        return SGQ_ERR_DEVICE;
    std::call_once(g_setup_once[dev], [dev]() {
        void *addr = nullptr;
        g_setup_err[dev] = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
        if (g_setup_err[dev] == cudaSuccess)
            g_scratch_addr[dev] = static_cast<float *>(addr);
    });
    if (g_setup_err[dev] != cudaSuccess)
        return sgq::record_cuda_error(g_setup_err[dev]);
    if (launchable(qweight, sz, N, K, group, x, y, y_f32)) {
        e = cudaMemsetAsync(g_scratch_addr[dev], 0, (size_t)N * sizeof(float),
                            static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess)
            return sgq::record_cuda_error(e);
    }
    return sgq_gemv_thresh(qweight, sz, N, K, group, x, t, y, y_f32, g_scratch_addr[dev],
                           sizeof(g_noalloc_scratch), status, stream);
}
