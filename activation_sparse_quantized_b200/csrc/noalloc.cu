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
// the variable, not a device address, so the first call on each device looks
// up the real address with cudaGetSymbolAddress (with that device current)
// and clears the array; later calls reuse the cached address. That first call
// synchronises with cudaMemset and must come before any stream capture. Every
// call leaves the entries it used at zero again (the epilogue kernel re-zeroes
// them), so the next call starts from zero; calls that overlap on the GPU (two
// streams, or two host threads on one device without ordering) share the
// array and race.
#include "sgq_launch.h"

#include <cuda_runtime.h>

static __device__ __align__(256) float g_noalloc_scratch[SGQ_NOALLOC_MAX_N];

namespace {

constexpr int kMaxDevices = 64;
float *g_scratch_addr[kMaxDevices]; // device address per device; nullptr = not set up

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
    if (!g_scratch_addr[dev]) {
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
        if (e != cudaSuccess)
            return sgq::record_cuda_error(e);
        e = cudaMemset(addr, 0, sizeof(g_noalloc_scratch));
        if (e != cudaSuccess)
            return sgq::record_cuda_error(e);
        g_scratch_addr[dev] = static_cast<float *>(addr);
    }
    return sgq_gemv_thresh(qweight, sz, N, K, group, x, t, y, y_f32, g_scratch_addr[dev],
                           sizeof(g_noalloc_scratch), status, stream);
}
