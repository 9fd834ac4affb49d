// noalloc.cu -- fp4_hessian_blocks_noalloc: the Hessian-block accumulation of
// fp4_hessian_blocks for callers that cannot allocate device memory.
//
// Who needs it: code that only holds the tensors it was handed and has no
// allocator of its own -- a plugin running inside another framework's
// pre-planned memory arena, a layer-streaming calibration loop that has
// budgeted every byte of the device, or a latency-sensitive path that must
// not call cudaMalloc because cudaMalloc can synchronize the whole device.
// fp4_hessian_blocks needs a caller-provided workspace for its per-chunk
// partial sums; this variant takes its scratch from a fixed array that lives
// in the library's own device memory instead.
//
// The scratch array is file-scope device memory of kScratchFloats floats
// (16 MiB); every GPU that loads the library holds it until the process
// exits.  The first call on each device looks up the array's device address
// on that device (cudaGetSymbolAddress); make that first call before any
// stream capture begins.  All calls share the array, so two calls whose
// kernels overlap on the GPU (different streams, or different host threads)
// race on it; order them on one stream.  Each call overwrites every partial
// it later reads, so nothing needs clearing between calls.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/fp4q.h"
#include "fp4q_internal.h"

namespace {

// 4096 partial 32x32 blocks of fp32 = 16 MiB: enough for 8192 tokens x 4096
// columns (32 chunks of 256 tokens x 128 column blocks).
constexpr size_t kScratchBlocks = 4096;
constexpr size_t kScratchFloats = kScratchBlocks * 1024;

static __device__ __align__(256) float g_hessian_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the host-side symbol is only a stand-in, not a device address).
int scratch_for_current_device(float** out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return FP4Q_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_hessian_scratch) != cudaSuccess || !p)
            return FP4Q_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_ptr[dev];
    return FP4Q_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int fp4_hessian_blocks_noalloc(const void* x, int dtype, int64_t rows, int64_t cols,
                               const float* chan_scale, int hadamard32, float* hess_blocks,
                               void* stream)
{
    if (!x || !hess_blocks || (dtype != FP4Q_F32 && dtype != FP4Q_BF16) || rows < 0 || cols < 0 ||
        cols % 32 != 0)
        return FP4Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(hess_blocks) ||
        (chan_scale && !aligned16(chan_scale)))
        return FP4Q_ERR_ALIGN;
    if (cols == 0)
        return FP4Q_OK;
    const size_t need = fp4q::hessian_ws_bytes(rows, cols);
    if (need > kScratchFloats * sizeof(float))
        return FP4Q_ERR_TOO_LARGE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0)
        return cudaMemsetAsync(hess_blocks, 0, (size_t)(cols / 32) * 1024 * sizeof(float), s) ==
                       cudaSuccess
                   ? FP4Q_OK
                   : FP4Q_ERR_CUDA;
    float* scratch = nullptr;
    const int st = scratch_for_current_device(&scratch);
    if (st != FP4Q_OK)
        return st;
    return fp4q::launch_hessian_blocks(x, dtype, rows, cols, chan_scale, hadamard32 != 0,
                                       hess_blocks, scratch, s) == cudaSuccess
               ? FP4Q_OK
               : FP4Q_ERR_CUDA;
}

}  // extern "C"
