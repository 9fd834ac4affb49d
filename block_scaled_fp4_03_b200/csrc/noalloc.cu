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
// exits.  Every call looks up the array's device address on the current
// device (cudaGetSymbolAddress; nothing is cached, so a device reset that
// reloads the module at another address is picked up).  The first lookup on
// a device loads the library's device code there; make that first call
// before any stream capture begins.  All calls share the array, so two calls
// whose kernels overlap on the GPU (different streams, or different host
// threads) race on it; order them on one stream.  Each call overwrites every
// partial it later reads, so the partials need no clearing; the error word
// beside them (set when a bounded device wait gives up, read by
// fp4q_hessian_status(NULL, stream)) is cleared at the start of every call.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/fp4q.h"
#include "fp4q_internal.h"

namespace {

// 4096 partial 32x32 blocks of fp32 = 16 MiB: enough for 8192 tokens x 4096
// columns (32 chunks of 256 tokens x 128 column blocks).
constexpr size_t kScratchBlocks = 4096;
constexpr size_t kScratchFloats = kScratchBlocks * 1024;

static __device__ __align__(256) float g_hessian_scratch[kScratchFloats];
static __device__ __align__(16) int g_hessian_err;

// Device addresses of the scratch array and of the error word on the current
// device (in host code the symbols are only stand-ins, not device addresses).
bool lookup_scratch(float** scratch, int** err)
{
    void* p = nullptr;
    void* e = nullptr;
    if (cudaGetSymbolAddress(&p, g_hessian_scratch) != cudaSuccess || !p ||
        cudaGetSymbolAddress(&e, g_hessian_err) != cudaSuccess || !e)
        return false;
    *scratch = static_cast<float*>(p);
    *err = static_cast<int*>(e);
    return true;
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
    float* scratch = nullptr;
    int* err = nullptr;
    if (!lookup_scratch(&scratch, &err) || cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    if (rows == 0)
        return cudaMemsetAsync(hess_blocks, 0, (size_t)(cols / 32) * 1024 * sizeof(float), s) ==
                       cudaSuccess
                   ? FP4Q_OK
                   : FP4Q_ERR_CUDA;
    return fp4q::launch_hessian_blocks(x, dtype, rows, cols, chan_scale, hadamard32 != 0,
                                       hess_blocks, scratch, err, s) == cudaSuccess
               ? FP4Q_OK
               : FP4Q_ERR_CUDA;
}

}  // extern "C"

namespace fp4q {

const int* noalloc_hessian_error_word()
{
    float* scratch = nullptr;
    int* err = nullptr;
    return lookup_scratch(&scratch, &err) ? err : nullptr;
}

}  // namespace fp4q
