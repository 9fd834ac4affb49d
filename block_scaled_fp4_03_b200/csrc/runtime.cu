// runtime.cu -- host-side state of the library: the SM count used to size
// persistent grids and the shared-memory opt-in of kernels that need more than
// the default 48 KiB of dynamic shared memory (both per device, so a process
// that drives several GPUs gets each one right), and the process-wide limit of
// the tensor-core kernels' bounded waits (fp4q_debug_set_wait_cycles).
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "../../include/fp4q.h"
#include "fp4q_internal.h"

namespace fp4q {

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];
std::mutex g_opt_mu;
std::set<std::pair<const void*, int>> g_opted;   // (kernel, device) pairs already opted in
std::atomic<long long> g_wait_cycles{0};         // 0: kDefaultWaitCycles
std::atomic<int> g_force_amax_pass{0};

}  // namespace

bool force_amax_pass() { return g_force_amax_pass.load(std::memory_order_relaxed) != 0; }

long long wait_limit_cycles()
{
    const long long v = g_wait_cycles.load(std::memory_order_relaxed);
    return v > 0 ? v : kDefaultWaitCycles;
}

int num_sms()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 148;
    int n = g_sms[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

cudaError_t smem_opt_in(const void* kernel, int bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lock(g_opt_mu);
    if (g_opted.count({kernel, dev}))
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        g_opted.insert({kernel, dev});
    return e;
}

}  // namespace fp4q

extern "C" int64_t fp4q_debug_set_wait_cycles(int64_t cycles)
{
    return fp4q::g_wait_cycles.exchange(cycles > 0 ? cycles : 0, std::memory_order_relaxed);
}

extern "C" int fp4q_debug_force_amax_pass(int on)
{
    return fp4q::g_force_amax_pass.exchange(on != 0 ? 1 : 0, std::memory_order_relaxed);
}
