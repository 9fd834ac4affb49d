// fp4q_internal.h -- launchers behind the C ABI of include/fp4q.h.
// Every launcher enqueues on `stream` and returns the cudaError_t of its
// launches; argument checking is done by the C ABI layer before these run.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fp4q {

// Default limit of the bounded device-side waits (SM clock cycles, about 2 s
// at the boost clock).
constexpr long long kDefaultWaitCycles = 4000000000LL;

// The limit the next launch gives its main-loop waits: the process-wide
// setting of fp4q_debug_set_wait_cycles, or kDefaultWaitCycles.
long long wait_limit_cycles();
// fp4q_debug_force_amax_pass: take the separate amax pass instead of the fused one
bool force_amax_pass();

// Global-scale source for a quantizer launch.
struct GsArgs {
    int mode;                 // 0 none (g = 1), 1 amax partials in ws, 2 given (device float),
                              // 3 amax computed in the quantizer launch itself (fused)
    const float* partials;    // mode 1: per-CTA block maxima written by launch_amax
    int n_partials;
    float denom;              // modes 1, 3: 6 * largest scale of the format (2688, 180, 6 * 114688)
    const float* given;       // mode 2
    float* out;               // nullable: where to write the g that was used
    // mode 3: the whole input (n elements), one partial maximum per CTA, and the
    // grid barrier's arrival counter (zero before the launch)
    const void* x;
    int64_t n;
    float* fused_partials;
    unsigned int* counter;
    long long wait_limit;
};

// Number of partial maxima launch_amax writes (fixed; the workspace holds them).
constexpr int kAmaxPartials = 592;   // 148 SMs x 4
// Largest grid of a fused-amax quantizer launch (its partials area holds this many).
constexpr int kFusedMaxCtas = 960;

// SM count of the current device (cached per device).
int num_sms();

// Raise `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel, device); thread-safe.
cudaError_t smem_opt_in(const void* kernel, int bytes);

cudaError_t launch_amax(const void* x, int dtype, int64_t n, float* partials, cudaStream_t s);

// evals (nullable): brute force adds its number of block-candidate evaluations;
// ue5m3: the block scales are UE5M3 instead of E4M3
cudaError_t launch_nvfp4_quant(const void* x, int dtype, int64_t rows, int64_t cols, int block,
                               int rule, const GsArgs& gs, uint8_t* codes, uint8_t* scales,
                               int mma_layout, float* deq, float* mse, unsigned long long* evals,
                               cudaStream_t s, int ue5m3 = 0);

cudaError_t launch_razer_quant(const void* x, int dtype, int64_t rows, int64_t cols, int sf,
                               const float* specials_host, int n_special, const GsArgs& gs,
                               uint8_t* codes, uint8_t* meta, float* deq, float* mse,
                               cudaStream_t s);

cudaError_t launch_dequant_mse(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                               int64_t cols, int block, int sf, const float* specials_host,
                               int n_special, const float* gs_dev, const void* ref, int ref_dt,
                               float* deq, float* mse, cudaStream_t s);

cudaError_t launch_mx_channel_scale(const void* x, int xdt, int64_t tokens, const void* w, int wdt,
                                    int64_t n_out, int64_t cols, float alpha, float* t,
                                    float* t_inv, void* ws, cudaStream_t s);

// part: the partial-sum area (hessian_ws_bytes(rows, cols) bytes); err: a
// device int set to 1 when a bounded wait gave up (the caller clears it)
cudaError_t launch_hessian_blocks(const void* x, int dtype, int64_t rows, int64_t cols,
                                  const float* chan_scale, int hadamard, float* hess, float* part,
                                  int* err, cudaStream_t s);

// mma_layout: scales in the MMA scale layout (rows % 128 == 0, cols % 128 == 0)
cudaError_t launch_mxfp4_quant(const void* x, int dtype, int64_t rows, int64_t cols,
                               const float* chan_scale, int hadamard, int rule, const float* hess,
                               uint8_t* codes, uint8_t* scales, float* deq, float* mse,
                               cudaStream_t s, int mma_layout = 0);

// Flip-Refinement of MX codes in place (exponents fixed); moves nullable.
cudaError_t launch_mxfp4_flip_refine(const void* w, int dtype, int64_t rows, int64_t cols,
                                     const float* tinv, int hadamard, const float* hess, int max_moves,
                                     uint8_t* codes, const uint8_t* scales, int32_t* moves, void* ws,
                                     cudaStream_t s);
size_t flip_refine_smem_bytes(int64_t cols);
size_t flip_refine_ws_bytes(int64_t rows, int64_t cols);

bool gemm_shape_supported(int64_t M, int64_t N, int64_t K);

// a1_codes / w1_codes (nullable): second code tensors sharing the scales of
// A / W; the GEMM then sums the products of every pair of present tensors,
// out = (A + A1) . (W + W1)^T, as extra passes over K into one accumulator.
// mx: MXFP4 operands (E8M0 scales per 32 elements in the MMA layout; ga, gw
// NULL = no global scale).
// out_f32: fp32 output instead of bf16 (same layout, M x N row-major).
cudaError_t launch_w4a4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* ga,
                             const uint8_t* w_codes, const uint8_t* w_sf, const float* gw, int64_t M,
                             int64_t N, int64_t K, void* out, int out_f32, int* err, cudaStream_t s,
                             const uint8_t* a1_codes = nullptr, const uint8_t* w1_codes = nullptr,
                             int mx = 0, int after_prologue = 0);
// after_prologue: the kernel before it on the stream is the operand prologue
// (a kernel that executes griddepcontrol.launch_dependents); the GEMM is then
// launched as its programmatic dependent, overlapping its setup with the
// prologue's tail.

// The tensor-pipe ceiling probe: every SM pair issues iters x 4 back-to-back
// 256x256x64 block-scaled FP4 MMAs (mx: kind::mxf4) on resident operands;
// *err (device) is set to 1 if a bounded wait gave up.
cudaError_t launch_mma_ceiling(int mx, int iters, int* err, cudaStream_t s);
int mma_ceiling_pairs();

// Row-major scale bytes [rows][nscales] -> the MMA scale layout (rows % 128 == 0,
// nscales % 4 == 0).
cudaError_t launch_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t nscales, uint8_t* out,
                                 cudaStream_t s);

// RaZeR codes + meta -> (main codes, extra codes, E4M3 scale bytes in the MMA
// layout) with main + extra = the RaZeR values exactly.  p_code / q_code:
// per selector, the E2M1 codes whose values sum to the special value.
cudaError_t launch_razer_gemm_prepare(const uint8_t* codes, const uint8_t* meta, int64_t rows,
                                      int64_t cols, int sf, const uint8_t* p_code,
                                      const uint8_t* q_code, uint8_t* main_codes,
                                      uint8_t* extra_codes, uint8_t* scales_mma, cudaStream_t s);

// Device address of fp4_hessian_blocks_noalloc's error word on the current
// device (NULL if it cannot be looked up).
const int* noalloc_hessian_error_word();

// Workspace (bytes) launch_hessian_blocks / launch_mx_channel_scale need.
size_t hessian_ws_bytes(int64_t rows, int64_t cols);
size_t channel_scale_ws_bytes(int64_t tokens, int64_t n_out, int64_t cols);

}  // namespace fp4q
