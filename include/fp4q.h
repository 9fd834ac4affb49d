/*
 * fp4q.h -- C ABI of the block-scaled 4-bit quantization library for NVIDIA
 * B200 (sm_100a).  Plain pointers and sizes only.
 *
 * Sources (web pages; cited by title and section):
 *   [NVFP4] "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the
 *           Recurrent Half of a Hybrid 27B LLM" review, section 1 (NVFP4: E2M1
 *           values with one E4M3 scale per 16 elements; W4A4) and section 3
 *           (one global scale shared across fused GEMMs).
 *   [RaZeR] "RaZeR: Redundant Zero Remapping" technical summary, section 1
 *           (E2M1 value set; the always-positive E4M3 scale wastes its sign
 *           bit), section 2.1 (E3M3 weight scale frees 2 bits, E4M3
 *           activation scale frees 1), section 2.2 (the -0 code is remapped to
 *           a per-block special value picked for least squared error).
 *   [MACaQ] "MACaQ: Fast, Model Agnostic Calibrated Quantization for
 *           Low-Precision Weights and Activations" review, section 1 (MXFP4 =
 *           E2M1 + E8M0 per 32 elements; online per-channel scale and size-32
 *           block-Hadamard; Hessian-weighted exponent among {+1, 0, -1}) and
 *           section 3 (t_j ~ (sigma_j^W / rms_j^X)^0.75, H = X^T X).
 *   [Finer] "Finer is Better (with the Right Scaling)" summary, Methodology
 *           1-2 (block sizes 4..32; abs-max, prevent-zero, 4-over-6, brute
 *           force and hierarchical scaling).
 *
 * Conventions for every entry point:
 *  - Tensors are row-major.  Blocks are contiguous runs along the last
 *    dimension; cols must be a multiple of the block size.
 *  - Packed codes: byte i holds element 2i in bits 3:0 and element 2i+1 in
 *    bits 7:4; an E2M1 code is sign<<3 | magnitude index (0, .5, 1, 1.5, 2, 3,
 *    4, 6).  rows * cols / 2 bytes.
 *  - Scale bytes, one per block, row-major [rows][cols/block] unless an MMA
 *    layout is requested.
 *  - "device" pointers are CUDA device memory owned by the caller; the library
 *    allocates and frees nothing and keeps no state between calls (apart from
 *    the debug settings of fp4q_debug_set_wait_cycles and
 *    fp4q_debug_force_amax_pass, and the fixed scratch
 *    of fp4_hessian_blocks_noalloc).  "host" pointers are read during the call
 *    only.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous: outputs are valid once the stream reaches
 *    the call.  Argument errors are found on the host before anything is
 *    launched and leave all outputs untouched.
 *  - Pointers to vectors of 4-byte or wider elements and code buffers must
 *    be 16-byte aligned (FP4Q_ERR_ALIGN otherwise).
 *  - Inputs must be finite; scales/global scales passed in must be positive
 *    and finite.  Results for other inputs are unspecified.
 *  - Every fp32 decision (scale choice, special value, exponent) is computed
 *    with IEEE round-to-nearest operations in a fixed order and is
 *    reproducible bit for bit.
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP4Q_API __attribute__((visibility("default")))
#else
#define FP4Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4Q_OK = 0,
    FP4Q_ERR_ARG = 1,          /* a size, enum or pointer argument is invalid */
    FP4Q_ERR_ALIGN = 2,        /* a pointer is not aligned as required */
    FP4Q_ERR_UNSUPPORTED = 3,  /* valid request this build does not implement */
    FP4Q_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
    FP4Q_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up */
    FP4Q_ERR_WORKSPACE = 6,    /* the workspace is missing or too small */
    FP4Q_ERR_TOO_LARGE = 7     /* the problem needs more than the library's built-in scratch */
} fp4q_status;

typedef enum { FP4Q_F32 = 0, FP4Q_BF16 = 1, FP4Q_NVFP4_PACKED = 2, FP4Q_MXFP4_PACKED = 3 } fp4q_dtype;

/* Block-scale formats: E4M3 = OCP FP8 E4M3FN (NVFP4 and RaZeR activations),
 * E3M3 = 6-bit unsigned, bias 3, 2^-5..30 (RaZeR weights, [RaZeR] 2.1),
 * E8M0 = 2^(byte-127) (MXFP4, [MACaQ] 1). */
typedef enum { FP4Q_SF_E4M3 = 0, FP4Q_SF_E3M3 = 1, FP4Q_SF_E8M0 = 2, FP4Q_SF_UE5M3 = 3 } fp4q_scale_fmt;

/* Block-scale selection rules ([Finer] Methodology 2; [MACaQ] 1):
 *  ABSMAX        scale = E4M3(amax_b / (6 g)), ties to even, saturating at 448
 *  PREVENT_ZERO  ABSMAX, but a zero scale becomes the smallest positive E4M3 (2^-9)
 *  FOUR_OVER_SIX the 6-mapping scale or the 4-mapping scale E4M3(amax_b / (4 g)),
 *                whichever gives the strictly smaller block squared error
 *  BRUTE_FORCE   every finite positive E4M3 scale; least squared error, ties to
 *                the smallest scale
 *  HESSIAN_EXP   MXFP4 only: OCP exponent plus offset 0, +1 or -1 (tried in that
 *                order), least H'-weighted error d^T H'_k d, ties to the earlier */
typedef enum {
    FP4Q_ABSMAX = 0,
    FP4Q_PREVENT_ZERO = 1,
    FP4Q_FOUR_OVER_SIX = 2,
    FP4Q_BRUTE_FORCE = 3,
    FP4Q_HESSIAN_EXP = 4
} fp4q_rule;

/* Per-tensor FP32 global scale g of hierarchical scaling ([Finer] Methodology 2):
 *  NONE   g = 1
 *  AMAX   g = amax(x) / (6 * S_max), S_max = 448 (E4M3) or 30 (E3M3); g = 1 for
 *         an all-zero tensor.  Computed on the device inside the quantizer's
 *         own launch: every CTA takes the maximum of its slice of x, the CTAs
 *         meet at a bounded grid barrier (a cooperative launch; a CTA whose
 *         wait runs out takes the maximum of all of x itself, same result),
 *         and x is then read again for the quantization, mostly from L2.
 *         Needs a workspace; the g used is written to *global_scale if
 *         non-NULL.
 *  GIVEN  g read from *global_scale (device) -- e.g. one g shared by fused
 *         projections, the global-scale mismatch fix of [NVFP4] 3. */
typedef enum { FP4Q_GS_NONE = 0, FP4Q_GS_AMAX = 1, FP4Q_GS_GIVEN = 2 } fp4q_gs_mode;

/* Scale-byte layouts: ROWMAJOR [rows][cols/block]; MMA = the tcgen05 block-scaled
 * MMA scale-factor layout (128-row x 4-scale atoms of 512 bytes, atoms ordered
 * with the scale column fastest, row r of an atom at 16*(r%32) + 4*((r/32)%4),
 * scale column c at c%4).  MMA needs block 16, rows % 128 == 0 and
 * (cols/16) % 4 == 0. */
typedef enum { FP4Q_SFLAYOUT_ROWMAJOR = 0, FP4Q_SFLAYOUT_MMA = 1 } fp4q_sf_layout;

/* Workspace queries for fp4q_workspace_size(). */
typedef enum {
    FP4Q_OP_QUANTIZE = 0,       /* nvfp4_quantize / razer_quantize with GS_AMAX */
    FP4Q_OP_HESSIAN = 1,        /* fp4_hessian_blocks (rows, cols) */
    FP4Q_OP_CHANNEL_SCALE = 2,  /* mxfp4_channel_scale (tokens=rows, cols, n_out=n) */
    FP4Q_OP_GEMM = 3,           /* w4a4_gemm with bf16 A (M=rows, K=cols, N=n) */
    FP4Q_OP_FLIP = 4,           /* mxfp4_flip_refine (rows, cols) */
    FP4Q_OP_MX_GEMM = 5         /* mxfp4_gemm with bf16/fp32 A (M=rows, K=cols) */
} fp4q_op;

/* Bytes of device workspace an entry point needs (0 if none). */
FP4Q_API size_t fp4q_workspace_size(int op, int64_t rows, int64_t cols, int64_t n);

/* Human-readable name of a status code (static storage). */
FP4Q_API const char* fp4q_status_str(int status);

/* Library version, e.g. "fp4q 0.1.0 sm_100a". */
FP4Q_API const char* fp4q_version(void);

/*
 * NVFP4 quantization with a choice of block size and scale rule.
 * [NVFP4] 1 (format), [Finer] Methodology 1-2 (block sizes, rules, hierarchical).
 *
 *  x            device, rows x cols, dtype FP4Q_F32 or FP4Q_BF16, 16-byte aligned
 *  block        4, 8, 16 or 32 (cols % block == 0)
 *  rule         ABSMAX, PREVENT_ZERO, FOUR_OVER_SIX or BRUTE_FORCE
 *  gs_mode      NONE / AMAX / GIVEN; global_scale: device float, out for AMAX
 *               (nullable), in for GIVEN (required), ignored for NONE
 *  codes        device, rows*cols/2 bytes (out), 16-byte aligned
 *  scales       device, rows*cols/block E4M3 bytes (out), layout per sf_layout
 *  dequant      device fp32 rows x cols (out, nullable): v * (sc * g)
 *  block_mse    device fp32 rows x cols/block (out, nullable): sum((x-deq)^2)/block
 *  workspace    device, >= fp4q_workspace_size(FP4Q_OP_QUANTIZE, ...) bytes when
 *               gs_mode == AMAX (else may be NULL), 16-byte aligned
 * Brute force with a workspace also ADDS to the uint64 at workspace byte
 * offset FP4Q_WS_BF_EVALS the number of (block, candidate scale) error
 * evaluations the call performed (the exact shortcuts skip the rest); the
 * caller zeroes it to start a count.  Nothing else reads or resets it.
 * Errors: ERR_ARG (bad enum/size/null), ERR_ALIGN, ERR_WORKSPACE, ERR_CUDA.
 */
#define FP4Q_WS_BF_EVALS 3072
FP4Q_API int nvfp4_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int block, int rule,
                   int gs_mode, float* global_scale, uint8_t* codes, uint8_t* scales,
                   int sf_layout, float* dequant, float* block_mse, void* workspace,
                   size_t workspace_bytes, void* stream);

/*
 * nvfp4_quantize with the block-scale format as a parameter: FP4Q_SF_E4M3
 * (NVFP4, identical to nvfp4_quantize) or FP4Q_SF_UE5M3, the wide-exponent
 * scale of [Finer] (findings: E4M3 with 4-over-6 and hierarchical scaling
 * reaches UE5M3's quality).  UE5M3 is read as an unsigned 8-bit float with 5
 * exponent bits (bias 15), 3 mantissa bits and subnormals, codes 0..254
 * finite (0 .. 114688); the rules are unchanged, brute force searches codes
 * 1..254, prevent-zero uses code 1 (2^-17), AMAX mode g = amax / (6 * 114688).
 * UE5M3 scales are row-major only (the GEMM consumes E4M3).
 */
FP4Q_API int fp4_block_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int block,
                   int rule, int scale_fmt, int gs_mode, float* global_scale, uint8_t* codes,
                   uint8_t* scales, int sf_layout, float* dequant, float* block_mse,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * RaZeR quantization, blocks of 16 ([RaZeR] 2.1-2.2).  The block scale is the
 * abs-max scale in `scale_fmt`; for each special value the block is quantized
 * with the -0 code standing for that value (an element takes it when the
 * value, of the same sign, is strictly nearer than its E2M1 neighbour;
 * elements that round to zero take +0); the least squared error wins, ties to
 * the earlier table entry.
 *
 *  scale_fmt    FP4Q_SF_E3M3 (weights: meta = sel<<6 | e3m3, up to 4 specials)
 *               or FP4Q_SF_E4M3 (activations: meta = sel<<7 | e4m3, up to 2)
 *  specials     host, n_special values, each a non-zero multiple of 0.5 with
 *               magnitude <= 32
 *  meta         device, rows*cols/16 bytes (out)
 *  other arguments as nvfp4_quantize (g = amax / (6 * S_max) for AMAX).
 */
FP4Q_API int razer_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int scale_fmt,
                   const float* specials, int n_special, int gs_mode, float* global_scale,
                   uint8_t* codes, uint8_t* meta, float* dequant, float* block_mse,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * MXFP4 quantization with the online transform of [MACaQ] 1: u = x * t (per
 * column, if chan_scale != NULL), then for each 32-column block the
 * normalised Sylvester Hadamard rotation (if hadamard32), then E2M1 codes
 * with an E8M0 shared exponent.  rule ABSMAX: OCP exponent
 * floor(log2 amax_b) - 2; rule HESSIAN_EXP: that exponent plus 0, +1 or -1,
 * least d^T H'_k d.
 *
 *  chan_scale   device fp32 [cols] (nullable), 16-byte aligned
 *  hess_blocks  device fp32 [cols/32][32][32] (HESSIAN_EXP only)
 *  codes        device rows*cols/2 (out); scales: device rows*cols/32 E8M0 bytes
 *  dequant / block_mse  nullable; both refer to the transformed values u'
 * Errors: ERR_ARG (cols % 32, rule, missing hess), ERR_ALIGN, ERR_CUDA.
 */
FP4Q_API int mxfp4_quantize(const void* x, int dtype, int64_t rows, int64_t cols,
                   const float* chan_scale, int hadamard32, int rule, const float* hess_blocks,
                   uint8_t* codes, uint8_t* scales, float* dequant, float* block_mse,
                   void* stream);

/*
 * Flip-Refinement of MXFP4 weight codes ([MACaQ] 1 "Flip-Refinement", 3
 * "Exponent selection and Flip-Refinement"): starting from the codes of an
 * mxfp4_quantize call (round to nearest at the chosen exponents, which stay
 * fixed), each row repeatedly moves the one code whose shift to the
 * neighbouring E2M1 level below or above gives the largest decrease of
 * sum_k d_k^T H'_k d_k (d = u - deq, u the transformed row), computed in
 * closed form as 2 D g_i - D^2 H_ii with g = H' d updated incrementally
 * (g_j -= D H_ji); ties go to the lowest element, then the downward move.
 * A row stops when no move decreases the objective or after max_moves moves.
 *
 *  w            device rows x cols (F32 or BF16), the weights given to
 *               mxfp4_quantize; chan_scale / hadamard32 as there
 *  hess_blocks  device fp32 [cols/32][32][32] (H'_k, as fp4_hessian_blocks)
 *  max_moves    0 .. 2^20 accepted moves per row (the pages' setting: 128)
 *  codes        device rows*cols/2, in/out; scales: device E8M0 bytes (in)
 *  moves        device int32 [rows] (out, nullable): moves taken per row
 *  workspace    device, >= fp4q_workspace_size(FP4Q_OP_FLIP, rows, cols, 0)
 *               bytes, 16-byte aligned (each block's first moves, a row list)
 * Errors: ERR_ARG, ERR_ALIGN, ERR_WORKSPACE, ERR_UNSUPPORTED (cols > 8192:
 * a row's state is kept in shared memory), ERR_CUDA.
 */
FP4Q_API int mxfp4_flip_refine(const void* w, int dtype, int64_t rows, int64_t cols,
                   const float* chan_scale, int hadamard32, const float* hess_blocks,
                   int max_moves, uint8_t* codes, const uint8_t* scales, int32_t* moves,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Diagonal 32x32 blocks of the Hessian of the transformed activations,
 * H'_k = X'_k^T X'_k with X' = transform(x) as in mxfp4_quantize ([MACaQ] 1,
 * H = X^T X).  Computed on the tcgen05 tensor cores in tf32 with every value
 * split into two tf32 parts (hi + lo) and fp32 accumulation: about fp32
 * accuracy (tolerance, not bit-exact); partial sums per 256 tokens are added
 * in a fixed order, so the result is deterministic.
 *  hess_blocks  device fp32 [cols/32][32][32] (out)
 *  workspace    >= fp4q_workspace_size(FP4Q_OP_HESSIAN, rows, cols, 0) bytes
 *               (cols > 0), 16-byte aligned: an error word, then the partials
 * The kernel's waits on its own barriers are bounded.  If one gives up, the
 * blocks of the CTAs concerned come out NaN and the workspace's error word is
 * set: fp4q_hessian_status(workspace, stream) then returns FP4Q_ERR_TIMEOUT
 * (the call itself has already returned FP4Q_OK, having only enqueued work).
 * Errors: ERR_ARG, ERR_ALIGN, ERR_WORKSPACE, ERR_CUDA.
 */
FP4Q_API int fp4_hessian_blocks(const void* x, int dtype, int64_t rows, int64_t cols,
                       const float* chan_scale, int hadamard32, float* hess_blocks,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * fp4_hessian_blocks for callers that cannot allocate device memory.  No page
 * has a counterpart: this is a packaging of the same computation.
 *
 * Same arguments, layout and result as fp4_hessian_blocks, minus the
 * workspace: the per-chunk partial sums go to a 16 MiB scratch array that
 * the library keeps in device memory (held on every GPU that loads the
 * library, until the process exits).  Meant for code that owns no allocator
 * -- e.g. a plugin living in another framework's fixed memory plan, or a
 * path that must not call cudaMalloc because it can synchronize the device.
 * The scratch needed is ceil(rows/256) * (cols/32) * 4 KiB; problems above
 * 16 MiB of it (e.g. more than 8192 rows at 4096 columns) return
 * FP4Q_ERR_TOO_LARGE before anything runs.  Nothing is allocated or freed.
 * All calls share the one scratch array: calls whose work overlaps on the
 * GPU (other streams, other threads) race -- order them on one stream.  Every
 * call looks up the scratch's device address on the current device (the
 * first lookup on a device loads the library's device code there: make that
 * first call before any stream capture begins).  A bounded device wait that
 * gives up is reported by fp4q_hessian_status(NULL, stream) (FP4Q_ERR_TIMEOUT,
 * blocks NaN); the error word is cleared by every call.
 */
FP4Q_API int fp4_hessian_blocks_noalloc(const void* x, int dtype, int64_t rows, int64_t cols,
                                        const float* chan_scale, int hadamard32,
                                        float* hess_blocks, void* stream);

/*
 * Synchronizes `stream` and reports whether the last fp4_hessian_blocks call
 * that used `workspace` (or, for workspace == NULL, the last
 * fp4_hessian_blocks_noalloc call on the current device) finished normally
 * (FP4Q_OK) or had a bounded device-side wait give up (FP4Q_ERR_TIMEOUT: the
 * blocks of the CTAs concerned are NaN).  ERR_CUDA if the word cannot be read.
 */
FP4Q_API int fp4q_hessian_status(const void* workspace, void* stream);

/*
 * Online per-channel scale of [MACaQ] 3: t_j = (sigma_j^W / rms_j^X)^alpha,
 * sigma_j^W the population std of weight column j over n_out rows, rms_j^X =
 * sqrt(sum_t x_tj^2 / tokens) (the Hessian diagonal); t_j = 1 where either is
 * zero.  fp64 statistics, t rounded to fp32, t_inv = 1/t in fp32.
 *  x  device [tokens][cols]; w  device [n_out][cols]; cols % 8 == 0
 *  t, t_inv  device fp32 [cols] (out; t_inv nullable)
 *  workspace >= fp4q_workspace_size(FP4Q_OP_CHANNEL_SCALE, tokens, cols, n_out)
 */
FP4Q_API int mxfp4_channel_scale(const void* x, int x_dtype, int64_t tokens, const void* w,
                        int w_dtype, int64_t n_out, int64_t cols, float alpha, float* t,
                        float* t_inv, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dequantization with per-block MSE (the selection criterion of [RaZeR] 2.2
 * and [Finer] Methodology 2, as a standalone pass).
 *  codes, scales  as produced by the quantizers (row-major scale bytes)
 *  block          4/8/16/32 (E8M0: 32; RaZeR: 16)
 *  scale_fmt      E4M3 / E3M3 / UE5M3: deq = v * (sc * g); E8M0: deq = v * 2^(byte-127)
 *                 (UE5M3 takes no specials)
 *  specials       host, nullable: RaZeR tables (selector in the scale byte's top bits)
 *  global_scale   device float g, nullable (= 1); ignored for E8M0
 *  ref            device reference tensor (ref_dtype), nullable; needed for block_mse
 *  dequant        device fp32 (out, nullable); block_mse device fp32 (out, nullable)
 */
FP4Q_API int fp4_dequant_mse(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                    int block, int scale_fmt, const float* specials, int n_special,
                    const float* global_scale, const void* ref, int ref_dtype, float* dequant,
                    float* block_mse, void* stream);

/*
 * W4A4 GEMM on NVFP4 operands ([NVFP4] 1: W4A4 inference with E2M1 values and
 * E4M3 scales per 16 elements; [NVFP4] 3: per-tensor global scales).
 *
 *   out[m][n] = bf16( g_a * g_w * sum_k (v_a sc_a)[m][k] * (v_w sc_w)[n][k] ),
 *   i.e. out = A . W^T, A: M x K, W: N x K, out: M x N row-major.
 *
 *  a, a_format    FP4Q_F32 / FP4Q_BF16: A is a dense M x K tensor quantized here
 *                 (block 16, rule a_rule of ABSMAX/PREVENT_ZERO/FOUR_OVER_SIX/BRUTE_FORCE,
 *                 g_a = amax(A)/2688) into the workspace, then multiplied;
 *                 FP4Q_NVFP4_PACKED: a = packed codes (M*K/2 bytes), a_scales = E4M3
 *                 bytes in the MMA layout (FP4Q_SFLAYOUT_MMA), a_global_scale = device g_a
 *  w_codes        device N*K/2 packed codes; w_scales E4M3 bytes in the MMA layout;
 *                 w_global_scale device g_w
 *  M % 128 == 0, N % 256 == 0, K % 256 == 0 (FP4Q_ERR_UNSUPPORTED otherwise)
 *  out, out_dtype device M x N; FP4Q_BF16 (the W4A4 output) or FP4Q_F32: the fp32
 *                 accumulator times g_a g_w without the bf16 rounding (for accuracy
 *                 checks against an fp64 reference, or consumers that keep fp32)
 *  workspace      >= fp4q_workspace_size(FP4Q_OP_GEMM, M, K, N) bytes (at least 8 KiB
 *                 for packed A), 16-byte aligned; it also holds the error word read by
 *                 fp4q_gemm_status
 * The product runs on tcgen05 tensor cores with fp32 accumulation in TMEM.
 */
FP4Q_API int w4a4_gemm(const void* a, int a_format, int a_rule, const uint8_t* a_scales,
                       const float* a_global_scale, const uint8_t* w_codes,
                       const uint8_t* w_scales, const float* w_global_scale, int64_t M,
                       int64_t N, int64_t K, void* out, int out_dtype, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * RaZeR operands for the tensor-core GEMM ([RaZeR] 2.2: the -0 code of a
 * block stands for the block's special value; [RaZeR] 2.3: the Blackwell
 * kernels handle the remapping in two passes on the existing tensor cores).
 * Splits RaZeR codes into two E2M1 tensors that share one set of E4M3 block
 * scales: every special value v is written as p + q with p, q E2M1 values
 * (p the largest magnitude of v's sign leaving an E2M1 remainder: +-5 =
 * +-(4 + 1), +-3.5 = +-(3 + 0.5)),
 *   main_codes   the codes with each -0 replaced by p of the block's selector
 *   extra_codes  q at the -0 positions, +0 everywhere else
 * so v_main * sc + v_extra * sc equals the RaZeR value v * sc exactly.
 *
 *  codes, meta    device, razer_quantize output: rows*cols/2 code bytes
 *                 (16-byte aligned) and rows*cols/16 meta bytes
 *  scale_fmt      FP4Q_SF_E3M3 (meta = sel<<6 | e3m3, up to 4 specials) or
 *                 FP4Q_SF_E4M3 (meta = sel<<7 | e4m3, up to 2)
 *  specials       host, the table razer_quantize was given
 *  main_codes, extra_codes   device, rows*cols/2 bytes each (out), 16-byte aligned
 *  scales_mma     device, rows*cols/16 E4M3 bytes in FP4Q_SFLAYOUT_MMA (out)
 *                 (E3M3 values are E4M3 values: the conversion is exact)
 *  rows % 128 == 0, cols % 64 == 0 (FP4Q_ERR_ARG otherwise).
 * Errors: ERR_ARG (sizes, format, table), ERR_UNSUPPORTED (a special that is
 * not the sum of two E2M1 values, e.g. 5.5 = 4 + 1.5 is fine, 11 is not),
 * ERR_ALIGN, ERR_CUDA.  Weights are prepared once, offline.
 */
FP4Q_API int razer_gemm_prepare(const uint8_t* codes, const uint8_t* meta, int64_t rows, int64_t cols,
                                int scale_fmt, const float* specials, int n_special,
                                uint8_t* main_codes, uint8_t* extra_codes, uint8_t* scales_mma,
                                void* stream);

/*
 * RaZeR-aware W4A4 GEMM: out = bf16(g_a * g_w * (A + A1) . (W + W1)^T) where
 * A, A1 (and W, W1) are E2M1 code tensors sharing the block scales a_scales
 * (w_scales) -- the razer_gemm_prepare split of a RaZeR operand, or a plain
 * NVFP4 operand with its extra tensor NULL.  Each present pair of tensors is
 * one pass over K into the same fp32 TMEM accumulator (2 passes for RaZeR
 * weights, 4 when both operands are RaZeR).
 *
 *  a_codes, a_extra (nullable)   device M*K/2 bytes; a_scales E4M3 MMA layout;
 *                                a_global_scale device g_a
 *  w_codes, w_extra (nullable)   device N*K/2 bytes; w_scales E4M3 MMA layout;
 *                                w_global_scale device g_w
 *  shapes, out / out_dtype, workspace (>= 8 KiB) and errors as w4a4_gemm;
 *  fp4q_gemm_status reports a device timeout.
 */
FP4Q_API int razer_w4a4_gemm(const uint8_t* a_codes, const uint8_t* a_extra, const uint8_t* a_scales,
                             const float* a_global_scale, const uint8_t* w_codes,
                             const uint8_t* w_extra, const uint8_t* w_scales,
                             const float* w_global_scale, int64_t M, int64_t N, int64_t K, void* out,
                             int out_dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Scale bytes from the row-major layout [rows][nscales] to FP4Q_SFLAYOUT_MMA
 * (the tcgen05 scale layout; works for E4M3 scales per 16 and E8M0 scales per
 * 32 alike), e.g. for MXFP4 weights quantized row-major and refined by
 * mxfp4_flip_refine.  rows % 128 == 0, nscales % 4 == 0; both pointers device,
 * 16-byte aligned, rows*nscales bytes.  Errors: ERR_ARG, ERR_ALIGN, ERR_CUDA.
 */
FP4Q_API int fp4_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t nscales, uint8_t* out,
                               void* stream);

/*
 * MXFP4 W4A4 GEMM ([MACaQ] 1: W4A4 inference with MXFP4 operands, E2M1 values
 * and one E8M0 exponent per 32 elements, the activations rotated online):
 *
 *   out[m][n] = bf16( sum_k (v_a 2^(ea - 127))[m][k] * (v_w 2^(ew - 127))[n][k] ),
 *
 * on tcgen05 tensor cores (kind::mxf4, block 32).  With the online transform
 * X' = (X * t) B (t per channel, B the normalised 32-block Hadamard) and the
 * weights prepared as W' = (W / t) B (mxfp4_quantize with 1/t), out
 * approximates X W^T.
 *
 *  a, a_format  FP4Q_F32 / FP4Q_BF16: A is a dense M x K tensor; the prologue
 *               (a * chan_scale, the 32-block rotation if hadamard32, OCP E8M0
 *               exponent, E2M1 codes) runs here into the workspace, scales
 *               written in the GEMM's layout, and the GEMM kernel is launched
 *               on the same stream as its programmatic dependent (its setup
 *               overlaps the prologue's tail; it reads A only after the
 *               prologue completed); FP4Q_MXFP4_PACKED: a = codes
 *               (M*K/2 bytes), a_scales = E8M0 bytes in FP4Q_SFLAYOUT_MMA
 *               (chan_scale must be NULL)
 *  chan_scale   device fp32 [K] (nullable): t for the dense A
 *  w_codes      device N*K/2 bytes; w_scales E8M0 bytes in FP4Q_SFLAYOUT_MMA
 *               (mxfp4_quantize + fp4_scales_to_mma)
 *  M % 128 == 0, N % 256 == 0, K % 256 == 0 (FP4Q_ERR_UNSUPPORTED otherwise)
 *  out, out_dtype as w4a4_gemm (FP4Q_BF16 or FP4Q_F32)
 *  workspace    >= fp4q_workspace_size(FP4Q_OP_MX_GEMM, M, K, N) for dense A,
 *               8 KiB for packed A; 16-byte aligned; holds the error word read
 *               by fp4q_gemm_status
 */
FP4Q_API int mxfp4_gemm(const void* a, int a_format, const uint8_t* a_scales, const float* chan_scale,
                        int hadamard32, const uint8_t* w_codes, const uint8_t* w_scales, int64_t M,
                        int64_t N, int64_t K, void* out, int out_dtype, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * Synchronizes `stream` and reports whether the last GEMM call (w4a4_gemm,
 * razer_w4a4_gemm or mxfp4_gemm) that used this workspace finished normally
 * (FP4Q_OK) or had a bounded device-side wait give up (FP4Q_ERR_TIMEOUT; its
 * output is then incomplete).  Every GEMM call clears the word first.
 */
FP4Q_API int fp4q_gemm_status(const void* workspace, void* stream);

/*
 * Diagnostic: the tensor-pipe ceiling the GEMMs are measured against.  Launches
 * a kernel in which every pair of SMs issues `iters` groups of four
 * back-to-back block-scaled FP4 MMAs of the GEMMs' shape (CTA pair, 256 x 256
 * x 64; mx = 0: kind::mxf4nvf4 with UE4M3 scales per 16, mx = 1: kind::mxf4
 * with UE8M0 scales per 32) on operand tiles held in shared memory (hashed
 * code bytes, so the operands toggle like real data) and scales copied into
 * TMEM once -- no global traffic and no waits inside the loop.
 * Enqueued on `stream`; time it with events on that stream and divide
 * fp4q_mma_ceiling_flops(iters) (the flops one launch performs on the current
 * device) by the time.  err: device int (4-byte aligned), set to 1 if the
 * final bounded wait gave up (the caller clears it).  1 <= iters <= 2^20 (a
 * launch then stays far inside the wait's bound).
 * Errors: ERR_ARG, ERR_ALIGN, ERR_CUDA.
 */
FP4Q_API int fp4q_mma_ceiling(int mx, int iters, int* err, void* stream);
FP4Q_API double fp4q_mma_ceiling_flops(int iters);

/*
 * Debug: the limit, in SM clock cycles, after which the main-loop waits of the
 * tensor-core kernels (the three GEMMs and the Hessian blocks) give up; 0 or a
 * negative value restores the default (4e9 cycles, about 2 s at the boost
 * clock).  Process-wide; read when a call launches its kernels.  Meant for
 * tests of the timeout path: with a limit of 1 cycle a wait that is not
 * satisfied at once gives up, the kernel winds down (letting its own copies
 * and MMAs finish under the default limit), and the status call of that
 * entry point reports FP4Q_ERR_TIMEOUT.  Returns the previous setting.
 */
FP4Q_API int64_t fp4q_debug_set_wait_cycles(int64_t cycles);

/*
 * Debug: with on != 0, every later call that computes a hierarchical global
 * scale (FP4Q_GS_AMAX) takes the path used when the device cannot make the
 * quantizer's launch cooperative: a separate amax pass over x writes partial
 * maxima into the workspace, and the quantizer reduces them (the same exact
 * maximum, so the same results).  Process-wide, for tests of that path.
 * Returns the previous setting.
 */
FP4Q_API int fp4q_debug_force_amax_pass(int on);

#ifdef __cplusplus
}
#endif

#endif /* FP4Q_H */
