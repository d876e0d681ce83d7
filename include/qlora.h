/*
 * qlora.h -- C ABI of libqlora, the B200 (sm_100a) QLoRA NF4 linear layer.
 *
 * The layer (per "Unsloth v0.1.463-beta: Fixes Studio Crash and llama-server Permission Issue",
 * kongchang.com, section "About the Unsloth Project", paragraph "How LoRA and QLoRA work"; "unsloth",
 * pyshine.com, section "Why You Need This"; "Inside Unsloth: How the Fastest LLM Fine-Tuning Library
 * Works", thriftbooks.com, section "What You'll Learn", item "LoRA and QLoRA"):
 *
 *     y  = x deq(W)^T + s (x A^T) B^T                      forward
 *     dX = dY deq(W) + s (dY B) A,  dA = s (dY B)^T x,  dB = s dY^T (x A^T)      backward (W frozen)
 *
 * with x [M,K] bf16 activations, W [N,K] stored as blockwise NF4 (4-bit codes + one fp32 absmax per
 * 64-element block), LoRA adapters A [r,K] and B [N,r] in bf16 and the scaling s = lora_alpha / r.
 *
 * Conventions for every entry point
 *   - Matrices are row-major and contiguous.  "bf16" buffers hold bfloat16 bit patterns (uint16_t).
 *   - All data pointers are DEVICE pointers, 16-byte aligned.  The caller owns every buffer; the library
 *     never allocates, frees or synchronizes (except ql_get_device_error, which says so).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls are asynchronous.
 *   - Argument errors are detected on the host before any launch and return QL_ERR_INVALID_ARG (or
 *     QL_ERR_UNSUPPORTED for valid but unimplemented parameters); nothing is launched then.  A failed
 *     launch returns QL_ERR_CUDA.  Faults detected on the device (a bounded wait that gave up, a
 *     non-finite block maximum) are latched in a device error word read by ql_get_device_error.
 *   - The library keeps no state between calls apart from per-device constants (the NF4 table).
 *   - Entry points need the CUDA device of `stream` to be current.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QL_API __attribute__((visibility("default")))
#else
#define QL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QL_OK = 0,
  QL_ERR_INVALID_ARG = 1,  /* bad shape, null or misaligned pointer, too-small workspace */
  QL_ERR_UNSUPPORTED = 2,  /* valid parameters this build does not implement (e.g. blocksize != 64) */
  QL_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed */
  QL_ERR_TIMEOUT = 4       /* a kernel's bounded wait expired (reported by ql_get_device_error) */
} ql_status;

typedef enum { QL_F32 = 0, QL_BF16 = 1 } ql_dtype;
typedef enum { QL_PASS_FWD = 0, QL_PASS_BWD = 1 } ql_pass;

/* Human-readable name of a status code (static string). */
QL_API const char* ql_status_string(int status);

/* ABI version of this library (incremented on incompatible changes). */
QL_API int ql_abi_version(void);

/* Copies the library's 16-entry NF4 level table (fp32, ascending) into host memory `out`.
 * Host-only; needs no GPU.  The table follows the normal-quantile rule (8 positive and 7 negative
 * standard-normal quantiles normalised to [-1, 1], plus an exact 0 at index 7). */
QL_API void ql_nf4_codebook(float out[16]);

/* Reads and clears the device error word of the current device after synchronizing `stream`.
 * Returns QL_OK, QL_ERR_TIMEOUT (a kernel's bounded wait expired), QL_ERR_INVALID_ARG (nf4_quantize met
 * a non-finite block), or QL_ERR_CUDA.  This is the only entry point that synchronizes. */
QL_API ql_status ql_get_device_error(void* stream);

/* Number of kernels this library has launched in the process so far (all devices).  Host-only. */
QL_API uint64_t ql_launch_count(void);

/* Observability hook.  `which` = 0: the fused forward GEMM of qlora_linear_fwd; 1: the fused dX GEMM of
 * qlora_linear_bwd.  When `start`/`stop` (cudaEvent_t as void*) are non-NULL the library records them on
 * the call's stream immediately before and after that one kernel; NULL disables.  Process-wide setting;
 * the events stay owned by the caller.  Returns QL_ERR_INVALID_ARG for an unknown `which`. */
QL_API ql_status ql_set_profile_events(int which, void* start, void* stop);

/* Failure-detection self-test: launches one tiny kernel that waits on an mbarrier nobody arrives on, with
 * the same bounded-wait code the GEMM kernels use but a limit of `wait_cycles` clock cycles (1 .. 2^32).
 * The wait gives up, latches the timeout bit in the device error word and the kernel returns normally;
 * ql_get_device_error then reports QL_ERR_TIMEOUT and the context stays usable. */
QL_API ql_status ql_selftest_wait_timeout(int64_t wait_cycles, void* stream);

/*
 * ql_selftest_arm_gemm_stall -- failure-path test hook (the paper has no counterpart).  Arms the NEXT dequantizing
 * GEMM launch of this process (the fused forward or dX kernel of any layer call) so that one warp role leaves
 * before doing anything: role 1 the MMA issuer, 2 the activation (B) producer, 3 the codes producer.  None of them
 * then has a copy or an MMA in flight.  Every wait of that launch is bounded by wait_cycles (>= 100000) instead
 * of about 2 s, so the other roles' waits expire: the kernel raises its abort flag, drains the copies it issued,
 * frees its tensor memory and returns; ql_get_device_error then reports QL_ERR_TIMEOUT and the call's outputs
 * are undefined.  (A unit's LoRA stages follow its main stages, so with role 3 no stage of the first unit is ever
 * complete, whatever the rank.)  The arming is consumed by that one launch.
 */
QL_API ql_status ql_selftest_arm_gemm_stall(int role, int64_t wait_cycles);

/*
 * nf4_quantize -- blockwise NF4 quantization of a frozen base weight ("How LoRA and QLoRA work", as above).
 *   w        [numel] fp32, the flat row-major weight (W [N,K] gives numel = N*K).
 *   numel    number of elements; a positive multiple of `blocksize`.
 *   blocksize elements per absmax block; only 64 is supported (QL_ERR_UNSUPPORTED otherwise).
 *   codes    [numel/2] uint8 out: element 2j in the HIGH nibble of byte j, element 2j+1 in the low nibble.
 *   absmax   [numel/blocksize] fp32 out: max |w| of each block.
 * Per block: n = w / absmax in IEEE fp32; code = number of level midpoints strictly below n (a value on
 * a midpoint takes the lower code); an all-zero block stores absmax 0 and code 7 everywhere.  Bit-exact
 * and deterministic.  Non-finite weights are outside the domain: the device error word records them.
 */
QL_API ql_status nf4_quantize(const float* w, int64_t numel, int blocksize, uint8_t* codes, float* absmax,
                       void* stream);

/*
 * nf4_dequantize -- w' = fl32(level[code] * absmax) ("unsloth", pyshine.com, section "Why You Need This":
 * NF4 weights dequantized on the fly; here materialized for checking and export).
 *   codes, absmax  as produced by nf4_quantize; numel, blocksize as there.
 *   out_dtype      QL_F32: out is float[numel] holding w';  QL_BF16: out is bf16[numel] holding
 *                  round-to-nearest-even(w').
 * Bit-exact and deterministic.
 */
QL_API ql_status nf4_dequantize(const uint8_t* codes, const float* absmax, int64_t numel, int blocksize,
                         ql_dtype out_dtype, void* out, void* stream);

/*
 * qlora_merge_lora -- merged weight W' = deq(W) + s * B * A of one layer ("unsloth", pyshine.com, section
 * "Why You Need This", the paragraph on saving: adapters folded into the base layer by layer).
 *   N, K     W is [N,K]: N >= 1, K a positive multiple of 64.
 *   r        LoRA rank, 0 <= r <= 256 (r = 0: W' = deq(W)).
 *   codes, absmax  the base weight as produced by nf4_quantize (16-byte aligned).
 *   A        [r,K] bf16 row-major;  B [N,r] bf16 row-major (16-byte aligned; may be null when r = 0).
 *   s        the LoRA scaling.
 *   out_dtype QL_F32: out is float[N*K];  QL_BF16: out is bf16[N*K] (round-to-nearest-even of W').
 * Arithmetic, per element, in IEEE fp32 with no fused multiply-add: d = level * absmax; acc = sum over j
 * of B[n,j] * A[j,k], added left to right starting from 0; W' = d + s * acc.  Bit-exact and deterministic.
 * QL_ERR_INVALID_ARG on bad sizes, null or misaligned pointers, or another out_dtype.
 */
QL_API ql_status qlora_merge_lora(int64_t N, int64_t K, int64_t r, const uint8_t* codes, const float* absmax,
                                  const uint16_t* A, const uint16_t* B, float s, ql_dtype out_dtype, void* out,
                                  void* stream);

/*
 * qlora_merge_lora_nf4 -- W' as above, requantized in the same pass by the nf4_quantize rule, so the merged
 * layer stays 4-bit and W' never reaches HBM.
 *   codes_out  [N*K/2] uint8, absmax_out [N*K/64] fp32 (16-byte aligned).  They may be the input buffers
 *              themselves (in-place merge): each 64-element block is read in full before it is written.
 * Bit-exact and deterministic.  A non-finite W' is recorded in the device error word, as in nf4_quantize.
 */
QL_API ql_status qlora_merge_lora_nf4(int64_t N, int64_t K, int64_t r, const uint8_t* codes, const float* absmax,
                                      const uint16_t* A, const uint16_t* B, float s, uint8_t* codes_out,
                                      float* absmax_out, void* stream);

/*
 * qlora_workspace_bytes -- device scratch needed by qlora_linear_fwd (pass = QL_PASS_FWD) or
 * qlora_linear_bwd (QL_PASS_BWD) for these sizes on the current device (split-K or stream-K partial sums,
 * the rank-r intermediates s*x*A^T and s*dY*B).  Host-only.  Returns 0 when nothing is needed.
 */
QL_API size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, ql_pass pass);

/*
 * qlora_linear_fwd -- y = x deq(W)^T + s (x A^T) B^T in one fused pass over the NF4 weight
 * ("Inside Unsloth ...", section "What You'll Learn", item "LoRA and QLoRA": NF4 dequantization, matrix
 * multiplication and LoRA correction fused; "unsloth", pyshine.com: the LoRA matmul that fuses the base
 * quantized weight and the adapter delta into one call, and the dequantize-on-the-fly GEMV for small M).
 *   M, N, K, r  x [M,K], W [N,K], A [r,K], B [N,r], y [M,N].  M >= 0; N >= 1 with N % 8 == 0;
 *               K >= 64 with K % 64 == 0; 0 <= r <= 256 with r % 8 == 0 (r = 0: plain NF4 layer, A/B unused).
 *   x           bf16 [M,K].
 *   codes, absmax  NF4 weight from nf4_quantize of W (blocksize 64).
 *   A, B        bf16 LoRA adapters.
 *   s           LoRA scaling (lora_alpha / r).
 *   y           bf16 [M,N] out (round-to-nearest-even of the fp32 accumulator).
 *   su_out      nullable bf16 [M,r] out: s * x A^T rounded to bf16, the rank-r term the product uses;
 *               pass it to qlora_linear_bwd to skip recomputing it.
 *   workspace, ws_bytes  device scratch of at least qlora_workspace_bytes(M,N,K,r,QL_PASS_FWD) bytes
 *               (may be NULL when that is 0).
 * Products run on the tensor cores in bf16 with fp32 accumulation; deq(W) is formed tile by tile in tensor
 * memory (TMEM), where the MMA reads it, and never written to global memory.  The result is deterministic
 * for given sizes.
 */
QL_API ql_status qlora_linear_fwd(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x, const uint8_t* codes,
                           const float* absmax, const uint16_t* A, const uint16_t* B, float s, uint16_t* y,
                           uint16_t* su_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * qlora_linear_fwd_noalloc -- the forward above for callers that cannot allocate device memory at all, not
 * even a workspace to lend: code running while a stream is captured in global mode (where cudaMalloc is an
 * error) or a plug-in whose host program owns all device memory and forbids allocation after start-up.
 * The paper has no counterpart; this is a property of this library's interface.
 *   Arguments as qlora_linear_fwd, without workspace/ws_bytes.  The scratch lives in an 8 MiB array
 *   compiled into the library, which every GPU that loads the library holds until the process exits.
 *   Sizes whose qlora_workspace_bytes(M,N,K,r,QL_PASS_FWD) exceeds 8 MiB (8388608 bytes) return
 *   QL_ERR_INVALID_ARG before any launch.  No cudaMalloc, cudaFree or allocating routine is called.
 *   Every call looks up the array's device address in the current context (cudaGetSymbolAddress, with the
 *   device current), since the address belongs to the context: it changes after cudaDeviceReset, and a
 *   non-primary context has its own copy.  The first call in a context also loads every kernel the forward
 *   can launch (module loading may allocate), so make that first call before any stream capture.  All
 *   calls share the one array and it keeps the last call's contents (the forward overwrites every scratch
 *   byte it reads), so calls that overlap on the GPU -- on different streams, or from several threads --
 *   race; serialize them.
 */
QL_API ql_status qlora_linear_fwd_noalloc(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x,
                                          const uint8_t* codes, const float* absmax, const uint16_t* A,
                                          const uint16_t* B, float s, uint16_t* y, uint16_t* su_out, void* stream);

/*
 * qlora_linear_bwd -- gradients of the layer with the base weight frozen ("How LoRA and QLoRA work": only
 * the adapters train; "Unsloth v0.1.47-beta ..." (kongchang.com), section on LoRA/QLoRA: the rewritten
 * backward keeps numerical equivalence).
 *   dy          bf16 [M,N] upstream gradient.
 *   x, codes, absmax, A, B, s   as in the forward (same size rules).
 *   su          nullable bf16 [M,r]: the forward's su_out; recomputed when NULL.
 *   dx          nullable bf16 [M,K] out: dY deq(W) + s (dY B) A.
 *   dA          nullable fp32 [r,K] out: s (dY B)^T x.
 *   dB          nullable fp32 [N,r] out: s dY^T (x A^T).
 *   workspace, ws_bytes  at least qlora_workspace_bytes(M,N,K,r,QL_PASS_BWD) bytes.
 * deq(W)^T tiles are formed in shared memory on the fly (never in global memory).  M = 0 writes dA = 0
 * and dB = 0.  Deterministic for given sizes.
 */
QL_API ql_status qlora_linear_bwd(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* dy, const uint16_t* x,
                           const uint8_t* codes, const float* absmax, const uint16_t* A, const uint16_t* B,
                           float s, const uint16_t* su, uint16_t* dx, float* dA, float* dB, void* workspace,
                           size_t ws_bytes, void* stream);

/*
 * qlora_swiglu_fwd -- h = silu(g) * u elementwise, silu(g) = g / (1 + exp(-g)), in fp32, h rounded to
 * bf16 ("Inside Unsloth ...", section "What You'll Learn", item "Triton Kernel Internals": the fused
 * SwiGLU; "unsloth", pyshine.com: swiglu.py fuses the gated MLP activation).
 *   numel >= 0; g, u, h bf16 [numel].
 */
QL_API ql_status qlora_swiglu_fwd(int64_t numel, const uint16_t* g, const uint16_t* u, uint16_t* h, void* stream);

/*
 * qlora_swiglu_bwd -- dg = dh * u * sigma(g) (1 + g (1 - sigma(g))), du = dh * silu(g), in fp32, rounded
 * to bf16.  numel >= 0; all buffers bf16 [numel].  dg/du may alias dh (read before write per element).
 */
QL_API ql_status qlora_swiglu_bwd(int64_t numel, const uint16_t* dh, const uint16_t* g, const uint16_t* u, uint16_t* dg,
                           uint16_t* du, void* stream);

/*
 * qlora_swiglu_gated_fwd -- SwiGLU over the output of the fused gate/up projection of a gated MLP
 * ("Inside Unsloth ...", section "What You'll Learn", item "Triton Kernel Internals": the SwiGLU kernels).
 * gu is bf16 [M, 2F]: row m holds the gate pre-activation g in columns [0, F) and the up projection in
 * [F, 2F) -- the y of qlora_linear_fwd on the stacked weight [W_gate; W_up].  h = silu(g) * up, bf16
 * [M, F], computed in fp32.  F % 8 == 0; buffers 16-byte aligned.
 */
QL_API ql_status qlora_swiglu_gated_fwd(int64_t M, int64_t F, const uint16_t* gu, uint16_t* h, void* stream);

/*
 * qlora_swiglu_gated_bwd -- its backward: dgu [M, 2F] bf16 receives dh * up * silu'(g) in columns [0, F)
 * and dh * silu(g) in [F, 2F): the upstream gradient of the stacked gate/up projection.  dh bf16 [M, F].
 */
QL_API ql_status qlora_swiglu_gated_bwd(int64_t M, int64_t F, const uint16_t* dh, const uint16_t* gu,
                                        uint16_t* dgu, void* stream);

/* ------------------------------------------------------------------------------------------------------
 * Layer calls on a weight in any supported format.
 * ------------------------------------------------------------------------------------------------------ */

typedef enum { QL_W_NF4 = 0, QL_W_NF4_DQ = 1, QL_W_NVFP4 = 2 } ql_wformat;

/* A frozen base weight W [N,K] (K a multiple of 64); all pointers device pointers, 16-byte aligned.
 *   QL_W_NF4     codes [N*K/2] (nf4_quantize), absmax [N*K/64] fp32.
 *   QL_W_NF4_DQ  codes, and the double-quantized constants of nf4_double_quantize: code8 [N*K/64] (readable to
 *                a multiple of 4 bytes), c1 [ceil(N*K/64/256)] fp32, mu [1] fp32.
 *   QL_W_NVFP4   codes [N*K/2] and scales [N*K/16] of nvfp4_quantize, tensor_scale [1] fp32.
 * Pointers a format does not use are ignored. */
typedef struct {
  int format; /* ql_wformat */
  const uint8_t* codes;
  const float* absmax;
  const uint8_t* code8;
  const float* c1;
  const float* mu;
  const uint8_t* scales;
  const float* tensor_scale;
} ql_weight;

/* qlora_linear_fwd / qlora_linear_bwd on a ql_weight: the same operation, layouts, workspace and errors, with
 * deq(W) the weight's own dequantization (NF4: level * absmax; NF4_DQ: level * absmax' with the constants'
 * double dequantization; NVFP4: E2M1 value * decoded group scale).  QL_ERR_INVALID_ARG for an unknown format or
 * a null or misaligned pointer the format uses. */
QL_API ql_status qlora_linear_fwd_w(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x, const ql_weight* w,
                                    const uint16_t* A, const uint16_t* B, float s, uint16_t* y, uint16_t* su_out,
                                    void* workspace, size_t ws_bytes, void* stream);
QL_API ql_status qlora_linear_bwd_w(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* dy, const uint16_t* x,
                                    const ql_weight* w, const uint16_t* A, const uint16_t* B, float s,
                                    const uint16_t* su_in, uint16_t* dx, float* dA, float* dB, void* workspace,
                                    size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------------------
 * Gated MLP with the SwiGLU fused into the projections' epilogues.
 *
 * The gate/up projection is one layer over the stacked weight [2F, K] in the INTERLEAVED row order: within
 * every 32 rows, the 16 gate rows of features 16q .. 16q + 15, then the 16 up rows of the same features
 * (gate feature f at row 32 (f / 16) + f % 16, up feature f 16 rows below).  Its output gu [M, 2F] has the
 * same column order.  F % 16 == 0.
 * ------------------------------------------------------------------------------------------------------ */

/* Workspace of the gated calls (the forward: that of qlora_linear_fwd; the down backward: that of
 * qlora_linear_bwd plus, when its dX GEMM splits its contraction, a dh buffer of M*F bf16). */
QL_API size_t qlora_gated_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r, ql_pass pass);

/* Forward of the interleaved gate/up layer (qlora_linear_fwd with N = 2F) that also writes
 * h [M, F] bf16 = silu(g) * up, g and up the bf16 values written to gu.  Bit-identical to qlora_linear_fwd
 * followed by the SwiGLU of gu. */
QL_API ql_status qlora_gate_up_fwd_swiglu(int64_t M, int64_t F, int64_t K, int64_t r, const uint16_t* x,
                                          const uint8_t* codes, const float* absmax, const uint16_t* A,
                                          const uint16_t* B, float s, uint16_t* gu, uint16_t* h, uint16_t* su_out,
                                          void* workspace, size_t ws_bytes, void* stream);

/* Backward of the down projection (W [N, F], input h) whose input gradient dh goes straight into the SwiGLU
 * backward: dgu [M, 2F] (interleaved) = (dh * up * silu'(g), dh * silu(g)) with dh rounded to bf16 and g, up
 * read from gu.  dA, dB as in qlora_linear_bwd.  Bit-identical to qlora_linear_bwd (dX = dh) followed by the
 * SwiGLU backward. */
QL_API ql_status qlora_down_bwd_dswiglu(int64_t M, int64_t N, int64_t F, int64_t r, const uint16_t* dy,
                                        const uint16_t* h, const uint8_t* codes, const float* absmax,
                                        const uint16_t* A, const uint16_t* B, float s, const uint16_t* su,
                                        const uint16_t* gu, uint16_t* dgu, float* dA, float* dB, void* workspace,
                                        size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------------------------------
 * Weight-format conversions (their own translation unit; their own launch counter and device error word).
 * ------------------------------------------------------------------------------------------------------ */

/* Number of format-conversion kernels launched in the process so far (all devices).  Host-only. */
QL_API uint64_t ql_formats_launch_count(void);

/* Reads and clears the format conversions' device error word after synchronizing `stream`.  Returns
 * QL_ERR_INVALID_ARG if a conversion met a non-finite input (or a negative block constant, or a NaN code),
 * QL_OK otherwise, or QL_ERR_CUDA.  Synchronizes. */
QL_API ql_status ql_formats_get_device_error(void* stream);

/*
 * nf4_double_quantize -- double quantization of the NF4 block constants ("Unsloth v0.1.463-beta: Fixes
 * Studio Crash and llama-server Permission Issue", kongchang.com, section "About the Unsloth Project",
 * paragraph "How LoRA and QLoRA work": QLoRA quantizes its quantization constants a second time).
 *   absmax   [nb] fp32, the block constants as nf4_quantize writes them (finite, >= 0), nb >= 1.
 *   code8    [nb] uint8 out: per constant, the E4M3 bit pattern of the level nearest to n = fl32(d / c1),
 *            d = fl32(absmax - mu); the levels are the finite E4M3 values / 448 rounded to fp32; a tie
 *            goes to the lower level; c1 = 0 gives code 0x00.
 *   c1       [ceil(nb / 256)] fp32 out: per group of 256 consecutive constants (the last may be shorter),
 *            max |d| over the group.
 *   mu       [1] fp32 out (device): the mean of all constants, summed in fp64 group by group in index
 *            order, the group sums added in order, divided by nb in fp64, rounded to fp32.
 *   scratch  device scratch of at least nf4_double_quantize_scratch_bytes(nb) bytes (the group sums).
 * Dequantized by nf4_double_dequantize.  Storage: about 0.127 bit per weight instead of 0.5.  Bit-exact and
 * deterministic.  All pointers 16-byte aligned.  QL_ERR_INVALID_ARG on bad sizes, null or misaligned
 * pointers, or too little scratch.  A non-finite or negative constant is recorded in the format device
 * error word.  The mean is one sequential fp64 sum over the groups: a one-time conversion.
 */
QL_API size_t nf4_double_quantize_scratch_bytes(int64_t nb);
QL_API ql_status nf4_double_quantize(const float* absmax, int64_t nb, uint8_t* code8, float* c1, float* mu,
                                     void* scratch, size_t scratch_bytes, void* stream);

/*
 * nf4_double_dequantize -- absmax'[i] = fl32(fl32(L[code8[i]] * c1[i / 256]) + mu), fp32 [nb], from the
 * outputs of nf4_double_quantize (mu a device pointer).  A NaN code (0x7F, 0xFF) gives NaN and is recorded
 * in the format device error word.  Bit-exact.  Pointers 16-byte aligned.
 */
QL_API ql_status nf4_double_dequantize(const uint8_t* code8, const float* c1, const float* mu, int64_t nb,
                                       float* absmax_out, void* stream);

/*
 * nvfp4_quantize -- NVFP4 quantization of a weight ("Major Unsloth Update: NVFP4 Quantization Export and
 * DeepSeek-V4 Training Support", kongchang.com, section "NVFP4: A Quantization Format for the Next
 * Generation of Hardware": E2M1 values with a range of about +-6, one FP8 scale per small group).
 *   w            [numel] fp32, flat row-major; numel a positive multiple of 16 (blocks never straddle rows
 *                when the row length is a multiple of 16).
 *   codes        [numel / 2] uint8 out: E2M1 patterns, element 2j in the LOW nibble of byte j.
 *   scales       [numel / 16] uint8 out: E4M3 pattern of each block's scale.
 *   tensor_scale [1] fp32 out (device): S = fl32(amax / 2688), amax = max |w| (0 for an all-zero tensor).
 * Per block of 16 with largest magnitude a: t = fl32(a / fl32(6 S)); scale = E4M3 of t (nearest, ties to
 * even, saturating at 448); D = fl32(value(scale) * S); code = E2M1 of fl32(w / D) (nearest, ties to the
 * even mantissa, saturating at 6, sign kept), or +0 when D = 0.  Bit-exact and deterministic.  Pointers
 * 16-byte aligned.  A non-finite weight is recorded in the format device error word.
 */
QL_API ql_status nvfp4_quantize(const float* w, int64_t numel, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                void* stream);

/*
 * nvfp4_dequantize -- w' = fl32(value(code) * D), D = fl32(value(scale) * S), from the outputs of
 * nvfp4_quantize.  out_dtype QL_F32: out is float[numel]; QL_BF16: bf16[numel], round-to-nearest-even of
 * w'.  Bit-exact.  Pointers 16-byte aligned.
 */
QL_API ql_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                                  int64_t numel, ql_dtype out_dtype, void* out, void* stream);

/*
 * The NVFP4 form of the layer on the block-scaled FP4 tensor core ("Major Unsloth Update: NVFP4 Quantization Export
 * and DeepSeek-V4 Training Support" (kongchang.com), section "NVFP4: A Quantization Format for the Next Generation
 * of Hardware": E2M1 values sharing an FP8 scale per group, multiplied directly by Blackwell's FP4 tensor cores).
 *
 * nvfp4_scales_to_mma -- lays a weight's NVFP4 scales (nvfp4_quantize's row-major [rows, K/16] E4M3 bytes) out as
 * the tensor core reads them: rows in blocks of 128, K in steps of 64 elements (4 scales), one 512-byte atom per
 * (row block, step), the steps of a row block consecutive and padded with zero scales to a multiple of 4, row
 * blocks consecutive; inside an atom the scale of group g of row 32 r1 + r0 is byte 16 r0 + 4 r1 + g.  Rows past
 * `rows` up to the next multiple of 128 hold zero scales.
 *   rows >= 1, K >= 64 with K % 64 == 0; out 16-byte aligned, nvfp4_mma_scales_bytes(rows, K) bytes.  Runs once
 *   per frozen weight.
 */
QL_API size_t nvfp4_mma_scales_bytes(int64_t rows, int64_t K);
QL_API ql_status nvfp4_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t K, uint8_t* out, void* stream);

/*
 * qlora_linear_fwd_fp4 -- y = q(x) q(W)^T + s (x A^T) B^T, with q() the NVFP4 rule of nvfp4_quantize (E2M1 codes,
 * an E4M3 scale per 16 elements along K, one fp32 tensor scale per operand).  The weight comes quantized (codes,
 * its scales in the MMA layout of nvfp4_scales_to_mma, its tensor scale on the device); the activations are
 * quantized by the same rule on every call, with their own tensor scale, into the workspace.  The base product
 * runs as tcgen05.mma kind::mxf4nvf4 with 16-element scale blocks into one TMEM accumulator, scaled by both tensor
 * scales in the epilogue; the rank-r term keeps the unquantized activations: su = s x A^T is rounded to bf16 and
 * multiplied by B with bf16 MMAs into a second accumulator.
 *   M, N, K, r   as qlora_linear_fwd (K % 64 == 0, N % 8 == 0, r % 8 == 0, r <= 256).
 *   x            bf16 [M,K], 16-byte aligned.
 *   w_codes      uint8 [N, K/2]: E2M1 codes, element 2j in the low nibble of byte j (nvfp4_quantize of W [N,K]).
 *   w_sf_mma     the weight's scales in the MMA layout, w_S its fp32 tensor scale (device).
 *   A, B, s      the LoRA pair and scaling (unused when r = 0).
 *   y            bf16 [M,N] out; su_out nullable bf16 [M,r] out (s x A^T).
 *   workspace    qlora_fp4_workspace_bytes(M,N,K,r) bytes: the activations' codes, scales and tensor scale, su.
 * Errors as qlora_linear_fwd; a non-finite activation sets the device error word (QL_ERR_INVALID_ARG from
 * ql_get_device_error).
 */
QL_API size_t qlora_fp4_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t r);
QL_API ql_status qlora_linear_fwd_fp4(int64_t M, int64_t N, int64_t K, int64_t r, const uint16_t* x,
                                      const uint8_t* w_codes, const uint8_t* w_sf_mma, const float* w_S,
                                      const uint16_t* A, const uint16_t* B, float s, uint16_t* y, uint16_t* su_out,
                                      void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
