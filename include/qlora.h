/*
 * qlora.h -- C ABI of the frozen-NF4 linear layer with a LoRA adapter,
 * for NVIDIA B200 (sm_100a).
 *
 * What the calls compute (sources are the web pages on QLoRA this library
 * restates; they describe the method in prose, without formulas):
 *   - "AI Glossary: QLoRA" (mangrove.ai), definition and second paragraph:
 *     the frozen weights are stored as 4-bit numbers; each time the layer is
 *     used they are turned back into BFloat16 for the product; weight
 *     gradients are computed only for the LoRA matrices; NF4 is the 4-bit
 *     type for normally distributed values; the scaling constants are
 *     themselves quantized.
 *   - "QLoRA: Fine-Tuning 65-Billion Parameter Models on a Single Consumer
 *     GPU" (deepfa.ir): "LoRA: Prerequisite for Understanding QLoRA" (the
 *     update is a d x r times r x k product), "QLoRA's Technical Innovations"
 *     (1. 4-bit NormalFloat, 2. Double Quantization) and "QLoRA's Working
 *     Process" (quantize, freeze, add bf16 adapters, backpropagate through the
 *     frozen 4-bit weights, dequantize on the fly).
 *
 * Conventions shared by every call:
 *   - bf16 tensors are passed as uint16_t bit patterns; all tensors are
 *     row-major and contiguous.
 *   - W  [N x K]  frozen weight (out x in).  X [M x K].  A [K x r].
 *     B [r x N].  Y, dY [M x N].  The LoRA scale s is a float argument.
 *   - Every pointer is a DEVICE pointer, 16-byte aligned, allocated and owned
 *     by the caller.  The library allocates no device memory and frees none.
 *   - `stream` is a cudaStream_t (passed as void*); every call only enqueues
 *     work on it and returns without synchronising.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns an error and enqueues nothing.  QLORA_ERR_CUDA
 *     means a launch failed (see qlora_last_cuda_error).
 *
 * Packed NF4 format (the layout every call below agrees on):
 *   - Flatten W row-major; blocks of 64 consecutive elements share one
 *     absmax constant c_b; groups of 256 consecutive blocks share one float
 *     c1 = max c_b.  NB = ceil(numel / 64) blocks, NB2 = ceil(NB / 256) groups.
 *   - codes        uint8[ceil(numel / 2)]: element 2j in the high nibble of
 *                  byte j, element 2j + 1 in the low nibble; the code is the
 *                  index (0..15) of the nearest NF4 level to fp32(x / c_b),
 *                  ties to the lower index, 7 (the exact zero) for an
 *                  all-zero block and for a padding nibble.
 *   - absmax_q     uint8[NB]: nearest k in 0..255 of fp32(k / 255) to
 *                  fp32(c_b / c1), ties to the lower k, 0 when c1 = 0.
 *   - absmax_scale float[NB2]: c1 per group.
 *   - Dequantized weight: a' = fp32(fp32(k / 255) * c1),
 *                         w' = bf16_rne(fp32(q[code] * a')).
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, non-finite scale */
  QLORA_ERR_ALIGNMENT = 2,   /* a pointer is not 16-byte aligned */
  QLORA_ERR_UNSUPPORTED = 3, /* a shape outside the supported set (see each call) */
  QLORA_ERR_WORKSPACE = 4,   /* workspace pointer null or smaller than qlora_workspace_bytes */
  QLORA_ERR_CUDA = 5,        /* a CUDA launch or query failed */
  QLORA_ERR_TIMEOUT = 6      /* a kernel gave up waiting on a pipeline barrier (qlora_check_status) */
} qlora_status;

/*
 * 4-bit codes of the packed format.  NF4 is the method's type; FP4 and Int4
 * are the two 4-bit types the pages compare it with ("1. 4-bit NormalFloat
 * (NF4)": Integer 4-bit and Float 4-bit, with NF4 the lower-error one;
 * "Performance and Evaluation", "NF4 efficiency").  The pages define neither;
 * this library reads them as
 *   QLORA_CODE_FP4   the float with 1 sign, 2 exponent and 1 mantissa bit
 *                    (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) divided by 6,
 *   QLORA_CODE_INT4  the symmetric integer code k / 7, k = -7..7.
 * Both keep everything else of the packed format (blocks of 64, double
 * quantization, nibble order, zero level at index 7).  Their 15 distinct
 * levels fill indices 0..14 in ascending order and index 15 repeats +1; the
 * nearest-level rule (ties to the lower index) never produces code 15.
 */
typedef enum { QLORA_CODE_NF4 = 0, QLORA_CODE_FP4 = 1, QLORA_CODE_INT4 = 2 } qlora_code;

/*
 * Second reading of "2. Double Quantization" (the pages say only that the
 * constants are quantized; this is the original QLoRA paper's variant, not
 * printed on the pages).  OR-ed into a qlora_code, it codes the constants as
 * 8-bit floats after removing their mean:
 *   mu   = fp32(exact mean of every block absmax c_b of the tensor)
 *   s_g  = fp32(max |fp32(c_b - mu)| over the 256-group / 448)
 *   k_b  = E4M3 code (sign, 4 exponent bits with bias 7, 3 mantissa bits)
 *          nearest to fp32(fp32(c_b - mu) / s_g), ties to the even code,
 *          saturating at +-448, -0 kept; 0 when s_g = 0
 *   a'   = fp32(fp32(E4M3(k_b) * s_g) + mu)
 * absmax_q holds k_b; absmax_scale holds NB2 + 1 floats: s_g per group,
 * then mu.  The 4-bit codes still use the true c_b.  Quantization runs three
 * kernels (exact per-exponent sums of the absmaxes in a device array of this
 * library, their mean, then the codes): centred quantizations on one device
 * must not overlap on the GPU, and numel is limited to 2^38.
 */
#define QLORA_DQ_CENTRED_FP8 0x100

/*
 * Blockwise NF4 quantization with double-quantized constants.
 * "AI Glossary: QLoRA", second paragraph; "1. 4-bit NormalFloat (NF4)" and
 * "2. Double Quantization" in "QLoRA: Fine-Tuning 65-Billion Parameter
 * Models ...".
 *   W             in   bf16[numel]      any numel >= 1 (a partial last block
 *                                       takes its absmax over the elements
 *                                       present, a partial last group its max
 *                                       over the constants present)
 *   codes         out  uint8[ceil(numel/2)]
 *   absmax_q      out  uint8[NB]
 *   absmax_scale  out  float[NB2]
 * Deterministic: the result depends only on W.
 */
QLORA_API qlora_status qlora_quantize_nf4(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* absmax_q,
                                float* absmax_scale, void* stream);

/* The same quantization with the levels of `code` (a qlora_code, optionally
 * OR QLORA_DQ_CENTRED_FP8; any other value returns QLORA_ERR_INVALID_ARG).
 * qlora_quantize_nf4 is this call with QLORA_CODE_NF4. */
QLORA_API qlora_status qlora_quantize_4bit(const uint16_t* W, int64_t numel, int32_t code, uint8_t* codes,
                                           uint8_t* absmax_q, float* absmax_scale, void* stream);

/*
 * Dequantization to bf16 (the weight the linear calls multiply by).
 * "AI Glossary: QLoRA", second paragraph (4-bit weights turned back into
 * BFloat16 for the calculation).
 *   codes, absmax_q, absmax_scale  in   packed format above, for numel weights
 *   W_out                          out  bf16[numel]
 */
QLORA_API qlora_status qlora_dequantize_nf4(const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                                  int64_t numel, uint16_t* W_out, void* stream);

/* Dequantization of a weight packed with the levels of `code`. */
QLORA_API qlora_status qlora_dequantize_4bit(const uint8_t* codes, const uint8_t* absmax_q,
                                             const float* absmax_scale, int64_t numel, int32_t code,
                                             uint16_t* W_out, void* stream);

/*
 * Forward of the frozen-NF4 linear layer with a LoRA adapter.
 * "AI Glossary: QLoRA", second paragraph; "LoRA: Prerequisite for
 * Understanding QLoRA"; "QLoRA's Working Process", steps 3-4.
 *   T_save = fp32(s * X A)                [M x r]   (kept for the backward)
 *   Y      = bf16(X W'^T + T_save B)      [M x N]   (fp32 accumulation)
 * where W' is the dequantized weight, decoded tile by tile inside the
 * product (no bf16 copy of W is written).  T enters the tensor-core product
 * as the bf16 pair hi = bf16(T), lo = bf16(T - hi) (about 16 significant
 * bits), so it loses no accuracy to a bf16 rounding.
 *   X             in   bf16[M x K]
 *   codes...      in   packed W [N x K] (numel = N*K)
 *   A             in   bf16[K x r]
 *   B             in   bf16[r x N]
 *   Y             out  bf16[M x N]
 *   T_save        out  float[M x r]
 *   workspace     in/out device scratch of at least qlora_workspace_bytes(M,K,N,r)
 *                 bytes, filled with zeros once before its first use.  It
 *                 holds the status word read by qlora_check_status (first
 *                 256 bytes) and counters that every call leaves at zero;
 *                 everything else is overwritten before it is read.  After
 *                 qlora_check_status reports QLORA_ERR_TIMEOUT, fill it with
 *                 zeros again before the next call.
 * Supported: K % 64 == 0, N % 8 == 0 (the weight's blocks and the row
 * strides of Y, dY and B, which are copied by TMA, in 16-byte units),
 * 1 <= r <= 256, M, N, K < 2^31.  Otherwise QLORA_ERR_UNSUPPORTED.  Ranks
 * that are not multiples of 8 run with A, B, T_save, dA and dB padded with
 * zeros to the next multiple of 8 inside the workspace (a few small copy
 * kernels around the GEMM); ranks above 128 always take the pair GEMMs.
 * For up to 8 tokens (up to 16 when N*K >= 2^27) the forward is two
 * launches chained by programmatic dependent launch: a weight stream that
 * also forms T, and a small kernel that sums its partials and adds T B;
 * neither needs its blocks to be resident together.  On this path the block
 * constant multiplies each 64-input block's partial product (bf16 level
 * times x, float32 sums) rather than each weight; either way a term carries
 * one bf16 rounding.  For other M <= 128 the forward is one launch whose
 * thread blocks wait for one another (cooperative launch: all of them must
 * be resident at once); if the device cannot hold them next to other work
 * the call returns QLORA_ERR_CUDA and launches nothing.  For larger M it is
 * one launch in which blocks that finished T for a 512-row block release
 * the output tiles of those rows (work is handed out in that order, so no
 * residency is needed).  Sums are taken in a fixed order: results are
 * bit-reproducible run to run.
 */
QLORA_API qlora_status qlora_linear_fwd(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* codes,
                              const uint8_t* absmax_q, const float* absmax_scale, const uint16_t* A,
                              const uint16_t* B, int32_t r, float scale, uint16_t* Y, float* T_save,
                              void* workspace, size_t ws_bytes, void* stream);

/* qlora_linear_fwd for a weight packed with the levels of `code`. */
QLORA_API qlora_status qlora_linear_fwd_4bit(const uint16_t* X, int64_t M, int64_t K, int64_t N,
                                             const uint8_t* codes, const uint8_t* absmax_q,
                                             const float* absmax_scale, int32_t code, const uint16_t* A,
                                             const uint16_t* B, int32_t r, float scale, uint16_t* Y, float* T_save,
                                             void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward of the same layer for an upstream gradient dY.  Gradients are
 * produced only for the adapter; the frozen base weight gets none
 * ("AI Glossary: QLoRA", second paragraph; "QLoRA's Working Process",
 * step 5: gradients flow through the frozen 4-bit weights into LoRA).
 *   U  = s * dY B^T           fp32        [M x r]   (workspace, as a bf16 pair)
 *   dB = T_save^T dY          fp32        [r x N]
 *   dX = bf16(dY W' + U A^T)              [M x K]
 *   dA = X^T U                fp32        [K x r]
 *   dY, X          in   bf16
 *   T_save         in   float[M x r] as written by qlora_linear_fwd
 *   dX             out  bf16[M x K]
 *   dA, dB         out  float (overwritten, not accumulated)
 * Same supported shapes and workspace rule as qlora_linear_fwd.  Results
 * are bit-reproducible run to run.
 * Each reduction (U over N; dA, dB over M) is a single float32 chain in
 * tensor-core accumulators, in a fixed order.
 */
QLORA_API qlora_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, const float* T_save, int64_t M, int64_t K,
                              int64_t N, const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                              const uint16_t* A, const uint16_t* B, int32_t r, float scale, uint16_t* dX, float* dA,
                              float* dB, void* workspace, size_t ws_bytes, void* stream);

/* qlora_linear_bwd for a weight packed with the levels of `code`. */
QLORA_API qlora_status qlora_linear_bwd_4bit(const uint16_t* dY, const uint16_t* X, const float* T_save, int64_t M,
                                             int64_t K, int64_t N, const uint8_t* codes, const uint8_t* absmax_q,
                                             const float* absmax_scale, int32_t code, const uint16_t* A,
                                             const uint16_t* B, int32_t r, float scale, uint16_t* dX, float* dA,
                                             float* dB, void* workspace, size_t ws_bytes, void* stream);

/*
 * qlora_linear_fwd without a workspace argument, for callers that cannot
 * allocate device memory (code running inside an allocator or memory-pool
 * callback, on a path where the framework forbids allocation, or in an
 * embedding that owns all device memory up front).  The QLoRA pages have no
 * counterpart to this call; it exists for those callers only.
 *   Same arguments, outputs and supported shapes as qlora_linear_fwd, minus
 *   workspace/ws_bytes and ranks that are not multiples of 8
 *   (QLORA_ERR_UNSUPPORTED: the padded adapter needs a workspace); the
 *   results agree with qlora_linear_fwd to within
 *   float32 summation order: for every M this call runs the pair GEMM of the
 *   large-M forward, while qlora_linear_fwd takes the weight-streaming kernel
 *   for M <= 128.
 *   The call allocates nothing:
 *   its scratch is one fixed 16 MiB device array inside this library, which
 *   every GPU that loads the library keeps until the process exits.
 *   - Shapes whose forward scratch (status word, counters and the bf16 pair
 *     of T: 256 + round256(4*(2 + ceil(M/512))) + round256(4*M*rp) bytes with
 *     rp = r rounded up to 64) exceeds 16 MiB return QLORA_ERR_WORKSPACE and
 *     launch nothing; 4096 tokens at r = 64 need about 1 MiB, so up to 32768
 *     tokens fit at r <= 64.
 *   - The first call on a device (with that device current, and `stream`
 *     belonging to it) looks up the array's device address once; make that
 *     first call before any stream capture on that device.
 *   - All calls on a device share the array.  Calls that may overlap on the
 *     GPU (other streams, or host threads without ordering) race and must be
 *     serialised by the caller.
 *   - Each call clears the counters it uses.  A pipeline wait that gives up
 *     sets the array's status word, which stays set until
 *     qlora_check_status(NULL, stream) (or with any workspace) on that device
 *     reports QLORA_ERR_TIMEOUT and clears it.
 *   - For M > 128 it runs the same GEMM launch as qlora_linear_fwd and gives
 *     the same bits.
 */
QLORA_API qlora_status qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, int64_t K, int64_t N,
                                                const uint8_t* codes, const uint8_t* absmax_q,
                                                const float* absmax_scale, const uint16_t* A, const uint16_t* B,
                                                int32_t r, float scale, uint16_t* Y, float* T_save, void* stream);

/*
 * SiLU gate between the linears of a gated MLP (the LLaMA feed-forward block
 * the QLoRA experiments fine-tune): glue between LoRA linears, not a step of
 * the method, so the pages have no counterpart.  Elementwise over n values,
 * float32 arithmetic, one bf16 rounding per output:
 *   forward   H  = silu(G) * U = G * sigmoid(G) * U
 *   backward  dG = dH * U * sigmoid(G) * (1 + G * (1 - sigmoid(G)))
 *             dU = dH * G * sigmoid(G)
 * All pointers bf16[n], 16-byte aligned; outputs may not alias inputs.
 */
QLORA_API qlora_status qlora_silu_gate_fwd(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n,
                                           void* stream);
QLORA_API qlora_status qlora_silu_gate_bwd(const uint16_t* G, const uint16_t* U, const uint16_t* dH, uint16_t* dG,
                                           uint16_t* dU, int64_t n, void* stream);

/*
 * Paged optimizer for the LoRA parameters.  "3. Paged Optimizers" and "AI
 * Glossary: QLoRA", second paragraph: only the LoRA matrices are trained,
 * and their optimizer states live in NVIDIA unified memory so that they can
 * move between GPU and CPU memory during memory spikes.
 *
 * qlora_paged_malloc / qlora_paged_free: unified (managed) memory for the
 * optimizer states, with the allocate/free signatures of PyTorch's pluggable
 * allocator (size, device, stream) / (ptr, size, device, stream).  These are
 * the only calls of this library that allocate; the memory belongs to the
 * caller.  malloc returns NULL on failure (qlora_last_cuda_error says why).
 * free synchronises `stream` (if any) before releasing the memory.
 *
 * qlora_paged_prefetch: asynchronously moves [ptr, ptr + bytes) to the
 * current device (to_device != 0) or to host memory (to_device == 0) on
 * `stream`.  Kernels may touch the memory wherever it is: pages that are on
 * the host migrate on demand.  qlora_paged_location reports where the range
 * was last prefetched (a device index, or -1 for the host).
 *
 * qlora_adamw_step: one AdamW step over n float32 parameters, in place:
 *   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2
 *   p = p - lr (m / (1 - b1^step) / (sqrt(v / (1 - b2^step)) + eps) + wd p)
 * step >= 1 counts the steps taken so far including this one; m and v start
 * at zero.  param_bf16 (may be NULL) receives bf16_rne(p), the adapter the
 * linear calls read.  param, grad, m, v: float[n], 4-byte aligned (16-byte
 * alignment takes the vector path); param_bf16 2-byte aligned.  The step is
 * the textbook AdamW; the pages name no optimizer formula.
 */
QLORA_API void* qlora_paged_malloc(size_t size, int device, void* stream);
QLORA_API void qlora_paged_free(void* ptr, size_t size, int device, void* stream);
QLORA_API qlora_status qlora_paged_prefetch(const void* ptr, size_t bytes, int32_t to_device, void* stream);
QLORA_API qlora_status qlora_paged_location(const void* ptr, size_t bytes, int32_t* location);
QLORA_API qlora_status qlora_adamw_step(float* param, uint16_t* param_bf16, const float* grad, float* m, float* v,
                                        int64_t n, int32_t step, float lr, float beta1, float beta2, float eps,
                                        float weight_decay, void* stream);

/* Workspace bytes needed by qlora_linear_fwd / qlora_linear_bwd for these sizes
 * (0 for an unsupported shape). */
QLORA_API size_t qlora_workspace_bytes(int64_t M, int64_t K, int64_t N, int32_t r);

/* Synchronises `stream`, then reads the status words: the one at the start
 * of `workspace` (skipped when workspace is NULL) and the two the library
 * keeps on the current device for calls that take no workspace
 * (qlora_quantize_nf4 and qlora_linear_fwd_noalloc).  Returns QLORA_OK, or
 * QLORA_ERR_TIMEOUT if a kernel of an earlier call gave up on a pipeline wait
 * (its outputs are then undefined).  Every word read is reset to zero. */
QLORA_API qlora_status qlora_check_status(void* workspace, void* stream);

/* Limit of every bounded wait inside the kernels (a pipeline barrier, a
 * count another thread block raises, a grid barrier), in nanoseconds; 0
 * restores the default of 2 s.  A wait that reaches the limit makes its
 * kernel stop waiting, let its own copies and tensor-core work end, free its
 * tensor memory and exit; qlora_check_status then reports QLORA_ERR_TIMEOUT.
 * Applies to launches made after the call, from any host thread.  Limits
 * above 60 s return QLORA_ERR_INVALID_ARG.  No counterpart on the pages:
 * failure handling of this library. */
QLORA_API qlora_status qlora_set_wait_timeout(uint64_t timeout_ns);
QLORA_API uint64_t qlora_get_wait_timeout(void);

/* The 16 NF4 levels (float32, ascending) this library encodes against. */
QLORA_API void qlora_nf4_codebook(float out[16]);

/* The 16 levels of `code` (float32, ascending; see qlora_code). */
QLORA_API qlora_status qlora_codebook(int32_t code, float out[16]);

/* Static description of a status code. */
QLORA_API const char* qlora_status_string(qlora_status s);

/* The last CUDA error string seen by a call of this thread ("" if none). */
QLORA_API const char* qlora_last_cuda_error(void);

/*
 * Optional kernel timing (no counterpart on the pages; measurement support).
 * qlora_profile_start clears earlier records and makes every later call of
 * this library record a pair of CUDA events on its stream around each of its
 * kernels (the rank-r products count their split and reduction launches as
 * one record).  qlora_profile_stop synchronises those events, disables the
 * recording and writes up to max_entries aggregated rows: names (48 bytes
 * each, NUL-terminated), total milliseconds, number of records and number of
 * kernel launches; it returns the number of rows written.
 */
QLORA_API void qlora_profile_start(void);
QLORA_API int qlora_profile_stop(int max_entries, char* names, float* total_ms, int* calls, int* launches);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
