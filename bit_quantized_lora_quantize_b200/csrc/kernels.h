// Internal host-side launch interface between the C-ABI layer (abi.cu) and
// the kernels.  Not part of the public header.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "nf4_device.cuh"

namespace qlora {

// Limit of every bounded wait in the kernels, as set by
// qlora_set_wait_timeout (kWaitTimeoutNs by default, at most
// kMaxWaitTimeoutNs).  Each launch copies it into its arguments.
constexpr uint64_t kMaxWaitTimeoutNs = 60000000000ull;  // 60 s
uint64_t wait_limit_ns();

// Multiprocessor count and L2 size of the current device, read once per
// device (148 SMs and 126 MB when they cannot be read).  Safe to call from
// several host threads.
int device_sm_count();
int device_l2_bytes();

// Status words the library keeps on the device for calls without a
// workspace: each reads the current device's word (after the stream's work),
// clears it if it was set and returns it in *word.
cudaError_t codec_status_take(cudaStream_t stream, int* word);
cudaError_t noalloc_status_take(cudaStream_t stream, int* word);

// Launch attribute that lets a kernel start before its predecessor in the
// stream has ended (programmatic dependent launch).  Every kernel launched
// with it calls griddep_wait before it reads anything its predecessor writes
// and before it writes anything its predecessor reads.
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a{};
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

cudaError_t launch_quantize_nf4(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* absmax_q,
                                float* absmax_scale, const Nf4Params& P, cudaStream_t stream);

cudaError_t launch_dequantize_nf4(const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                                  int64_t numel, uint16_t* out, const Nf4Params& P, cudaStream_t stream);

// The rank-r intermediates T = s X A and U = s dY B^T enter the tensor-core
// products as a bf16 pair matrix [rows x 2*rp] (rp = r rounded up to 64):
// columns [0, r) hold hi = bf16(v), columns [rp, rp + r) hold
// lo = bf16(v - hi), all other columns are 0.  hi + lo carries v to about 16
// significant bits, so rounding the intermediates costs no accuracy.
inline int lora_pad(int r) { return (r + 63) / 64 * 64; }

// Fused dequant-GEMM, forward: Y[M,N] = X[M,K] W'[N,K]^T + (T_hi + T_lo)[M,r] B[r,N].
// With `ctr` (fused_ctr_ints(M) ints, zero, left at zero) the kernel also
// computes T = s X A itself (T_save float32 and the pair in Tpair) in units
// that run ahead of the output tiles; with ctr == nullptr Tpair must be the
// output of the previous kernel in the stream (A, T_save, scale unused).
cudaError_t launch_fused_fwd(const uint16_t* X, const uint8_t* codes, const uint8_t* absmax_q,
                             const float* absmax_scale, uint16_t* Tpair, const uint16_t* B, int64_t M, int64_t K,
                             int64_t N, int r, uint16_t* Y, int* status, const Nf4Params& P, cudaStream_t stream,
                             const uint16_t* A = nullptr, float* T_save = nullptr, float scale = 0.0f,
                             int* ctr = nullptr);

// Fused dequant-GEMM, input gradient: dX[M,K] = dY[M,N] W'[N,K] + (U_hi + U_lo)[M,r] A[K,r]^T.
// With `ctr` the kernel also computes U = s dY B^T (its pair in Upair) the
// same way, and, when dA and dB are given, dA = X^T U and dB = T^T dY (the
// rank units write the bf16 pair of T_save into Tpair for that); with
// ctr == nullptr Upair comes from the previous kernel.
cudaError_t launch_fused_dx(const uint16_t* dY, const uint8_t* codes, const uint8_t* absmax_q,
                            const float* absmax_scale, uint16_t* Upair, const uint16_t* A, int64_t M, int64_t K,
                            int64_t N, int r, uint16_t* dX, int* status, const Nf4Params& P, cudaStream_t stream,
                            const uint16_t* B = nullptr, float scale = 0.0f, int* ctr = nullptr,
                            const uint16_t* X = nullptr, const float* T_save = nullptr, uint16_t* Tpair = nullptr,
                            float* dA = nullptr, float* dB = nullptr);

// Counter ints one fused launch with rank units needs for M rows.
int fused_ctr_ints(int64_t M);

// Small-M forward (M <= kSmallMMax tokens): the whole forward (T = s X A, its
// pair and Y) in one launch of a persistent weight-streaming kernel.
// `scratch` holds small_m_workspace_bytes(M, N, r) bytes, zero before the
// first call; the kernel leaves its counters at zero when it completes.
constexpr int64_t kSmallMMax = 128;
size_t small_m_workspace_bytes(int64_t M, int64_t N, int r);
cudaError_t launch_small_m_fwd(const uint16_t* X, const uint8_t* codes, const uint8_t* absmax_q,
                               const float* absmax_scale, const uint16_t* A, const uint16_t* B, int64_t M,
                               int64_t K, int64_t N, int r, float scale, uint16_t* Y, float* T_save, uint16_t* Tpair,
                               void* scratch, int* status, const Nf4Params& P, cudaStream_t stream);

// Small-M forward for M <= kSmallMRdMax tokens and ranks <= 128: T = s X A,
// the weight stream (float32 partials of Y in `scratch`) and
// Y = bf16(sum of partials + T B), three launches chained by programmatic
// dependent launch.  `scratch` holds small_m_rd_workspace_bytes(M, K, N, r)
// bytes, zero before the first call; the kernels leave their counters at zero.
constexpr int64_t kSmallMRdMax = 16;
size_t small_m_rd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r);
cudaError_t launch_small_m_rd(const uint16_t* X, const uint8_t* codes, const uint8_t* absmax_q,
                              const float* absmax_scale, const uint16_t* A, const uint16_t* B, int64_t M, int64_t K,
                              int64_t N, int r, float scale, uint16_t* Y, float* T_save, void* scratch, int* status,
                              const Nf4Params& P, cudaStream_t stream);

// Copy a rows x src_cols matrix (row stride src_ld elements of elem_bytes,
// 2 or 4) into dst (row stride dst_ld), filling columns [src_cols, dst_cols)
// and rows [rows, dst_rows) with zeros (dst_rows = rows when omitted).  Used to
// pad the adapter and its gradients to a multiple of 8 ranks.
cudaError_t launch_pad_copy(const void* src, int64_t rows, int64_t src_cols, int64_t src_ld, void* dst,
                            int64_t dst_cols, int64_t dst_ld, int elem_bytes, cudaStream_t stream,
                            int64_t dst_rows = -1);

// SiLU gate of a gated MLP (glue between linears): H = silu(G) * U and its
// backward dG, dU, elementwise over n bf16 values.
cudaError_t launch_silu_gate_fwd(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n, cudaStream_t stream);
cudaError_t launch_silu_gate_bwd(const uint16_t* G, const uint16_t* U, const uint16_t* dH, uint16_t* dG,
                                 uint16_t* dU, int64_t n, cudaStream_t stream);

}  // namespace qlora
