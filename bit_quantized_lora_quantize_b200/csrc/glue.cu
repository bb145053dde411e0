// SiLU gate between the linears of a gated MLP (LLaMA's feed-forward block):
// H = silu(G) * U and its backward; and the copy that pads the adapter to a
// multiple of 8 ranks.  This is glue between LoRA linears, not a
// step of the QLoRA method; it exists so that a whole gated MLP runs on this
// library's kernels.  Elementwise and HBM-bound: 16-byte vector loads and
// stores, float32 arithmetic, one bf16 rounding per output.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace qlora {

namespace {

constexpr int kGlueThreads = 256;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float sigmoid(float x) { return 1.0f / (1.0f + expf(-x)); }

// h = silu(g) * u = g * sigmoid(g) * u
__device__ __forceinline__ float gate_fwd(float g, float u) { return g * sigmoid(g) * u; }

// dG = dH * u * sigmoid(g) * (1 + g * (1 - sigmoid(g))), dU = dH * g * sigmoid(g)
__device__ __forceinline__ void gate_bwd(float g, float u, float dh, float& dg, float& du) {
  const float sg = sigmoid(g);
  dg = dh * u * sg * (1.0f + g * (1.0f - sg));
  du = dh * g * sg;
}

__global__ void __launch_bounds__(kGlueThreads) silu_gate_fwd_kernel(const uint4* __restrict__ G,
                                                                     const uint4* __restrict__ U,
                                                                     uint4* __restrict__ H, int64_t n8,
                                                                     const uint16_t* __restrict__ Gs,
                                                                     const uint16_t* __restrict__ Us,
                                                                     uint16_t* __restrict__ Hs, int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 g = __ldcs(G + i), u = __ldcs(U + i);
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16x2_rn(gate_fwd(bf_lo(gw[e]), bf_lo(uw[e])), gate_fwd(bf_hi(gw[e]), bf_hi(uw[e])));
    __stcs(H + i, make_uint4(o[0], o[1], o[2], o[3]));
  }
  // Elements past the last full vector of 8.
  const int64_t t = n8 * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < n) {
    const float g = __uint_as_float(static_cast<uint32_t>(Gs[t]) << 16);
    const float u = __uint_as_float(static_cast<uint32_t>(Us[t]) << 16);
    Hs[t] = __bfloat16_as_ushort(__float2bfloat16_rn(gate_fwd(g, u)));
  }
}

__global__ void __launch_bounds__(kGlueThreads) silu_gate_bwd_kernel(
    const uint4* __restrict__ G, const uint4* __restrict__ U, const uint4* __restrict__ dH, uint4* __restrict__ dG,
    uint4* __restrict__ dU, int64_t n8, const uint16_t* __restrict__ Gs, const uint16_t* __restrict__ Us,
    const uint16_t* __restrict__ dHs, uint16_t* __restrict__ dGs, uint16_t* __restrict__ dUs, int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 g = __ldcs(G + i), u = __ldcs(U + i), h = __ldcs(dH + i);
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w}, hw[4] = {h.x, h.y, h.z, h.w};
    uint32_t og[4], ou[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float g0, u0, g1, u1;
      gate_bwd(bf_lo(gw[e]), bf_lo(uw[e]), bf_lo(hw[e]), g0, u0);
      gate_bwd(bf_hi(gw[e]), bf_hi(uw[e]), bf_hi(hw[e]), g1, u1);
      og[e] = pack_bf16x2_rn(g0, g1);
      ou[e] = pack_bf16x2_rn(u0, u1);
    }
    __stcs(dG + i, make_uint4(og[0], og[1], og[2], og[3]));
    __stcs(dU + i, make_uint4(ou[0], ou[1], ou[2], ou[3]));
  }
  const int64_t t = n8 * 8 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < n) {
    float dg, du;
    gate_bwd(__uint_as_float(static_cast<uint32_t>(Gs[t]) << 16), __uint_as_float(static_cast<uint32_t>(Us[t]) << 16),
             __uint_as_float(static_cast<uint32_t>(dHs[t]) << 16), dg, du);
    dGs[t] = __bfloat16_as_ushort(__float2bfloat16_rn(dg));
    dUs[t] = __bfloat16_as_ushort(__float2bfloat16_rn(du));
  }
}

int glue_grid(int64_t n8) {
  const int64_t want = (n8 + kGlueThreads - 1) / kGlueThreads;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;  // 8 resident CTAs of 256 per SM
  return static_cast<int>(std::max<int64_t>(1, std::min(want, cap)));
}

template <typename T>
__global__ void __launch_bounds__(kGlueThreads) pad_copy_kernel(const T* __restrict__ src, int64_t rows,
                                                                int64_t src_cols, int64_t src_ld, T* __restrict__ dst,
                                                                int64_t dst_cols, int64_t dst_ld, int64_t dst_rows) {
  const int64_t n = dst_rows * dst_cols;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t r = i / dst_cols, c = i - r * dst_cols;
    dst[r * dst_ld + c] = (r < rows && c < src_cols) ? src[r * src_ld + c] : T(0);
  }
}

}  // namespace

cudaError_t launch_pad_copy(const void* src, int64_t rows, int64_t src_cols, int64_t src_ld, void* dst,
                            int64_t dst_cols, int64_t dst_ld, int elem_bytes, cudaStream_t stream,
                            int64_t dst_rows) {
  if (dst_rows < 0) dst_rows = rows;
  const int grid = glue_grid((dst_rows * dst_cols + 7) / 8);
  if (elem_bytes == 2)
    pad_copy_kernel<uint16_t><<<grid, kGlueThreads, 0, stream>>>(static_cast<const uint16_t*>(src), rows, src_cols,
                                                                  src_ld, static_cast<uint16_t*>(dst), dst_cols,
                                                                  dst_ld, dst_rows);
  else
    pad_copy_kernel<uint32_t><<<grid, kGlueThreads, 0, stream>>>(static_cast<const uint32_t*>(src), rows, src_cols,
                                                                  src_ld, static_cast<uint32_t*>(dst), dst_cols,
                                                                  dst_ld, dst_rows);
  return cudaGetLastError();
}

cudaError_t launch_silu_gate_fwd(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n, cudaStream_t stream) {
  const int64_t n8 = n / 8;
  silu_gate_fwd_kernel<<<glue_grid(n8), kGlueThreads, 0, stream>>>(
      reinterpret_cast<const uint4*>(G), reinterpret_cast<const uint4*>(U), reinterpret_cast<uint4*>(H), n8, G, U, H,
      n);
  return cudaGetLastError();
}

cudaError_t launch_silu_gate_bwd(const uint16_t* G, const uint16_t* U, const uint16_t* dH, uint16_t* dG,
                                 uint16_t* dU, int64_t n, cudaStream_t stream) {
  const int64_t n8 = n / 8;
  silu_gate_bwd_kernel<<<glue_grid(n8), kGlueThreads, 0, stream>>>(
      reinterpret_cast<const uint4*>(G), reinterpret_cast<const uint4*>(U), reinterpret_cast<const uint4*>(dH),
      reinterpret_cast<uint4*>(dG), reinterpret_cast<uint4*>(dU), n8, G, U, dH, dG, dU, n);
  return cudaGetLastError();
}

}  // namespace qlora
