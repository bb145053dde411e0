// NF4 quantization (blockwise absmax + nearest level + packing + double
// quantization of the constants) and the standalone dequantization to bf16.
//
// "AI Glossary: QLoRA", second paragraph; "QLoRA: Fine-Tuning 65-Billion
// Parameter Models on a Single Consumer GPU", "1. 4-bit NormalFloat (NF4)"
// and "2. Double Quantization".  Blocks of 64 weights share one absmax; 256
// absmax constants share one float32 maximum and are stored as 8-bit codes.
//
// One CTA handles one group of 256 blocks (16384 weights, 32 KB of bf16):
// the group maximum needed by the double quantization is then a CTA
// reduction and no intermediate constant ever goes to HBM.  Loads are
// coalesced 16-byte vectors staged in shared memory; each thread then owns
// one 64-element block.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "nf4_device.cuh"

namespace qlora {

constexpr int kBlock = 64;
constexpr int kGroup = 256;
constexpr int kGroupElems = kBlock * kGroup;  // 16384
constexpr int kThreads = 256;

// Shared tile: 256 blocks x 128 B.  Thread t reads its block's 16-byte chunk
// j at position (j + t) mod 8 of the row, which spreads the eight lanes of a
// quarter-warp over all banks.
__device__ __forceinline__ uint32_t chunk_pos(int row, int j) { return row * 128 + (((j + row) & 7) << 4); }

__global__ void __launch_bounds__(kThreads) quantize_nf4_kernel(const uint16_t* __restrict__ W, int64_t numel,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint8_t* __restrict__ absmax_q,
                                                                 float* __restrict__ absmax_scale, Nf4Params P) {
  __shared__ __align__(16) uint8_t tile[kGroupElems * 2];
  __shared__ float warp_max[kThreads / 32];
  const int tid = threadIdx.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kGroupElems;
  const bool full = base + kGroupElems <= numel;

  // Coalesced load of the group: chunk i (8 elements) -> block i / 8, chunk i % 8.
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int chunk = tid + it * kThreads;
    const int64_t e0 = base + static_cast<int64_t>(chunk) * 8;
    uint4 v;
    if (full) {
      v = __ldg(reinterpret_cast<const uint4*>(W + e0));
    } else {
      uint16_t h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = (e0 + e < numel) ? W[e0 + e] : static_cast<uint16_t>(0);
      v.x = h[0] | (static_cast<uint32_t>(h[1]) << 16);
      v.y = h[2] | (static_cast<uint32_t>(h[3]) << 16);
      v.z = h[4] | (static_cast<uint32_t>(h[5]) << 16);
      v.w = h[6] | (static_cast<uint32_t>(h[7]) << 16);
    }
    *reinterpret_cast<uint4*>(tile + chunk_pos(chunk >> 3, chunk & 7)) = v;
  }
  __syncthreads();

  // This thread's block: 32 bf16 pairs.
  uint32_t x[32];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + chunk_pos(tid, j));
    x[4 * j + 0] = v.x;
    x[4 * j + 1] = v.y;
    x[4 * j + 2] = v.z;
    x[4 * j + 3] = v.w;
  }
  // Block absmax (absent tail elements were loaded as zero).
  __nv_bfloat162 mx = __floats2bfloat162_rn(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    uint32_t a = x[i] & 0x7FFF7FFFu;
    mx = __hmax2(mx, *reinterpret_cast<__nv_bfloat162*>(&a));
  }
  const float c = fmaxf(__low2float(mx), __high2float(mx));

  // Group maximum c1.
  float m = c;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((tid & 31) == 0) warp_max[tid >> 5] = m;
  __syncthreads();
  float c1 = warp_max[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) c1 = fmaxf(c1, warp_max[w]);

  const int64_t blk = static_cast<int64_t>(blockIdx.x) * kGroup + tid;
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  if (blk < nb) {
    // 8-bit code of c / c1: nearest fp32(k / 255), ties to the lower k.
    uint32_t code2 = 0;
    if (c1 > 0.0f) {
      const float n2 = __fdiv_rn(c, c1);
      int k0 = __float2int_rn(n2 * 255.0f);
      k0 = max(2, min(253, k0));
      double best = 4.0;
#pragma unroll
      for (int d = -2; d <= 2; ++d) {
        const double dist = fabs(static_cast<double>(n2) - static_cast<double>(level2_value(k0 + d)));
        if (dist < best) {
          best = dist;
          code2 = static_cast<uint32_t>(k0 + d);
        }
      }
    }
    absmax_q[blk] = static_cast<uint8_t>(code2);
  }
  if (tid == 0) absmax_scale[blockIdx.x] = c1;

  // 4-bit codes of the block.
  const Nf4Thresholds T = make_thresholds(P, c);
  uint32_t out[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    out[j] = pack_codes8(encode_pair(T, x[4 * j]), encode_pair(T, x[4 * j + 1]), encode_pair(T, x[4 * j + 2]),
                         encode_pair(T, x[4 * j + 3]));

  const int64_t byte0 = (base + static_cast<int64_t>(tid) * kBlock) / 2;
  const int64_t nbytes = (numel + 1) / 2;
  if (byte0 + 32 <= nbytes) {
    uint4* dst = reinterpret_cast<uint4*>(codes + byte0);
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  } else {
    for (int b = 0; b < 32 && byte0 + b < nbytes; ++b) codes[byte0 + b] = static_cast<uint8_t>(out[b >> 2] >> (8 * (b & 3)));
  }
}

// Dequantization: one thread per 64-element block; output staged in shared
// memory and written back with coalesced 16-byte stores.
__global__ void __launch_bounds__(kThreads) dequantize_nf4_kernel(const uint8_t* __restrict__ codes,
                                                                   const uint8_t* __restrict__ absmax_q,
                                                                   const float* __restrict__ absmax_scale,
                                                                   int64_t numel, uint16_t* __restrict__ out,
                                                                   Nf4Params P) {
  __shared__ __align__(16) uint8_t tile[kGroupElems * 2];
  const int tid = threadIdx.x;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kGroupElems;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * kGroup + tid;
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t nbytes = (numel + 1) / 2;
  const bool full = base + kGroupElems <= numel;

  if (blk < nb) {
    const float a = block_constant(absmax_q[blk], absmax_scale[blockIdx.x]);
    const Nf4Lut L = make_lut(P, a);
    const int64_t byte0 = blk * (kBlock / 2);
    uint32_t w[8];
    if (byte0 + 32 <= nbytes) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(codes + byte0));
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(codes + byte0) + 1);
      w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
      w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t v = 0x77777777u;
        for (int b = 0; b < 4; ++b) {
          const int64_t idx = byte0 + 4 * j + b;
          if (idx < nbytes) v = (v & ~(0xFFu << (8 * b))) | (static_cast<uint32_t>(codes[idx]) << (8 * b));
        }
        w[j] = v;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t o[4];
      decode8(L, w[j], o);
      *reinterpret_cast<uint4*>(tile + chunk_pos(tid, j)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int chunk = tid + it * kThreads;
    const int64_t e0 = base + static_cast<int64_t>(chunk) * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(tile + chunk_pos(chunk >> 3, chunk & 7));
    if (full) {
      *reinterpret_cast<uint4*>(out + e0) = v;
    } else {
      const uint32_t h[4] = {v.x, v.y, v.z, v.w};
      for (int e = 0; e < 8; ++e)
        if (e0 + e < numel) out[e0 + e] = static_cast<uint16_t>(h[e >> 1] >> (16 * (e & 1)));
    }
  }
}

cudaError_t launch_quantize_nf4(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* absmax_q,
                                float* absmax_scale, const Nf4Params& P, cudaStream_t stream) {
  const int64_t groups = (numel + kGroupElems - 1) / kGroupElems;
  quantize_nf4_kernel<<<static_cast<unsigned>(groups), kThreads, 0, stream>>>(W, numel, codes, absmax_q,
                                                                              absmax_scale, P);
  return cudaGetLastError();
}

cudaError_t launch_dequantize_nf4(const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                                  int64_t numel, uint16_t* out, const Nf4Params& P, cudaStream_t stream) {
  const int64_t groups = (numel + kGroupElems - 1) / kGroupElems;
  dequantize_nf4_kernel<<<static_cast<unsigned>(groups), kThreads, 0, stream>>>(codes, absmax_q, absmax_scale,
                                                                                numel, out, P);
  return cudaGetLastError();
}

}  // namespace qlora
