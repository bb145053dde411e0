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
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "nf4_device.cuh"
#include "tensor_map.h"

namespace qlora {

constexpr int kBlock = 64;
constexpr int kGroup = 256;
constexpr int kGroupElems = kBlock * kGroup;  // 16384
constexpr int kThreads = 256;

// Shared tile: 256 blocks x 128 B.  Thread t reads its block's 16-byte chunk
// j at position (j + t) mod 8 of the row, which spreads the eight lanes of a
// quarter-warp over all banks (used by the dequantization kernel).
__device__ __forceinline__ uint32_t chunk_pos(int row, int j) { return row * 128 + (((j + row) & 7) << 4); }

// Quantization, persistent: each CTA walks over groups with a two-deep TMA
// pipeline.  The weight is viewed as [numel/64 rows x 64] bf16 (one absmax
// block per row); a 256-row box lands with the 128-byte swizzle, so thread t
// finds logical chunk j of its block at chunk position j ^ (t & 7) and the
// eight lanes of a quarter-warp hit eight different bank groups.  The group
// holding a partial last block (numel % 64 != 0) is staged with plain loads
// in the same layout.
constexpr int kQuantStages = 2;
// Stages | thresholds per bf16 mantissa (128 rows x 16 bf16) | fp32(k/255)
// as double (256) | barriers, warp maxima, abort flag.
constexpr int kThrOff = kQuantStages * kGroupElems * 2;
constexpr int kLvlOff = kThrOff + 128 * 16 * 2;
constexpr int kQuantSmem = kLvlOff + 256 * 8 + 128 + 1024;

// The thresholds T_j = RU_bf16(B_j * c) of a block constant c = m * 2^e
// (m in [1, 2), 128 bf16 mantissas) are RU_bf16(B_j * m) * 2^e: rounding up
// to a binary grid commutes with scaling by a power of two while every value
// stays normal.  With the biased exponent of c in [kFastExpLo, 254] every
// |T_j| (at least 2^-5 * 2^(e - 127) for the smallest boundary) is normal, so
// the threshold is the table entry of m with e - 127 added to its exponent
// field; other constants (subnormal or non-finite) take the exact product.
constexpr int kFastExpLo = 6;

// Status word of the codec kernels on this device: a quantization whose copy
// wait gave up records it here (the call has no workspace), and
// qlora_check_status reports and clears it.
__device__ int g_codec_status;

__global__ void __launch_bounds__(kThreads, 3)
    quantize_nf4_kernel(const __grid_constant__ CUtensorMap tmW, const uint16_t* __restrict__ W, int64_t numel,
                        uint8_t* __restrict__ codes, uint8_t* __restrict__ absmax_q,
                        float* __restrict__ absmax_scale, Nf4Params P, uint64_t wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* buf = smem;                                                   // 2 x 32 KB
  uint16_t* thr = reinterpret_cast<uint16_t*>(smem + kThrOff);           // [128][16] bf16
  double* lvl2 = reinterpret_cast<double*>(smem + kLvlOff);              // fp32(k/255), exact
  uint64_t* bar = reinterpret_cast<uint64_t*>(lvl2 + 256);
  float* warp_max = reinterpret_cast<float*>(bar + kQuantStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(warp_max + kThreads / 32);
  const int tid = threadIdx.x;
  const WaitCtx ctx{abort_flag, &g_codec_status, 5, wait_ns};

  const int64_t groups = (numel + kGroupElems - 1) / kGroupElems;
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t nbytes = (numel + 1) / 2;
  const bool ragged_tail = (numel % kBlock) != 0;  // last group staged with plain loads

  lvl2[tid] = static_cast<double>(level2_value(tid));
  for (int i = tid; i < 128 * 16; i += kThreads) {
    const int m = i >> 4, j = i & 15;
    const float cm = __uint_as_float(0x3F800000u | (static_cast<uint32_t>(m) << 16));  // 1 + m/128
    thr[i] = j < 15 ? static_cast<uint16_t>(threshold_pair(P.bnd[j], cm)) : static_cast<uint16_t>(0);
  }
  if (tid == 0) {
    for (int s = 0; s < kQuantStages; ++s) mbar_init(&bar[s], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  auto issue = [&](int64_t g, int stage) {
    // Thread 0 only.  A group that needs plain loads is staged by all threads
    // after the wait instead.
    if (ragged_tail && g == groups - 1) {
      mbar_arrive(&bar[stage]);
      return;
    }
    mbar_arrive_expect_tx(&bar[stage], kGroupElems * 2);
    tma_load_2d(&tmW, &bar[stage], buf + stage * kGroupElems * 2, 0, static_cast<int>(g * kGroup));
  };

  int it = 0;
  int64_t g = blockIdx.x;
  if (tid == 0 && g < groups) issue(g, 0);
  for (; g < groups; g += gridDim.x, ++it) {
    const int stage = it & 1;
    const uint32_t phase = (it >> 1) & 1;
    const int64_t gn = g + gridDim.x;
    if (tid == 0 && gn < groups) issue(gn, stage ^ 1);
    // Bounded wait: a copy that never lands ends the loop (the status word
    // records it and the codes are undefined) instead of hanging the device.
    // Both stages' copies in flight land before the CTA exits.
    if (!__syncthreads_and(mbar_wait(&bar[stage], phase, ctx))) {
      if (tid == 0) {
        mbar_drain(&bar[stage], phase);
        if (gn < groups) mbar_drain(&bar[stage ^ 1], ((it + 1) >> 1) & 1);
      }
      break;
    }
    uint8_t* tile = buf + stage * kGroupElems * 2;
    const int64_t base = g * kGroupElems;
    if (ragged_tail && g == groups - 1) {
      for (int chunk = tid; chunk < kGroupElems / 8; chunk += kThreads) {
        const int64_t e0 = base + static_cast<int64_t>(chunk) * 8;
        uint16_t h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = (e0 + e < numel) ? W[e0 + e] : static_cast<uint16_t>(0);
        const int row = chunk >> 3, c = chunk & 7;
        *reinterpret_cast<uint4*>(tile + row * 128 + ((c ^ (row & 7)) << 4)) =
            make_uint4(h[0] | (uint32_t(h[1]) << 16), h[2] | (uint32_t(h[3]) << 16), h[4] | (uint32_t(h[5]) << 16),
                       h[6] | (uint32_t(h[7]) << 16));
      }
      __syncthreads();
    }

    // This thread's block: 32 bf16 pairs in element order.
    uint32_t x[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 v = *reinterpret_cast<const uint4*>(tile + tid * 128 + ((j ^ (tid & 7)) << 4));
      x[4 * j + 0] = v.x;
      x[4 * j + 1] = v.y;
      x[4 * j + 2] = v.z;
      x[4 * j + 3] = v.w;
    }
    // Block absmax (elements beyond numel were staged as zero).
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
    __syncthreads();  // also: every thread has read `tile`
    float c1 = warp_max[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) c1 = fmaxf(c1, warp_max[w]);

    const int64_t blk = g * kGroup + tid;
    if (blk < nb) {
      // 8-bit code of c / c1: nearest fp32(k / 255), ties to the lower k.
      uint32_t code2 = 0;
      if (c1 > 0.0f) {
        const float n2 = __fdiv_rn(c, c1);
        int k0 = __float2int_rn(n2 * 255.0f);
        k0 = max(2, min(253, k0));
        double best = 4.0;
        const double n2d = static_cast<double>(n2);
#pragma unroll
        for (int d = -2; d <= 2; ++d) {
          const double dist = fabs(n2d - lvl2[k0 + d]);
          if (dist < best) {
            best = dist;
            code2 = static_cast<uint32_t>(k0 + d);
          }
        }
      }
      absmax_q[blk] = static_cast<uint8_t>(code2);
    }
    if (tid == 0) absmax_scale[g] = c1;

    // 4-bit codes of the block.
    Nf4Thresholds T;
    {
      const uint32_t cb = __float_as_uint(c > 0.0f ? c : 1.0f);  // all-zero block: every code is 7
      const uint32_t e = cb >> 23;                                // c > 0: no sign bit
      if (e >= kFastExpLo && e <= 254) {
        const uint4* row = reinterpret_cast<const uint4*>(thr + ((cb >> 16) & 0x7Fu) * 16);
        const uint4 r0 = row[0], r1 = row[1];
        const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
        // e - 127 added to the exponent field of both halves
        const uint32_t de = (e - 127u) * 0x00800080u;
#pragma unroll
        for (int j = 0; j < 15; ++j) T.t[j] = prmt(w[j >> 1], 0, (j & 1) ? 0x3232u : 0x1010u) + de;
      } else {
        T = make_thresholds(P, c);
      }
    }
    uint32_t out[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      out[j] = pack_codes8(encode_pair(T, x[4 * j]), encode_pair(T, x[4 * j + 1]), encode_pair(T, x[4 * j + 2]),
                           encode_pair(T, x[4 * j + 3]));
    const int64_t byte0 = blk * (kBlock / 2);
    if (byte0 + 32 <= nbytes) {
      uint4* dst = reinterpret_cast<uint4*>(codes + byte0);
      dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
      dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    } else {
      for (int b = 0; b < 32 && byte0 + b < nbytes; ++b)
        codes[byte0 + b] = static_cast<uint8_t>(out[b >> 2] >> (8 * (b & 3)));
    }
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
  const int64_t full_rows = numel / kBlock;
  CUtensorMap map;
  // A 2-D view needs at least one complete block; a smaller tensor is a
  // single ragged group staged with plain loads (the map is then unused).
  if (!make_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, kBlock, full_rows > 0 ? full_rows : 1, kBlock * 2,
                   kBlock, kGroup, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  static int sm_count = 0;
  if (sm_count == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sm_count <= 0)
      sm_count = 148;
  }
  cudaError_t e = cudaFuncSetAttribute(quantize_nf4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(groups, static_cast<int64_t>(sm_count) * 3);
  quantize_nf4_kernel<<<static_cast<unsigned>(grid), kThreads, kQuantSmem, stream>>>(map, W, numel, codes, absmax_q,
                                                                                      absmax_scale, P, wait_limit_ns());
  return cudaGetLastError();
}

cudaError_t codec_status_take(cudaStream_t stream, int* word) {
  *word = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(word, g_codec_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && *word != 0) {
    static const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_codec_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  }
  return e;
}

cudaError_t launch_dequantize_nf4(const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                                  int64_t numel, uint16_t* out, const Nf4Params& P, cudaStream_t stream) {
  const int64_t groups = (numel + kGroupElems - 1) / kGroupElems;
  dequantize_nf4_kernel<<<static_cast<unsigned>(groups), kThreads, 0, stream>>>(codes, absmax_q, absmax_scale,
                                                                                numel, out, P);
  return cudaGetLastError();
}

}  // namespace qlora
