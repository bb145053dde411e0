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

// ---------------------------------------------------------------- mean-centred scheme
// The mean mu of a tensor's block absmaxes is exact: every absmax c_b is a
// bf16 value mant * 2^(e - 134) (e the biased exponent, at least 1; mant
// 8 bits), so per-exponent integer sums of mant are exact and independent of
// order.  One kernel accumulates them, a second rounds their mean once to
// float32 with integer arithmetic, and the quantization kernel reads it.
// The sums live in this library's device array (cleared before each use):
// centred quantizations on one device must not overlap on the GPU.
__device__ unsigned long long g_mean_bins[256];

__global__ void __launch_bounds__(256) absmax_bins_kernel(const uint16_t* __restrict__ W, int64_t numel,
                                                          unsigned long long* __restrict__ bins) {
  __shared__ unsigned long long sb[256];
  sb[threadIdx.x] = 0;
  __syncthreads();
  const int64_t nb = (numel + kBlock - 1) / kBlock;
  const int64_t full = numel / kBlock;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nb; b += stride) {
    uint32_t mx = 0;  // |x| as bf16 bits, two halves: magnitudes order like unsigned integers
    if (b < full) {
      const uint4* p = reinterpret_cast<const uint4*>(W + b * kBlock);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = __ldg(p + i);
        mx = __vmaxu2(mx, v.x & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.y & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.z & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, v.w & 0x7FFF7FFFu);
      }
    } else {
      for (int64_t i = b * kBlock; i < numel; ++i) mx = __vmaxu2(mx, static_cast<uint32_t>(W[i]) & 0x7FFFu);
    }
    const uint32_t m = max(mx & 0xFFFFu, mx >> 16);
    const uint32_t e = m >> 7, f = m & 127u;
    if (m != 0) atomicAdd(&sb[e > 0 ? e : 1], static_cast<unsigned long long>(e > 0 ? 128u + f : f));
  }
  __syncthreads();
  if (sb[threadIdx.x] != 0) atomicAdd(&bins[threadIdx.x], sb[threadIdx.x]);
}

// mu = fp32(sum / nb), round to nearest even, from the per-exponent sums
// (one thread).  The sum scaled by 2^165 is an integer of at most 12 32-bit
// limbs; long division by nb (< 2^32) and rounding at the float32 quantum.
__global__ void centred_mean_kernel(const unsigned long long* __restrict__ bins, int64_t nb, float* __restrict__ mu) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  constexpr int kLimbs = 12;
  uint32_t L[kLimbs] = {};
  for (int e = 1; e < 256; ++e) {
    const unsigned long long v = bins[e];
    if (!v) continue;
    const int sh = e - 1 + 32;  // mant * 2^(e - 134) * 2^165 = mant * 2^(e - 1 + 32)
    const int li = sh >> 5, bo = sh & 31;
    const unsigned long long lo = v << bo;
    const unsigned long long hi = bo ? (v >> (64 - bo)) : 0ull;
    const uint32_t add[3] = {static_cast<uint32_t>(lo), static_cast<uint32_t>(lo >> 32), static_cast<uint32_t>(hi)};
    unsigned long long carry = 0;
    for (int i = li; i < kLimbs; ++i) {
      const unsigned long long t = static_cast<unsigned long long>(L[i]) + (i - li < 3 ? add[i - li] : 0u) + carry;
      L[i] = static_cast<uint32_t>(t);
      carry = t >> 32;
      if (i - li >= 2 && carry == 0) break;
    }
  }
  const unsigned long long d = static_cast<unsigned long long>(nb);
  uint32_t Q[kLimbs];
  unsigned long long rem = 0;
  for (int i = kLimbs - 1; i >= 0; --i) {
    const unsigned long long cur = (rem << 32) | L[i];
    Q[i] = static_cast<uint32_t>(cur / d);
    rem = cur % d;
  }
  int h = -1;  // highest set bit of Q
  for (int i = kLimbs - 1; i >= 0 && h < 0; --i)
    if (Q[i]) h = 32 * i + 31 - __clz(Q[i]);
  if (h < 0) {  // below 2^-165: rounds to zero
    *mu = 0.0f;
    return;
  }
  const int shift = max(h - 23, 16);  // float32 quantum 2^(shift - 165), at least 2^-149
  auto bit = [&](int pos) -> uint32_t { return pos < 0 ? 0u : (Q[pos >> 5] >> (pos & 31)) & 1u; };
  uint32_t mant = 0;
  for (int i = 23; i >= 0; --i) mant = (mant << 1) | bit(shift + i);
  const uint32_t half = bit(shift - 1);
  bool sticky = rem != 0;
  for (int pos = shift - 2; pos >= 0 && !sticky; --pos) sticky = bit(pos) != 0;
  if (half && (sticky || (mant & 1u))) ++mant;
  const int ex = shift - 165;
  const float p2 = ex >= -126 ? __uint_as_float(static_cast<uint32_t>(ex + 127) << 23) : __uint_as_float(1u << (ex + 149));
  *mu = __fmul_rn(static_cast<float>(mant), p2);  // exact
}

// Nearest E4M3 code of v, ties to even, saturating; the sign of a negative
// value is kept even when it rounds to zero.
__device__ __forceinline__ uint32_t e4m3_code(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return (static_cast<uint32_t>(r) & 0xFFu) | (v < 0.0f ? 0x80u : 0u);
}

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
  const float mu = centred_mu(absmax_scale, groups, P.centred);  // written by the mean kernel

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
    const int64_t blk = g * kGroup + tid;
    const float dcen = __fsub_rn(c, mu);  // centred scheme: c_b - mu

    // Group maximum c1 (of c_b, or of |c_b - mu| over the blocks present).
    float m = P.centred ? (blk < nb ? fabsf(dcen) : 0.0f) : c;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((tid & 31) == 0) warp_max[tid >> 5] = m;
    __syncthreads();  // also: every thread has read `tile`
    float c1 = warp_max[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) c1 = fmaxf(c1, warp_max[w]);

    const float sg = __fdiv_rn(c1, 448.0f);  // centred scheme: group scale
    if (blk < nb) {
      // 8-bit code of c / c1: nearest fp32(k / 255), ties to the lower k.
      // Centred scheme: E4M3 code of (c - mu) / sg.
      uint32_t code2 = 0;
      if (P.centred) {
        if (sg > 0.0f) code2 = e4m3_code(__fdiv_rn(dcen, sg));
      } else if (c1 > 0.0f) {
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
    if (tid == 0) absmax_scale[g] = P.centred ? sg : c1;

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
    const float mu = centred_mu(absmax_scale, (nb + kGroup - 1) / kGroup, P.centred);
    const float a = block_constant(absmax_q[blk], absmax_scale[blockIdx.x], P.centred, mu);
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
  const int sm_count = device_sm_count();
  cudaError_t e = cudaFuncSetAttribute(quantize_nf4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmem);
  if (e != cudaSuccess) return e;
  if (P.centred) {
    // The exact mean of the block absmaxes first (two small kernels).
    unsigned long long* bins = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&bins), g_mean_bins);
    if (e == cudaSuccess) e = cudaMemsetAsync(bins, 0, sizeof(unsigned long long) * 256, stream);
    if (e != cudaSuccess) return e;
    const int64_t nb = (numel + kBlock - 1) / kBlock;
    const int64_t bgrid = std::min<int64_t>((nb + 255) / 256, static_cast<int64_t>(sm_count) * 8);
    absmax_bins_kernel<<<static_cast<unsigned>(std::max<int64_t>(1, bgrid)), 256, 0, stream>>>(W, numel, bins);
    centred_mean_kernel<<<1, 32, 0, stream>>>(bins, nb, absmax_scale + groups);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
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
