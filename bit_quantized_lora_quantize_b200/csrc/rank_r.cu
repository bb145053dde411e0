// Rank-r products of the LoRA linear layer on sm_100a:
//   T  = s X A      [M x r]   (forward; kept for the backward)
//   U  = s dY B^T   [M x r]
//   dB = T^T dY     [r x N]   (fp32)
//   dA = X^T U      [K x r]   (fp32)
// "AI Glossary: QLoRA", second paragraph: weight gradients are formed only
// for the LoRA matrices; "LoRA: Prerequisite for Understanding QLoRA": the
// update is the product of a d x r and an r x k matrix.
//
// Each product streams one large operand (X or dY) once and is bound by HBM.
// There are few 128-row output tiles (M / 128 = 32 at 4096 tokens), so the
// reduction is split over up to eight CTAs per tile, and those CTAs form one
// thread-block cluster.  Warp 0 issues TMA (no multicast), warp 1 the
// tcgen05.mma into TMEM, warps 2-5 move the finished fp32 accumulator into
// the CTA's own shared memory.  After a cluster barrier, CTA k of the cluster
// sums rows [k*128/S, (k+1)*128/S) of all S partial tiles, reading its peers'
// shared memory (DSMEM) in rank order: a fixed summation order, so results
// are bit-reproducible, with no global partials, counters or second kernel.
//
// T and U are produced as float32 plus a bf16 pair [rows x 2rp]
// (hi = bf16(v) in columns [0, r), lo = bf16(v - hi) in [rp, rp + r)); the
// consumers (dA, dB) read the pair as their B operand and add the two halves.
#include <algorithm>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "nf4_device.cuh"
#include "ptx.cuh"
#include "tensor_map.h"

namespace qlora {

namespace {

constexpr int kTile = 128;       // output rows per tile (one M = 128 MMA)
constexpr int kDepth = 64;       // reduction depth of one stage
constexpr int kMaxSplits = 8;    // portable cluster size
constexpr int kCtaSlots = 2 * 148;  // two 96 KB CTAs on each of the 148 SMs
constexpr int kRankThreads = 192;

struct RankArgs {
  int64_t rows;      // output rows (M, M, N or K)
  int nkb;           // 64-deep reduction blocks of the whole product
  int kps;           // blocks per split
  int splits;        // cluster size
  int r, rp;
  float scale;
  int kind;          // SkinnyKind
  float* f32;        // T (may be null), dA, dB
  uint16_t* pair;    // T / U pair
  // Partial tiles of the splits, [tile][split][BN / 4][128 rows] float4, or
  // null: then each CTA keeps its partial in shared memory and the cluster
  // reads it through distributed shared memory (slower, needs no scratch).
  float4* scratch;
  int* status;
};

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}
__device__ __forceinline__ float4 ld_peer4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// Output of four adjacent columns [j, j + 4) of one row.
__device__ __forceinline__ void emit4(const RankArgs& a, int64_t row, int j, float4 v) {
  const int kind = a.kind;
  if (kind == static_cast<int>(SkinnyKind::kXA) || kind == static_cast<int>(SkinnyKind::kDyBt)) {
    float s[4] = {v.x, v.y, v.z, v.w};
    uint16_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s[e] = (j + e < a.r) ? __fmul_rn(a.scale, s[e]) : 0.0f;
      const __nv_bfloat16 h = __float2bfloat16_rn(s[e]);
      hi[e] = *reinterpret_cast<const uint16_t*>(&h);
      lo[e] = bf16_bits(__fsub_rn(s[e], __bfloat162float(h)));
    }
    if (a.f32 && j < a.r) *reinterpret_cast<float4*>(a.f32 + row * a.r + j) = make_float4(s[0], s[1], s[2], s[3]);
    uint16_t* ph = a.pair + row * 2 * a.rp + j;
    *reinterpret_cast<uint2*>(ph) = make_uint2(hi[0] | (uint32_t(hi[1]) << 16), hi[2] | (uint32_t(hi[3]) << 16));
    *reinterpret_cast<uint2*>(ph + a.rp) =
        make_uint2(lo[0] | (uint32_t(lo[1]) << 16), lo[2] | (uint32_t(lo[3]) << 16));
  } else if (kind == static_cast<int>(SkinnyKind::kXtU)) {
    if (j < a.r) *reinterpret_cast<float4*>(a.f32 + row * a.r + j) = v;
  } else {  // kTtDy: dB[j][n]
    if (j < a.r) {
      a.f32[static_cast<int64_t>(j) * a.rows + row] = v.x;
      a.f32[static_cast<int64_t>(j + 1) * a.rows + row] = v.y;
      a.f32[static_cast<int64_t>(j + 2) * a.rows + row] = v.z;
      a.f32[static_cast<int64_t>(j + 3) * a.rows + row] = v.w;
    }
  }
}

template <int BN, int STAGES>
struct RankSmem {
  static constexpr int kABytes = kTile * kDepth * 2;  // 16 KB
  static constexpr int kBBytes = BN * kDepth * 2;
  static constexpr int kPStride = BN + 4;             // floats per partial row (padding spreads banks)
  static constexpr int kStageArea = STAGES * (kABytes + kBBytes);
  static constexpr int kPartial = kTile * kPStride * 4;
  static constexpr int kArea = kStageArea > kPartial ? kStageArea : kPartial;
  static constexpr int kBar = kArea;
  static constexpr int kTotal = kBar + (2 * STAGES + 1) * 8 + 16;
  static constexpr int kDynamic = kTotal + 1024;
};

template <int BN, int STAGES, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kRankThreads, 1)
    rank_r_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const RankArgs a) {
  using L = RankSmem<BN, STAGES>;
  constexpr int kABytes = L::kABytes;
  constexpr int kBBytes = L::kBBytes;
  constexpr uint32_t kTmemCols = BN <= 32 ? 32 : BN;
  const bool consumer = a.kind == static_cast<int>(SkinnyKind::kTtDy) || a.kind == static_cast<int>(SkinnyKind::kXtU);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * kABytes;
  float* P = reinterpret_cast<float*>(smem);  // reuses the stage area once the products are done
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;  // == rank in the cluster
  const int tile = blockIdx.y;
  const int kb0 = split * a.kps;
  const int n = max(0, min(a.kps, a.nkb - kb0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;
  // The set-up above overlaps the previous kernel; the operands may be its
  // outputs, so every thread waits for it here.
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      const WaitCtx ctx{abort_flag, a.status, 11};
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, ctx)) break;
        const int kb = kb0 + i;
        uint8_t* a_dst = sA + s * kABytes;
        uint8_t* b_dst = sB + s * kBBytes;
        mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
        if (!A_MN) {
          tma_load_2d(&tmA, &full[s], a_dst, kb * kDepth, tile * kTile);
        } else {
          tma_load_2d(&tmA, &full[s], a_dst, tile * kTile, kb * kDepth);
          tma_load_2d(&tmA, &full[s], a_dst + 8192, tile * kTile + 64, kb * kDepth);
        }
        if (!B_MN) {
          tma_load_2d(&tmB, &full[s], b_dst, kb * kDepth, 0);
        } else {
#pragma unroll
          for (int q = 0; q < BN / 64; ++q) tma_load_2d(&tmB, &full[s], b_dst + q * 8192, q * 64, kb * kDepth);
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[i % STAGES], (i / STAGES) & 1) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && n > 0) {
      const WaitCtx ctx{abort_flag, a.status, 12};
      const uint32_t idesc = idesc_bf16_f32(kTile, BN, A_MN, B_MN);
      bool ok = true;
      for (int i = 0; i < n; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full[s], ph, ctx)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + s * kABytes);
        const uint32_t b_base = smem_u32(sB + s * kBBytes);
#pragma unroll
        for (int kk = 0; kk < kDepth / 16; ++kk) {
          const uint64_t ad = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(b_base + kk * 32, 16, 1024);
          umma_bf16(tmem_acc, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(acc_full);
    }
  } else {
    // warps 2-5: accumulator -> own shared memory (fp32, padded rows)
    const WaitCtx ctx{abort_flag, a.status, 13};
    const int q = warp & 3;
    const int lrow = q * 32 + lane;
    const bool ok = (n == 0) || __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, ctx));
    tc_fence_after();
    float* prow = P + lrow * L::kPStride;
    // Column group g of this row: global scratch (coalesced over rows) or
    // the padded shared-memory row.
    float4* grow = a.scratch ? a.scratch + (static_cast<int64_t>(tile) * a.splits + split) * (BN / 4) * kTile + lrow
                             : nullptr;
    auto put = [&](int g, float4 v) {
      if (grow) grow[g * kTile] = v;
      else *reinterpret_cast<float4*>(prow + 4 * g) = v;
    };
    if (n == 0 || !ok) {
      for (int g = 0; g < BN / 4; ++g) put(g, make_float4(0.f, 0.f, 0.f, 0.f));
    } else {
      const uint32_t t_row = tmem_acc + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int j0 = 0; j0 < BN; j0 += 32) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(t_row + j0, u);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 8; ++g)
          put(j0 / 4 + g, make_float4(__uint_as_float(u[4 * g]), __uint_as_float(u[4 * g + 1]),
                                      __uint_as_float(u[4 * g + 2]), __uint_as_float(u[4 * g + 3])));
      }
    }
    if (grow) __threadfence();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // every CTA's partial tile is in place (release/acquire at cluster scope)

  // Sum rows [r0, r1) of the S partial tiles in rank order.
  const int S = a.splits;
  const int R = kTile / S;
  const int r0 = split * R;
  const int c4 = a.rp / 4;  // output column groups
  const uint32_t p_local = smem_u32(P);
  const bool rows_fastest = a.kind == static_cast<int>(SkinnyKind::kTtDy);
  // All peers' loads of an item are issued before any is used, so the
  // distributed-shared-memory round trips overlap; the sums then run in rank
  // order (fixed, hence bit-reproducible).
  uint32_t peer[kMaxSplits];
#pragma unroll
  for (int k = 0; k < kMaxSplits; ++k) peer[k] = k < S ? peer_addr(p_local, k) : p_local;
  for (int t = threadIdx.x; t < R * c4; t += kRankThreads) {
    const int rr = rows_fastest ? (t % R) : (t / c4);
    const int jj = rows_fastest ? (t / R) : (t % c4);
    const int lrow = r0 + rr;
    const int64_t row = static_cast<int64_t>(tile) * kTile + lrow;
    const uint32_t off = static_cast<uint32_t>((lrow * L::kPStride + 4 * jj) * 4);
    float4 v[kMaxSplits], w[kMaxSplits];
    if (a.scratch) {
      // Partials in global memory (L2): all loads first, then the sums.
      const float4* base = a.scratch + static_cast<int64_t>(tile) * S * (BN / 4) * kTile + lrow;
#pragma unroll
      for (int k = 0; k < kMaxSplits; ++k) {
        if (k < S) {
          v[k] = __ldcg(base + (static_cast<int64_t>(k) * (BN / 4) + jj) * kTile);
          if (consumer) w[k] = __ldcg(base + (static_cast<int64_t>(k) * (BN / 4) + c4 + jj) * kTile);
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < kMaxSplits; ++k) {
        if (k < S) {
          v[k] = ld_peer4(peer[k] + off);
          if (consumer) w[k] = ld_peer4(peer[k] + off + a.rp * 4);
        }
      }
    }
    float4 acc = v[0], lo = consumer ? w[0] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 1; k < kMaxSplits; ++k) {
      if (k < S) {
        acc.x += v[k].x; acc.y += v[k].y; acc.z += v[k].z; acc.w += v[k].w;
        if (consumer) {
          lo.x += w[k].x; lo.y += w[k].y; lo.z += w[k].z; lo.w += w[k].w;
        }
      }
    }
    if (consumer) {
      acc.x += lo.x; acc.y += lo.y; acc.z += lo.z; acc.w += lo.w;
    }
    if (row < a.rows) emit4(a, row, 4 * jj, acc);
  }

  cluster_sync_all();  // peers are done reading this CTA's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, kTmemCols);
  }
}

int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Geometry {
  int64_t rows, red;
};

Geometry geometry(SkinnyKind kind, int64_t M, int64_t K, int64_t N) {
  switch (kind) {
    case SkinnyKind::kXA: return {M, K};
    case SkinnyKind::kDyBt: return {M, N};
    case SkinnyKind::kTtDy: return {N, M};
    default: return {K, M};
  }
}

template <int BN>
constexpr int rank_stages() {
  return BN >= 256 ? 3 : (96 * 1024) / (kTile * kDepth * 2 + BN * kDepth * 2);
}

template <int BN, bool A_MN, bool B_MN>
cudaError_t launch_rank_bn(const CUtensorMap& ma, const CUtensorMap& mb, const RankArgs& a, int tiles,
                           cudaStream_t stream) {
  constexpr int kStages = rank_stages<BN>();
  using L = RankSmem<BN, kStages>;
  auto kern = rank_r_kernel<BN, kStages, A_MN, B_MN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynamic);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.splits), static_cast<unsigned>(tiles), 1);
  cfg.blockDim = dim3(kRankThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kDynamic;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(a.splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, ma, mb, a);
}

template <bool A_MN, bool B_MN>
cudaError_t dispatch_rank(int bn, const CUtensorMap& ma, const CUtensorMap& mb, const RankArgs& a, int tiles,
                          cudaStream_t st) {
  switch (bn) {
    case 64: return launch_rank_bn<64, A_MN, B_MN>(ma, mb, a, tiles, st);
    case 128: return launch_rank_bn<128, A_MN, B_MN>(ma, mb, a, tiles, st);
    case 256: return launch_rank_bn<256, A_MN, B_MN>(ma, mb, a, tiles, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

SkinnyPlan plan_skinny(SkinnyKind kind, int64_t M, int64_t K, int64_t N, int r) {
  const Geometry geo = geometry(kind, M, K, N);
  const bool producer = kind == SkinnyKind::kXA || kind == SkinnyKind::kDyBt;
  SkinnyPlan p{};
  p.tiles = static_cast<int>(ceil_div64(geo.rows, kTile));
  p.nkb = static_cast<int>(ceil_div64(geo.red, kDepth));
  p.bn = producer ? lora_pad(r) : 2 * lora_pad(r);
  // Largest power-of-two cluster (<= 8) that keeps one wave and at least two
  // 64-deep blocks per split.
  int s = 1;
  while (s < kMaxSplits && static_cast<int64_t>(p.tiles) * (2 * s) <= kCtaSlots && p.nkb >= 2 * (2 * s)) s *= 2;
  p.splits = s;
  p.kps = static_cast<int>(ceil_div64(p.nkb, s));
  return p;
}

size_t skinny_scratch_bytes(SkinnyKind kind, int64_t M, int64_t K, int64_t N, int r) {
  const SkinnyPlan p = plan_skinny(kind, M, K, N, r);
  return static_cast<size_t>(p.tiles) * p.splits * kTile * p.bn * 4;
}

cudaError_t launch_skinny(SkinnyKind kind, const uint16_t* P0, const uint16_t* P1, int64_t M, int64_t K, int64_t N,
                          int r, float scale, SkinnyOut out, float* scratch, int* status, cudaStream_t stream) {
  const SkinnyPlan p = plan_skinny(kind, M, K, N, r);
  const Geometry geo = geometry(kind, M, K, N);
  const int rp = lora_pad(r);
  const int64_t pair_stride = static_cast<int64_t>(rp) * 4;
  const uint32_t bn = static_cast<uint32_t>(p.bn);
  CUtensorMap ma, mb;
  bool ok = false;
  switch (kind) {
    case SkinnyKind::kXA:  // A = X [M,K] K-major; B = A_lora [K,r] MN-major
      ok = make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P0, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P1, r, K, static_cast<int64_t>(r) * 2, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
      break;
    case SkinnyKind::kDyBt:  // A = dY [M,N] K-major; B = B_lora [r,N] K-major
      ok = make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P0, N, M, N * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P1, N, r, N * 2, 64, bn, CU_TENSOR_MAP_SWIZZLE_128B);
      break;
    case SkinnyKind::kTtDy:  // A = dY^T MN-major; B = T pair [M,2rp] MN-major
      ok = make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P0, N, M, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P1, 2 * rp, M, pair_stride, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
      break;
    default:  // kXtU: A = X^T MN-major; B = U pair [M,2rp] MN-major
      ok = make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P0, K, M, K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
           make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, P1, 2 * rp, M, pair_stride, 64, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
      break;
  }
  if (!ok) return cudaErrorInvalidValue;
  RankArgs a{};
  a.rows = geo.rows;
  a.nkb = p.nkb;
  a.kps = p.kps;
  a.splits = p.splits;
  a.r = r;
  a.rp = rp;
  a.scale = scale;
  a.kind = static_cast<int>(kind);
  a.f32 = out.f32;
  a.pair = out.pair;
  a.scratch = reinterpret_cast<float4*>(scratch);
  a.status = status;
  switch (kind) {
    case SkinnyKind::kXA: return dispatch_rank<false, true>(p.bn, ma, mb, a, p.tiles, stream);
    case SkinnyKind::kDyBt: return dispatch_rank<false, false>(p.bn, ma, mb, a, p.tiles, stream);
    default: return dispatch_rank<true, true>(p.bn, ma, mb, a, p.tiles, stream);
  }
}

// bf16 pair of a float32 [rows x r] matrix.
__global__ void split_pair_kernel(const float* __restrict__ v, int64_t rows, int r, int rp, uint16_t* __restrict__ pair) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * rp) return;
  const int64_t row = idx / rp;
  const int j = static_cast<int>(idx % rp);
  uint16_t hi = 0, lo = 0;
  if (j < r) {
    const float x = v[row * r + j];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const __nv_bfloat16 l = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(h)));
    hi = *reinterpret_cast<const uint16_t*>(&h);
    lo = *reinterpret_cast<const uint16_t*>(&l);
  }
  pair[row * 2 * rp + j] = hi;
  pair[row * 2 * rp + rp + j] = lo;
}

cudaError_t launch_split_pair(const float* v, int64_t rows, int r, uint16_t* pair, cudaStream_t stream) {
  const int rp = lora_pad(r);
  const int64_t n = rows * rp;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div64(n, 256)), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, split_pair_kernel, v, rows, r, rp, pair);
}

}  // namespace qlora
