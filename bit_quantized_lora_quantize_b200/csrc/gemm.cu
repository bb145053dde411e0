// Tensor-core GEMMs of the frozen-NF4 LoRA linear layer on sm_100a.
//
// "AI Glossary: QLoRA", second paragraph: each time the layer is used its
// 4-bit weights are turned back into BFloat16 for the product, and weight
// gradients are formed only for the LoRA matrices.  "QLoRA's Working
// Process": the conversion happens on the fly, without a stored
// high-precision copy.  So the two large products (forward Y and input
// gradient dX) decode the packed NF4 tile straight into the shared-memory
// operand of the tensor-core MMA; the full bf16 weight never exists in HBM.
//
// One kernel template, warp-specialised, one 128-row output tile per CTA:
//   warp 0      TMA producer (activation tiles, packed-code tiles, LoRA tiles)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 4-11  NF4 decoders (fused kernels only): one 64-weight block per
//               thread per stage, written in the 128-byte-swizzled layout the
//               MMA descriptor expects (K-major for Y, MN-major for dX)
//   warps 4-7   epilogue: tcgen05.ld from TMEM, convert, store
// The LoRA term of the fused kernels is one (or, for r > 64, a few) extra
// 64-deep reduction stage appended to the same TMEM accumulator:
//   Y  = [X | T] [W'^T ; B]      dX = [dY | U] [W' ; A^T]
#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "nf4_device.cuh"
#include "ptx.cuh"
#include "tensor_map.h"

namespace qlora {

enum BKind : int { kBTmaK = 0, kBTmaMN = 1, kBNf4K = 2, kBNf4MN = 3 };
enum EpiKind : int { kEpiBf16 = 0, kEpiPartial = 1 };

constexpr int kBM = 128;                // rows of one tcgen05.mma (cta_group::1)
constexpr int kBK = 64;
constexpr int kCodeBytes = 8192;        // 256 x 32 B (Y) or 64 x 128 B (dX)

struct GemmArgs {
  int nkb_total;    // 64-deep reduction stages of the whole product
  int kb_per_split; // stages per split (blockIdx.z); the last split may be short
  int lora_kb;      // extra LoRA stages (fused kernels)
  int rows;       // output rows (bounds for bf16 stores)
  int cols;       // output columns
  int64_t ld_out; // leading dimension of the bf16 output
  void* out;
  float* partial; // [split][rows_pad][BN] for kEpiPartial
  const uint8_t* absmax_q;
  const float* absmax_scale;
  int64_t w_rows;  // N of the packed weight [N, K]
  int64_t w_cols;  // K
  int abs_tma;     // dX: the stage's 8-bit constant codes arrive by TMA (K % 1024 == 0)
  int lora_mod;    // padded rank rp: LoRA stage lk reads the adapter at (64*lk) mod rp
  int* status;
  Nf4Params nf4;
};

template <int BM, int BN, int STAGES, int BK_KIND>
struct SmemLayout {
  static constexpr bool kDecode = (BK_KIND == kBNf4K || BK_KIND == kBNf4MN);
  static constexpr int kABytes = BM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kCBytes = kDecode ? kCodeBytes : 0;
  static constexpr int kA = 0;
  static constexpr int kB = kA + STAGES * kABytes;
  static constexpr int kC = kB + STAGES * kBBytes;
  static constexpr int kLvl2 = kC + STAGES * kCBytes;            // fp32(k/255), 256 floats
  static constexpr int kAbs = kLvl2 + (kDecode ? 1024 : 0);       // 8-bit constant codes (dX)
  static constexpr int kAbsBytes = (BK_KIND == kBNf4MN) ? 1024 : 0;
  static constexpr int kBar = kAbs + STAGES * kAbsBytes;
  static constexpr int kNumBars = 3 * STAGES + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kTotal = kAbort + 4;
  static constexpr int kDynamic = kTotal + 1024;  // alignment slack
};

template <int BN>
struct TmemCols {
  static constexpr uint32_t value = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : BN <= 256 ? 256 : 512;
};

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void sts128(uint8_t* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4*>(p) = make_uint4(a, b, c, d);
}

template <int BM, int BN, int STAGES, bool A_MN, int BK_KIND, bool B2_MN, int EPI>
__global__ void __launch_bounds__((BK_KIND == kBNf4K || BK_KIND == kBNf4MN) ? 384 : 256, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                const __grid_constant__ CUtensorMap tmAbs, const GemmArgs args) {
  using L = SmemLayout<BM, BN, STAGES, BK_KIND>;
  constexpr bool kDecode = L::kDecode;
  constexpr bool kBMN = (BK_KIND == kBTmaMN || BK_KIND == kBNf4MN);
  constexpr int kHalves = BM / kBM;  // MMAs per K step sharing one B tile
  constexpr uint32_t kAccCols = TmemCols<BN>::value;
  constexpr uint32_t kTmemCols = kAccCols * kHalves;
  constexpr int kABytes = L::kABytes;
  constexpr int kDecoderWarps = 8;
  static_assert(BM == 128 || (BM == 256 && BN == 256 && !A_MN), "256-row tiles: fused kernels only");
  static_assert(kTmemCols <= 512, "TMEM budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + L::kA;
  uint8_t* sB = smem + L::kB;
  uint8_t* sC = smem + L::kC;
  float* lvl2 = reinterpret_cast<float*>(smem + L::kLvl2);
  uint8_t* sAbs = smem + L::kAbs;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + STAGES;
  uint64_t* decoded = empty + STAGES;
  uint64_t* acc_full = decoded + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile_n = blockIdx.x;
  const int tile_m = blockIdx.y;
  const int split = blockIdx.z;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&decoded[s], kDecoderWarps);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (args.lora_kb > 0) {
      tma_prefetch_desc(&tmA2);
      tma_prefetch_desc(&tmB2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  const int kb_begin = split * args.kb_per_split;
  const int num_kb = max(0, min(args.kb_per_split, args.nkb_total - kb_begin));
  const int total = num_kb + args.lora_kb;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const WaitCtx ctx{abort_flag, args.status, 1};
      int issued = 0;
      for (int i = 0; i < total; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, ctx)) break;
        uint8_t* a_dst = sA + s * kABytes;
        uint8_t* b_dst = sB + s * L::kBBytes;
        if (i < num_kb) {
          const int kb = kb_begin + i;
          const bool abs_tma = (BK_KIND == kBNf4MN) && args.abs_tma;
          mbar_arrive_expect_tx(&full[s], kABytes + (kDecode ? kCodeBytes : L::kBBytes) + (abs_tma ? 1024 : 0));
          if (!A_MN) {
            tma_load_2d(&tmA, &full[s], a_dst, kb * kBK, tile_m * BM);
          } else {
            tma_load_2d(&tmA, &full[s], a_dst, tile_m * kBM, kb * kBK);
            tma_load_2d(&tmA, &full[s], a_dst + 8192, tile_m * kBM + 64, kb * kBK);
          }
          if (BK_KIND == kBTmaK) {
            tma_load_2d(&tmB, &full[s], b_dst, kb * kBK, tile_n * BN);
          } else if (BK_KIND == kBTmaMN) {
#pragma unroll
            for (int a = 0; a < BN / 64; ++a) tma_load_2d(&tmB, &full[s], b_dst + a * 8192, tile_n * BN + a * 64, kb * kBK);
          } else if (BK_KIND == kBNf4K) {
            // codes [N, K/2] bytes: 256 rows x 32 bytes
            tma_load_2d(&tmB, &full[s], sC + s * kCodeBytes, kb * 32, tile_n * 256);
          } else {
            // codes: 64 rows (reduction) x 128 bytes (256 outputs)
            tma_load_2d(&tmB, &full[s], sC + s * kCodeBytes, tile_n * 128, kb * kBK);
            // 8-bit constant codes of those 64 rows: a 16-byte-wide box that
            // starts at the 16-aligned block column at or before tile_n * 4
            if (abs_tma) tma_load_2d(&tmAbs, &full[s], sAbs + s * 1024, (tile_n * 4) & ~15, kb * kBK);
          }
        } else {
          // LoRA stage: [T_hi | T_lo] (or U) against the adapter, which is read
          // twice (once per half of the pair).
          const int lk = i - num_kb;
          const int lb = (lk * kBK) % args.lora_mod;
          mbar_arrive_expect_tx(&full[s], kABytes + 256 * kBK * 2);
          tma_load_2d(&tmA2, &full[s], a_dst, lk * kBK, tile_m * BM);
          if (B2_MN) {
#pragma unroll
            for (int a = 0; a < 4; ++a) tma_load_2d(&tmB2, &full[s], b_dst + a * 8192, tile_n * 256 + a * 64, lb);
          } else {
            tma_load_2d(&tmB2, &full[s], b_dst, lb, tile_n * 256);
          }
        }
        ++issued;
      }
      if (*abort_flag) {
        // Let every copy already in flight land before the CTA exits.
        for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[i % STAGES], (i / STAGES) & 1) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const WaitCtx ctx{abort_flag, args.status, 2};
      const uint32_t idesc_main = idesc_bf16_f32(kBM, BN, A_MN, kBMN);
      const uint32_t idesc_lora = idesc_bf16_f32(kBM, 256, false, B2_MN);
      bool ok = true;
      for (int i = 0; i < total && ok; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        const bool main_stage = i < num_kb;
        if (!mbar_wait(&full[s], ph, ctx)) { ok = false; break; }
        if (kDecode && main_stage && !mbar_wait(&decoded[s], ph, ctx)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + s * kABytes);
        const uint32_t b_base = smem_u32(sB + s * L::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          uint64_t adesc, bdesc;
          uint32_t idesc;
          if (main_stage) {
            adesc = A_MN ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024) : smem_desc_sw128(a_base + kk * 32, 16, 1024);
            bdesc = kBMN ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024) : smem_desc_sw128(b_base + kk * 32, 16, 1024);
            idesc = idesc_main;
          } else {
            adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
            bdesc = B2_MN ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024) : smem_desc_sw128(b_base + kk * 32, 16, 1024);
            idesc = idesc_lora;
          }
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_bf16(tmem_acc, adesc, bdesc, idesc, acc);
          if (kHalves == 2) {
            // Rows 128..255 of the A tile start 16 atoms (16 KB) further on.
            const uint64_t adesc2 = smem_desc_sw128(a_base + 16384 + kk * 32, 16, 1024);
            umma_bf16(tmem_acc + kAccCols, adesc2, bdesc, idesc, acc);
          }
        }
        umma_commit(&empty[s]);
      }
      if (ok) umma_commit(acc_full);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ decoders
    if (kDecode) {
      const WaitCtx ctx{abort_flag, args.status, 3};
      const int d = threadIdx.x - 128;  // 0..255
      const int64_t blocks_per_row = args.w_cols / 64;
      lvl2[d] = level2_value(d);
      asm volatile("bar.sync 1, 256;" ::: "memory");  // decoder warps only
      if (BK_KIND == kBNf4K) {
        // Thread d decodes weight row n = tile_n*256 + d, one 64-wide block per stage.
        const int64_t n = static_cast<int64_t>(tile_n) * 256 + d;
        const bool row_ok = n < args.w_rows;
        const uint32_t b_row = (d >> 3) * 1024;
        const int r8 = d & 7;
        int64_t blk = n * blocks_per_row + kb_begin;
        uint32_t q2 = 0;
        float c1 = 0.0f;
        if (row_ok && num_kb > 0) {
          q2 = __ldg(args.absmax_q + blk);
          c1 = __ldg(args.absmax_scale + (blk >> 8));
        }
        for (int i = 0; i < num_kb; ++i) {
          const int s = i % STAGES;
          const uint32_t ph = (i / STAGES) & 1;
          // Prefetch the next block's constants while this one decodes.
          uint32_t q2n = 0;
          float c1n = 0.0f;
          if (row_ok && i + 1 < num_kb) {
            q2n = __ldg(args.absmax_q + blk + 1);
            c1n = __ldg(args.absmax_scale + ((blk + 1) >> 8));
          }
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], ph, ctx))) break;
          uint8_t* dst = sB + s * L::kBBytes + b_row;
          if (row_ok) {
            const uint8_t* src = sC + s * kCodeBytes + d * 32;
            const uint4 v0 = lds128(src);
            const uint4 v1 = lds128(src + 16);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const Nf4Lut lut = make_lut(args.nf4, __fmul_rn(lvl2[q2], c1));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o[4];
              decode8(lut, w[c], o);
              sts128(dst + sw128_offset(r8, c), o[0], o[1], o[2], o[3]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) sts128(dst + sw128_offset(r8, c), 0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&decoded[s]);
          q2 = q2n;
          c1 = c1n;
          ++blk;
        }
      } else {
        // Thread d: reduction row nl (0..63) of the stage, output atom j (64 outputs).
        const int nl = d & 63;
        const int j = d >> 6;
        const int64_t kob = static_cast<int64_t>(tile_n) * 4 + j;  // 64-wide output block along K
        const bool col_ok = kob < blocks_per_row;
        const uint32_t b_off = j * 8192 + (nl >> 3) * 1024;
        const int r8 = nl & 7;
        const bool abs_tma = args.abs_tma != 0;
        const int abs_col = static_cast<int>(kob - ((static_cast<int64_t>(tile_n) * 4) & ~int64_t(15)));
        auto load_const = [&](int i, uint32_t& q, float& c) {
          const int64_t n = static_cast<int64_t>(kb_begin + i) * 64 + nl;
          if (col_ok && n < args.w_rows) {
            const int64_t b = n * blocks_per_row + kob;
            q = abs_tma ? 0u : __ldg(args.absmax_q + b);
            c = __ldg(args.absmax_scale + (b >> 8));
            return true;
          }
          q = 0;
          c = 0.0f;
          return false;
        };
        uint32_t q2 = 0;
        float c1 = 0.0f;
        bool ok_cur = num_kb > 0 ? load_const(0, q2, c1) : false;
        for (int i = 0; i < num_kb; ++i) {
          const int s = i % STAGES;
          const uint32_t ph = (i / STAGES) & 1;
          uint32_t q2n = 0;
          float c1n = 0.0f;
          const bool ok_next = (i + 1 < num_kb) ? load_const(i + 1, q2n, c1n) : false;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], ph, ctx))) break;
          uint8_t* dst = sB + s * L::kBBytes + b_off;
          if (ok_cur) {
            const uint8_t* row = sC + s * kCodeBytes + nl * 128;
            const uint4 v0 = lds128(row + (((2 * j) ^ r8) << 4));
            const uint4 v1 = lds128(row + (((2 * j + 1) ^ r8) << 4));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            if (abs_tma) q2 = sAbs[s * 1024 + nl * 16 + abs_col];
            const Nf4Lut lut = make_lut(args.nf4, __fmul_rn(lvl2[q2], c1));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o[4];
              decode8(lut, w[c], o);
              sts128(dst + sw128_offset(r8, c), o[0], o[1], o[2], o[3]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) sts128(dst + sw128_offset(r8, c), 0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&decoded[s]);
          q2 = q2n;
          c1 = c1n;
          ok_cur = ok_next;
        }
      }
    }
    // ------------------------------------------------------------ epilogue
    if (warp < 4 + 4 * kHalves) {
      const WaitCtx ctx{abort_flag, args.status, 4};
      const int q = warp & 3;           // TMEM lane group this warp may access
      const int h = (warp - 4) >> 2;    // accumulator half (256-row tiles)
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, ctx));
      tc_fence_after();
      if (ok) {
        const int row = tile_m * BM + h * kBM + q * 32 + lane;
        const uint32_t t_row = tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + h * kAccCols;
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + cc * 32, v);
          tmem_wait_ld();
          const int col0 = tile_n * BN + cc * 32;
          if (EPI == kEpiBf16) {
            if (row < args.rows) {
              uint16_t* out = reinterpret_cast<uint16_t*>(args.out) + static_cast<int64_t>(row) * args.ld_out;
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                const int col = col0 + g * 8;
                if (col < args.cols) {
                  uint32_t p[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    p[e] = pack_bf16x2_rn(__uint_as_float(v[g * 8 + 2 * e]), __uint_as_float(v[g * 8 + 2 * e + 1]));
                  *reinterpret_cast<uint4*>(out + col) = make_uint4(p[0], p[1], p[2], p[3]);
                }
              }
            }
          } else {
            const int64_t rows_pad = static_cast<int64_t>(gridDim.y) * BM;
            float* dst = args.partial + (static_cast<int64_t>(split) * rows_pad + row) * BN + cc * 32;
#pragma unroll
            for (int g = 0; g < 8; ++g)
              *reinterpret_cast<uint4*>(dst + g * 4) = make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, kTmemCols);
  }
}

// ----------------------------------------------------------------- host side
template <int BM, int BN, int STAGES, bool A_MN, int BK_KIND, bool B2_MN, int EPI>
static cudaError_t launch_gemm(dim3 grid, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                               const CUtensorMap& b2, const CUtensorMap& abs, const GemmArgs& args,
                               cudaStream_t stream) {
  using L = SmemLayout<BM, BN, STAGES, BK_KIND>;
  auto kern = gemm_kernel<BM, BN, STAGES, A_MN, BK_KIND, B2_MN, EPI>;
  static_assert(L::kDynamic <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynamic);
  if (e != cudaSuccess) return e;
  const int threads = L::kDecode ? 384 : 256;
  kern<<<grid, threads, L::kDynamic, stream>>>(a, b, a2, b2, abs, args);
  return cudaGetLastError();
}

constexpr int kFusedBM = 256;
constexpr int kFusedStages = 3;

cudaError_t launch_fused_fwd(const uint16_t* X, const uint8_t* codes, const uint8_t* absmax_q,
                             const float* absmax_scale, const uint16_t* Tpair, const uint16_t* B, int64_t M, int64_t K,
                             int64_t N, int r, uint16_t* Y, int* status, const Nf4Params& P, cudaStream_t stream) {
  const int rp = lora_pad(r);
  CUtensorMap mX, mC, mT, mB;
  if (!make_map_2d(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, kFusedBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 32, 256, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&mT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Tpair, 2 * rp, M, static_cast<int64_t>(rp) * 4, 64, kFusedBM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, r, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  GemmArgs args{};
  args.nkb_total = static_cast<int>(K / 64);
  args.kb_per_split = args.nkb_total;
  args.lora_kb = 2 * rp / 64;
  args.lora_mod = rp;
  args.rows = static_cast<int>(M);
  args.cols = static_cast<int>(N);
  args.ld_out = N;
  args.out = Y;
  args.absmax_q = absmax_q;
  args.absmax_scale = absmax_scale;
  args.w_rows = N;
  args.w_cols = K;
  args.status = status;
  args.nf4 = P;
  dim3 grid(static_cast<unsigned>((N + 255) / 256), static_cast<unsigned>((M + kFusedBM - 1) / kFusedBM), 1);
  return launch_gemm<kFusedBM, 256, kFusedStages, false, kBNf4K, true, kEpiBf16>(grid, mX, mC, mT, mB, mB, args,
                                                                                   stream);
}

cudaError_t launch_fused_dx(const uint16_t* dY, const uint8_t* codes, const uint8_t* absmax_q,
                            const float* absmax_scale, const uint16_t* Upair, const uint16_t* A, int64_t M, int64_t K,
                            int64_t N, int r, uint16_t* dX, int* status, const Nf4Params& P, cudaStream_t stream) {
  const int rp = lora_pad(r);
  CUtensorMap mD, mC, mU, mA;
  if (!make_map_2d(&mD, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, N, M, N * 2, 64, kFusedBM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Upair, 2 * rp, M, static_cast<int64_t>(rp) * 4, 64, kFusedBM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, r, K, static_cast<int64_t>(r) * 2, 64, 256,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // The 8-bit constant codes as a [N x K/64] byte matrix; rows must be a
  // multiple of 16 bytes for TMA, i.e. K % 1024 == 0 (otherwise plain loads).
  CUtensorMap mAbs = mA;
  const bool abs_tma = (K % 1024 == 0) &&
                       make_map_2d(&mAbs, CU_TENSOR_MAP_DATA_TYPE_UINT8, absmax_q, K / 64, N, K / 64, 16, 64,
                                   CU_TENSOR_MAP_SWIZZLE_NONE);
  GemmArgs args{};
  args.abs_tma = abs_tma ? 1 : 0;
  args.nkb_total = static_cast<int>((N + 63) / 64);
  args.kb_per_split = args.nkb_total;
  args.lora_kb = 2 * rp / 64;
  args.lora_mod = rp;
  args.rows = static_cast<int>(M);
  args.cols = static_cast<int>(K);
  args.ld_out = K;
  args.out = dX;
  args.absmax_q = absmax_q;
  args.absmax_scale = absmax_scale;
  args.w_rows = N;
  args.w_cols = K;
  args.status = status;
  args.nf4 = P;
  dim3 grid(static_cast<unsigned>((K + 255) / 256), static_cast<unsigned>((M + kFusedBM - 1) / kFusedBM), 1);
  return launch_gemm<kFusedBM, 256, kFusedStages, false, kBNf4MN, false, kEpiBf16>(grid, mD, mC, mU, mA, mAbs, args,
                                                                                    stream);
}

}  // namespace qlora
