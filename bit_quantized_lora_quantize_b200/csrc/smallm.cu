// Small-M forward of the NF4 LoRA linear layer (M <= 128 tokens), sm_100a.
//
// "QLoRA: Fine-Tuning 65-Billion Parameter Models on a Single Consumer GPU",
// "QLoRA's Working Process" and the closing remark that 4-bit inference is
// still slow: with a handful of tokens the forward is a stream over the packed
// 4-bit weight, so this kernel is shaped to read the codes at HBM rate and to
// do the whole forward (T = s X A, the frozen product and the LoRA term) in
// one launch.
//
// Everything is computed transposed so that the 128-row side of the
// tensor-core MMA is filled by weight rows (or adapter ranks) and the tokens,
// padded with zero rows to MP = 16..128, are its N side:
//
//   T^T      = s A^T X^T                 (A^T tile from shared memory)
//   Y^T      = W' X^T + B^T T_pair^T     (W' from tensor memory, B^T from shared)
//
// Work units (each one 64-deep reduction block):
//   T unit      one 64-row block of A and of X^T;
//   weight unit one 128-row weight tile x 64 columns: TMA brings the packed
//               codes [128 x 32 B] and the X block into a shared ring (no
//               multicast); four decoder warps turn the codes into bf16 (one
//               weight row per thread, through a shared table of level pairs
//               indexed by code byte) and write them
//               straight into tensor memory with tcgen05.st -- the decoded
//               weight never passes through shared memory, whose bandwidth
//               would otherwise bound the stream; tcgen05.mma then reads A from
//               tensor memory and X from shared memory;
//   LoRA unit   one 64-column block of the T pair (hi, then lo) against the
//               matching B^T tile.
//
// Schedule of CTA c of the persistent, co-resident grid of G CTAs: its share
// of the T units first, then a contiguous range of the weight units (all
// tiles, tile by tile; the ranges are balanced over T and weight units
// together), then the LoRA units of every tile whose last weight unit it
// holds.  T partials are summed in a fixed two-level tree (groups of eight
// CTAs, then the groups) by whichever CTA arrives last at each level, which
// writes T (float32) and its bf16 hi/lo pair and raises a ready count; LoRA
// units wait for that count (bounded).  Every CTA stores its tile products as
// float32 partials (one per tile range it holds, plus the LoRA part); after a
// grid-wide barrier all threads of all CTAs sum them, tile by tile in CTA
// order, and write Y as bf16.  The order of every sum is fixed, so results do
// not depend on timing.  Counters are returned to zero by the CTA that
// finishes with them.
//
// Warp roles: 0 and 25-27 TMA producers, 1 TMEM allocation and MMA issue, 2, 3 and 24
// further MMA issuers (with few tokens an MMA is too small to cover its own
// issue time, so up to four threads issue them), 4-7 epilogue (T partials
// and tree, tile partials), 8-23 decoders (four groups of four warps taking
// the weight units round robin: enough warps to hide the latency of the
// shared-table decode); after a grid barrier all threads sum partials.
// Every wait is bounded (see ptx.cuh).
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

constexpr int kDepth = 64;
constexpr int kTileRows = 128;      // weight rows per tile (MMA M)
constexpr int kGroups = 4;          // decoder groups (weight units round robin)
constexpr int kDecWarp0 = 8;        // decoder warps 8 .. 8 + 4 kGroups - 1
constexpr int kIssuerWarp3 = kDecWarp0 + 4 * kGroups;  // the fourth MMA issuer
// One TMA issue takes its thread ~140 cycles, about as long as a weight unit
// takes to stream at the HBM rate, so the weight units' copies are issued by
// four producer threads (warp 0 and these three warps), round robin.
constexpr int kProducers = 4;
constexpr int kProducerWarp1 = kIssuerWarp3 + 1;
constexpr int kThreads = (kProducerWarp1 + kProducers - 1) * 32;
constexpr int kLoraSlots = 2;       // ring for T and LoRA units
constexpr int kPrefetch = 4;        // block constants are loaded this many own units ahead
constexpr int kMaxGrid = 256;       // workspace is sized for this many CTAs
constexpr int kTGroup = 8;          // first level of the T tree
constexpr int kMaxTGroups = kMaxGrid / kTGroup;
constexpr int kReadyCount = 4;      // one per epilogue warp of the final T reducer
constexpr int kSmemBudget = 220 * 1024;

template <int MP>
struct SmallLayout {
  static constexpr int kCodes = kTileRows * 32;        // 4 KB
  static constexpr int kX = MP * kDepth * 2;           // X block, K-major SW128
  static constexpr int kSlot = kCodes + kX;
  static constexpr int kAt = kTileRows * kDepth * 2;   // 16 KB: A^T or B^T tile, MN-major SW128
  static constexpr int kLSlot = kAt + kX;              // + X block or T-pair block
  static constexpr int kPairTab = 256 * 16 * 8;        // 32 KB: code byte -> two float32 levels, 16 copies
  static constexpr int kFixed = kLoraSlots * kLSlot + kPairTab + 1024 /*lvl2*/ + 1024 /*barriers*/;
  static constexpr int kStagesRaw = (kSmemBudget - kFixed) / kSlot;
  // Multiple of the decoder-group and producer counts: each ring slot always
  // belongs to the same decoder group and the same producer.
  static constexpr int kStages = std::min(24, kStagesRaw / kGroups * kGroups);
  static constexpr int offSlots = 0;
  static constexpr int offLora = offSlots + kStages * kSlot;
  static constexpr int offPairTab = offLora + kLoraSlots * kLSlot;
  static constexpr int offLvl2 = offPairTab + kPairTab;
  static constexpr int offBar = offLvl2 + 1024;
  // One tcgen05.mma issue takes an issuing thread ~130 cycles whatever its
  // size, so with few tokens the weight units are spread over kIssuers
  // threads (each with its own accumulator) to keep the MMA issue ahead of
  // the stream.
  static constexpr int kIssuers = MP <= 32 ? 4 : (MP == 64 ? 2 : 1);
  // Decoded-weight slots in tensor memory (32 columns each): what the
  // accumulators leave of the 512 columns, in multiples of the issuer and
  // decoder-group counts.
  static constexpr int kASlots = MP == 16 ? 12 : (MP == 128 ? 4 : 8);
  static constexpr int kAccCols = 2 * kIssuers * MP;  // two buffers x kIssuers accumulators
  // full/consumed per stage, lfull/lempty per LoRA slot, afull per A slot, accfull/accempty x2,
  // one MMA drain per issuer
  static constexpr int kNumBars = 2 * kStages + 2 * kLoraSlots + kASlots + 4 + 4;
  static constexpr int offSlot = offBar + kNumBars * 8;
  static constexpr int offAbort = offSlot + 4;
  static constexpr int kTotal = offAbort + 4;
  static constexpr int kDynamic = kTotal + 1024;
  // A decoder reuses A slot j % kASlots once unit j - kASlots is consumed;
  // with kStages >= kASlots that unit's ring barrier is still on its phase.
  static_assert(kStages >= kASlots, "pipeline depth");
  // A decoder announces unit j only after decoding its next unit j + kGroups
  // (hiding the store's latency) when ring and A slots leave room for that
  // unit while j is still unconsumed; otherwise it announces at once.
  static constexpr bool kDefer = false;
  static_assert(kStages >= kGroups && kASlots >= kGroups, "one unit in flight per decoder group");
  static_assert(kStages % kGroups == 0 && kASlots % kGroups == 0, "decoder groups own fixed slots");
  static_assert(kStages % kProducers == 0, "producers own fixed slots");
  static_assert(kASlots % kIssuers == 0, "an A slot is always consumed by the same issuer");
  static_assert(kAccCols + kASlots * 32 <= 512, "tensor memory budget");
};

struct SmallMArgs {
  int M, N, r, rp;
  int KB;          // 64-deep reduction blocks (K / 64)
  int L;           // LoRA units per tile (2 rp / 64)
  int tiles;       // 128-row weight tiles
  int64_t W;       // all units: KB T units + tiles * KB weight units
  int grid;        // G
  int nT;          // CTAs that take T units
  float scale;
  uint16_t* Y;
  float* T_save;
  uint16_t* Tpair;
  const uint8_t* absmax_q;
  const float* absmax_scale;
  int G4;          // groups of four tokens (partials hold 4 * G4 >= M values per row)
  int* tile_first; // per tile: CTA holding its first weight unit
  int* tile_last;  // per tile: CTA holding its last weight unit
  int* t_cnt1;     // 4 per group of the T tree
  int* t_cnt2;     // 4
  int* t_ready;    // 1
  int* bar_count;  // grid barrier: arrivals
  int* bar_gen;    // grid barrier: generation (only ever increases)
  // Partial slots of [G4][128][4] float32 (row-major in groups of four tokens):
  float* t_part;   // nT slots (T^T partials, rows = rank index)
  float* t_l1;     // ceil(nT / 8) slots
  float* partial;  // kMaxGrid + 2 * tiles slots: (c + t) weight range, kMaxGrid + tiles + t LoRA
  int* status;
  uint64_t wait_ns;  // limit of every bounded wait
  Nf4Params nf4;
};

// Schedule arithmetic (identical on host and device).
__host__ __device__ __forceinline__ int64_t t_cum(int c, const SmallMArgs& a) {
  const int cc = c < a.nT ? c : a.nT;
  return static_cast<int64_t>(cc) * a.KB / a.nT;
}
__host__ __device__ __forceinline__ int64_t pos_start(int c, const SmallMArgs& a) {
  return static_cast<int64_t>(c) * a.W / a.grid;
}
// Bounded wait until the T pair is complete.
__device__ __forceinline__ bool wait_t_ready(const SmallMArgs& a, const WaitCtx& ctx) {
  if (ld_acquire(a.t_ready) >= kReadyCount) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire(a.t_ready) >= kReadyCount) return true;
    if (*ctx.abort_flag) return false;
    if (globaltimer_ns() - t0 > ctx.limit_ns) return wait_gave_up(ctx);
  }
}

__device__ __forceinline__ uint16_t bf16_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// Row `row` of group g of a partial slot.
__device__ __forceinline__ float4* slot4(float* base, int64_t slot, int g, int row, const SmallMArgs& a) {
  return reinterpret_cast<float4*>(base) + (slot * a.G4 + g) * kTileRows + row;
}

// Grid-wide barrier of the co-resident grid (one thread per CTA).  The last
// CTA to arrive also returns the T ready count to zero: every CTA is past its
// last look at it.  Bounded; false when it gave up.
__device__ bool grid_barrier(const SmallMArgs& a, const WaitCtx& ctx) {
  const int g0 = ld_acquire(a.bar_gen);
  __threadfence();
  if (atomicAdd(a.bar_count, 1) == a.grid - 1) {
    *a.bar_count = 0;
    *a.t_ready = 0;
    __threadfence();
    st_release(a.bar_gen, g0 + 1);
    return true;
  }
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire(a.bar_gen) == g0) {
    __nanosleep(100);
    if (globaltimer_ns() - t0 > ctx.limit_ns) return wait_gave_up(ctx);
  }
  return true;
}

template <int MP>
__global__ void __launch_bounds__(kThreads, 1)
    smallm_fwd_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmT, const SmallMArgs args) {
  using L = SmallLayout<MP>;
  constexpr int S = L::kStages;
  constexpr uint32_t kTmemCols = 512;
  constexpr int I = L::kIssuers;
  constexpr uint32_t kAcol0 = L::kAccCols;  // first decoded-weight column

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sSlots = smem + L::offSlots;
  uint8_t* sLora = smem + L::offLora;
  float* lvl2 = reinterpret_cast<float*>(smem + L::offLvl2);
  float2* pair_tab = reinterpret_cast<float2*>(smem + L::offPairTab);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::offBar);
  uint64_t* consumed = full + S;  // weight unit j done: frees ring slot j % S and A slot j % L::kASlots
  uint64_t* lfull = consumed + S;
  uint64_t* lempty = lfull + kLoraSlots;
  uint64_t* afull = lempty + kLoraSlots;
  uint64_t* accfull = afull + L::kASlots;
  uint64_t* accempty = accfull + 2;
  uint64_t* mma_drain = accempty + 2;  // an issuer's MMAs ended (abort)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::offSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int KB = args.KB;
  // This CTA's schedule: T units [tk0, tk1), weight units [mx0, mx1), LoRA
  // units of tiles [lt0, lt1).
  const int64_t tk0 = t_cum(c, args), tk1 = t_cum(c + 1, args);
  const int64_t mx0 = pos_start(c, args) - tk0, mx1 = pos_start(c + 1, args) - tk1;
  const int lt0 = static_cast<int>((mx0 + KB) / KB) - 1;
  const int lt1 = static_cast<int>(mx1 / KB);
  const bool has_t = tk1 > tk0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&consumed[s], 1);
    }
    for (int s = 0; s < kLoraSlots; ++s) {
      mbar_init(&lfull[s], 1);
      mbar_init(&lempty[s], 1);
    }
    for (int s = 0; s < L::kASlots; ++s) mbar_init(&afull[s], 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], I);
      mbar_init(&accempty[b], 4);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&mma_drain[i], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x < 256) lvl2[threadIdx.x] = level2_value_for(threadIdx.x, args.nf4.centred);
  for (int i = threadIdx.x; i < 256 * 16; i += kThreads) {
    const int b = i >> 4;  // code byte: high nibble = first element
    pair_tab[i] = make_float2(args.nf4.q[b >> 4], args.nf4.q[b & 15]);
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmC);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmT);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp >= kProducerWarp1) {
    // ------------------------------------------------------------ producers
    // Producer p issues the copies of weight units jm = p (mod kProducers);
    // producer 0 also issues every T and LoRA unit.
    const int p = warp == 0 ? 0 : warp - kProducerWarp1 + 1;
    if (lane == 0) {
      const WaitCtx ctx{abort_flag, args.status, 41, args.wait_ns};
      int jm = 0, jl = 0;
      bool ok = true;
      auto lora_slot = [&](uint8_t*& dst) -> uint64_t* {
        const int ls = jl % kLoraSlots;
        if (!mbar_wait(&lempty[ls], ((jl / kLoraSlots) & 1) ^ 1, ctx)) return nullptr;
        dst = sLora + ls * L::kLSlot;
        mbar_arrive_expect_tx(&lfull[ls], L::kLSlot);
        ++jl;
        return &lfull[ls];
      };
      for (int64_t k = tk0; k < tk1 && ok && p == 0; ++k) {
        uint8_t* dst;
        uint64_t* bar = lora_slot(dst);
        if (!bar) { ok = false; break; }
        const int y = static_cast<int>(k) * kDepth;
        tma_load_2d(&tmA, bar, dst, 0, y);
        tma_load_2d(&tmA, bar, dst + 8192, 64, y);
        tma_load_2d(&tmX, bar, dst + L::kAt, y, 0);
      }
      int t = static_cast<int>(mx0 / KB), kb = static_cast<int>(mx0 % KB);
      for (int64_t x = mx0; x < mx1 && ok; ++x, ++jm) {
        if (jm % kProducers == p) {
          const int s = jm % S;
          if (!mbar_wait(&consumed[s], ((jm / S) & 1) ^ 1, ctx)) { ok = false; break; }
          uint8_t* dst = sSlots + s * L::kSlot;
          mbar_arrive_expect_tx(&full[s], L::kSlot);
          tma_load_2d(&tmC, &full[s], dst, kb * 32, t * kTileRows);
          tma_load_2d(&tmX, &full[s], dst + L::kCodes, kb * kDepth, 0);
        }
        if (++kb == KB) {
          kb = 0;
          ++t;
        }
      }
      if (ok && lt0 < lt1 && p == 0) {
        // The T pair is written by another CTA with ordinary stores and read
        // here by TMA: acquire the ready count, then order the async proxy.
        ok = wait_t_ready(args, ctx);
        fence_proxy_async_global();
      }
      for (int tt = lt0; tt < lt1 && ok && p == 0; ++tt) {
        for (int lk = 0; lk < args.L; ++lk) {
          uint8_t* dst;
          uint64_t* bar = lora_slot(dst);
          if (!bar) { ok = false; break; }
          const int jb = (lk * kDepth) % args.rp;
          tma_load_2d(&tmB, bar, dst, tt * kTileRows, jb);
          tma_load_2d(&tmB, bar, dst + 8192, tt * kTileRows + 64, jb);
          tma_load_2d(&tmT, bar, dst + L::kAt, lk * kDepth, 0);
        }
      }
      if (*abort_flag) {
        // Let the copies this thread issued land before the CTA exits.
        for (int i = (jm > S ? jm - S : 0); i < jm; ++i)
          if (i % kProducers == p) mbar_drain(&full[i % S], (i / S) & 1);
        for (int i = (jl > kLoraSlots ? jl - kLoraSlots : 0); i < jl; ++i)
          mbar_drain(&lfull[i % kLoraSlots], (i / kLoraSlots) & 1);
      }
    }
  } else if (((warp >= 1 && warp <= 3) || warp == kIssuerWarp3) && (warp == kIssuerWarp3 ? 3 : warp - 1) < I) {
    // ------------------------------------------------------------ MMA issue
    // Issuer i (warps 1, 2, 3, 24) takes the weight units jm = i (mod I) into
    // accumulator i of each segment; issuer 0 also takes every T and LoRA
    // unit.  All issuers commit to accfull at each segment's end.
    const int iss = warp == kIssuerWarp3 ? 3 : warp - 1;
    if (lane == 0) {
      const WaitCtx ctx{abort_flag, args.status, 42, args.wait_ns};
      const uint32_t idesc_main = idesc_bf16_f32(kTileRows, MP, false, false);
      const uint32_t idesc_smem = idesc_bf16_f32(kTileRows, MP, true, false);  // A^T / B^T tile, MN-major
      int jm = 0, jl = 0, seg = 0;
      bool ok = true;
      auto begin_seg = [&]() -> uint32_t {
        const int b = seg & 1;
        if (!mbar_wait(&accempty[b], ((seg >> 1) & 1) ^ 1, ctx)) {
          ok = false;
          return 0;
        }
        tc_fence_after();
        return tmem + (b * I + iss) * MP;
      };
      auto end_seg = [&]() {
        if (ok) umma_commit(&accfull[seg & 1]);
        ++seg;
      };
      auto smem_unit = [&](uint32_t d, bool first) {
        const int ls = jl % kLoraSlots;
        if (!mbar_wait(&lfull[ls], (jl / kLoraSlots) & 1, ctx)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t at = smem_u32(sLora + ls * L::kLSlot);
        const uint32_t bt = at + L::kAt;
#pragma unroll
        for (int kk = 0; kk < kDepth / 16; ++kk)
          umma_bf16(d, smem_desc_sw128(at + kk * 2048, 8192, 1024), smem_desc_sw128(bt + kk * 32, 16, 1024),
                    idesc_smem, (first && kk == 0) ? 0u : 1u);
        umma_commit(&lempty[ls]);
        ++jl;
      };
      if (has_t) {
        const uint32_t d = begin_seg();
        if (iss == 0)
          for (int64_t k = tk0; k < tk1 && ok; ++k) smem_unit(d, k == tk0);
        end_seg();
      }
      // Shared-memory descriptors of the X blocks, advanced by 16-byte units.
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(sSlots + L::kCodes), 16, 1024);
      int kb = static_cast<int>(mx0 % KB);
      for (int64_t x = mx0; x < mx1 && ok;) {
        const uint32_t d = begin_seg();
        bool first = true;
        while (x < mx1 && ok) {
          if (jm % I == iss) {
            const int s = jm % S;
            const int a = jm % L::kASlots;
            // Decoded first: its decoders saw this unit's copy land, so the
            // ring barrier cannot still show the phase of an older unit.
            if (!mbar_wait(&afull[a], (jm / L::kASlots) & 1, ctx) || !mbar_wait(&full[s], (jm / S) & 1, ctx)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t xd = xdesc0 + static_cast<uint64_t>((s * L::kSlot) >> 4);
            const uint32_t at = tmem + kAcol0 + a * 32;
#pragma unroll
            for (int kk = 0; kk < kDepth / 16; ++kk)
              umma_bf16_tmem_a(d, at + kk * 8, xd + kk * 2, idesc_main, (first && kk == 0) ? 0u : 1u);
            umma_commit(&consumed[s]);
            first = false;
          }
          ++jm;
          ++x;
          if (++kb == KB) {
            kb = 0;
            break;  // tile boundary: end of segment
          }
        }
        end_seg();
      }
      for (int tt = lt0; tt < lt1 && ok; ++tt) {
        const uint32_t d = begin_seg();
        if (iss == 0)
          for (int lk = 0; lk < args.L && ok; ++lk) smem_unit(d, lk == 0);
        end_seg();
      }
      if (!ok) {
        // Aborted: the MMAs this thread issued end before TMEM is freed.
        umma_commit(&mma_drain[iss]);
        mbar_drain(&mma_drain[iss], 0);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const WaitCtx ctx{abort_flag, args.status, 43, args.wait_ns};
    const int q = warp & 3;
    const int row = q * 32 + lane;  // accumulator lane: weight row of the tile, or rank index j
    const int G4 = args.G4;
    int seg = 0;
    // Drain accumulator buffer `seg` into partial slot `slot` of `base`,
    // summing the accumulators of the issuers in `present` (bit i: issuer i
    // took a unit of this segment) in issuer order; false when the wait gave
    // up.
    auto drain = [&](float* base, int64_t slot, uint32_t present) -> bool {
      const int b = seg & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&accfull[b], (seg >> 1) & 1, ctx))) return false;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * I * MP;
#pragma unroll 1
      for (int cc = 0; cc < MP; cc += 16) {
        float f[16];
        bool have = false;
#pragma unroll
        for (int i = 0; i < I; ++i) {
          if (!((present >> i) & 1)) continue;
          uint32_t v[16];
          tmem_ld_32x32b_x16(taddr + i * MP + cc, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) f[e] = have ? f[e] + __uint_as_float(v[e]) : __uint_as_float(v[e]);
          have = true;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int g = cc / 4 + e;
          if (g < G4) *slot4(base, slot, g, row, args) = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[b]);
      ++seg;
      return true;
    };
    // Count this warp's part of a partial sum; true for the last of `n`.
    auto arrive_last = [&](int* cnt, int n) -> bool {
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        last = atomicAdd(cnt, 1) == n - 1;
        if (last) *cnt = 0;
      }
      last = __shfl_sync(0xFFFFFFFFu, last, 0);
      if (last) __threadfence();
      return last != 0;
    };
    const int M = args.M;
    bool ok = true;
    if (has_t) {
      // T partial of this CTA, then the two-level tree (rows = rank index).
      const int r = args.r;
      ok = drain(args.t_part, c, 1u);
      const int g1 = c / kTGroup;
      const int gsize = min(kTGroup, args.nT - g1 * kTGroup);
      const int nG1 = (args.nT + kTGroup - 1) / kTGroup;
      if (ok && arrive_last(args.t_cnt1 + 4 * g1 + q, gsize)) {
        if (row < r) {
#pragma unroll 2
          for (int g = 0; g < G4; ++g) {
            float4 v[kTGroup];
#pragma unroll
            for (int k = 0; k < kTGroup; ++k)
              v[k] = k < gsize ? __ldcg(slot4(args.t_part, g1 * kTGroup + k, g, row, args)) : make_float4(0, 0, 0, 0);
            float4 s4 = v[0];
#pragma unroll
            for (int k = 1; k < kTGroup; ++k)
              if (k < gsize) s4 = add4(s4, v[k]);
            *slot4(args.t_l1, g1, g, row, args) = s4;
          }
        }
        if (arrive_last(args.t_cnt2 + q, nG1)) {
          const int rp = args.rp;
          if (row < rp) {
            for (int g = 0; g < G4; ++g) {
              float4 s4 = make_float4(0, 0, 0, 0);
              if (row < r) {
                s4 = __ldcg(slot4(args.t_l1, 0, g, row, args));
                for (int k = 1; k < nG1; ++k) s4 = add4(s4, __ldcg(slot4(args.t_l1, k, g, row, args)));
              }
              const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int m = 4 * g + e;
                if (m >= M) break;
                const float v = row < r ? __fmul_rn(args.scale, sv[e]) : 0.0f;
                if (row < r) args.T_save[static_cast<int64_t>(m) * r + row] = v;
                const __nv_bfloat16 h = __float2bfloat16_rn(v);
                uint16_t* pr = args.Tpair + static_cast<int64_t>(m) * 2 * rp + row;
                pr[0] = __bfloat16_as_ushort(h);
                pr[rp] = bf16_bits(__fsub_rn(v, __bfloat162float(h)));
              }
            }
          }
          fence_proxy_async_global();
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(args.t_ready, 1);
        }
      }
    }
    for (int64_t x = mx0; x < mx1 && ok;) {
      const int t = static_cast<int>(x / KB);
      const int64_t tile_end = static_cast<int64_t>(t + 1) * KB;
      if (threadIdx.x == 128 && x == static_cast<int64_t>(t) * KB) args.tile_first[t] = c;
      if (threadIdx.x == 128 && mx1 >= tile_end) args.tile_last[t] = c;
      const int64_t xe = mx1 < tile_end ? mx1 : tile_end;
      // Issuers that took a unit: jm = x - mx0 onwards, round robin.
      uint32_t present = 0;
      for (int64_t j = x - mx0; j < xe - mx0 && j < x - mx0 + I; ++j) present |= 1u << (j % I);
      x = xe;
      ok = drain(args.partial, c + t, present);
    }
    for (int t = lt0; t < lt1 && ok; ++t) ok = drain(args.partial, kMaxGrid + args.tiles + t, 1u);
  } else if (warp >= kDecWarp0 && warp < kIssuerWarp3) {
    // ------------------------------------------------------------ decoders
    // Group grp takes the weight units mx0 + grp, mx0 + grp + kGroups, ...; the
    // block constants of a unit are loaded kPrefetch own units ahead into a
    // register queue (the loop is unrolled so the queue stays in registers).
    // Unit positions advance by increments: no division in the loop.
    const WaitCtx ctx{abort_flag, args.status, 44, args.wait_ns};
    const int grp = (warp - kDecWarp0) >> 2;
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int sw = (nl >> 2) & 1;  // 32-byte swizzle of the codes tile
    const float2* tab_lane = pair_tab + (lane & 15);
    const int64_t units = mx1 - mx0;
    struct Cursor {
      int64_t j;  // own unit index within the range
      int t, kb;
    };
    auto cursor_at = [&](int64_t j) {
      const int64_t x = mx0 + j;
      return Cursor{j, static_cast<int>(x / KB), static_cast<int>(x % KB)};
    };
    auto advance = [&](Cursor& cu) {
      cu.j += kGroups;
      cu.kb += kGroups;
      while (cu.kb >= KB) {
        cu.kb -= KB;
        ++cu.t;
      }
    };
    auto fetch = [&](const Cursor& cu, uint32_t& q2, float& c1) {
      q2 = 0;
      c1 = 0.0f;
      const int n = cu.t * kTileRows + nl;
      if (cu.j < units && n < args.N) {
        const int64_t blk = static_cast<int64_t>(n) * KB + cu.kb;
        q2 = __ldg(args.absmax_q + blk);
        c1 = __ldg(args.absmax_scale + (blk >> 8));
      }
    };
    const float mu = centred_mu(args.absmax_scale, (static_cast<int64_t>(args.N) * KB + 255) / 256, args.nf4.centred);
    Cursor cur = cursor_at(grp);
    Cursor pre = cur;
    uint32_t pq[kPrefetch];
    float pc[kPrefetch];
#pragma unroll
    for (int i = 0; i < kPrefetch; ++i) {
      fetch(pre, pq[i], pc[i]);
      advance(pre);
    }
    bool run = cur.j < units;
    int pending = -1;  // A slot stored but not yet announced to the MMA
    while (run) {
#pragma unroll
      for (int i = 0; i < kPrefetch; ++i) {
        if (!run) continue;
        const int jm = static_cast<int>(cur.j);
        // 0 for rows past N (mu for the centred scheme: those rows are never stored)
        const float amax = __fadd_rn(__fmul_rn(lvl2[pq[i]], pc[i]), mu);
        fetch(pre, pq[i], pc[i]);
        advance(pre);
        const int s = jm % S;
        const int a = jm % L::kASlots;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], static_cast<uint32_t>(jm / S) & 1, ctx))) {
          run = false;
          continue;
        }
        const uint8_t* src = sSlots + s * L::kSlot + nl * 32;
        const uint4 v0 = *reinterpret_cast<const uint4*>(src + ((0 ^ sw) << 4));
        const uint4 v1 = *reinterpret_cast<const uint4*>(src + ((1 ^ sw) << 4));
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        // Decode through the shared pair table: each code byte gives two
        // float32 levels, scaled and rounded exactly as w' = bf16(fp32(q a)).
        // Lanes l and l + 16 share copy l % 16, whose 8-byte entries sit in
        // banks 2l and 2l + 1 only, so a warp's loads never conflict.
        auto decode_half = [&](int h, uint32_t (&o)[16]) {
#pragma unroll
          for (int cw = 0; cw < 4; ++cw) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t byte = __byte_perm(w[4 * h + cw], 0, 0x4440 + j);
              const float2 qq = tab_lane[byte * 16];
              o[4 * cw + j] = pack_bf16x2_rn(__fmul_rn(qq.x, amax), __fmul_rn(qq.y, amax));
            }
          }
        };
        uint32_t o0[16];
        decode_half(0, o0);
        // The previous unit's store has had this unit's decode to land.
        if (pending >= 0) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[pending]);
          pending = -1;
        }
        // A slot a was last used by unit jm - L::kASlots.
        if (jm >= L::kASlots &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(&consumed[(jm - L::kASlots) % S],
                                               static_cast<uint32_t>((jm - L::kASlots) / S) & 1, ctx))) {
          run = false;
          continue;
        }
        tc_fence_after();
        const uint32_t ta = tmem + lane_base + kAcol0 + a * 32;
        tmem_st_32x32b_x16(ta, o0);
        {
          uint32_t o1[16];
          decode_half(1, o1);
          tmem_st_32x32b_x16(ta + 16, o1);
        }
        pending = a;
        if (!L::kDefer) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afull[a]);
          pending = -1;
        }
        advance(cur);
        run = cur.j < units;
      }
    }
    tmem_wait_st();
    if (pending >= 0 && !*abort_flag) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[pending]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }

  // ---------------------------------------------------------------- final sums
  // After the grid barrier every partial is in place; each team of 128
  // threads sums (tile, token group) items: the tile's weight ranges in CTA
  // order, then its LoRA part.
  if (threadIdx.x == 0) {
    const WaitCtx ctx{abort_flag, args.status, 45, args.wait_ns};
    const bool ok = !*abort_flag && grid_barrier(args, ctx);
    *abort_flag = ok ? 0 : 1;
  }
  __syncthreads();
  if (*abort_flag) return;
  constexpr int kTeams = 4;  // teams of 128 threads per CTA for the final sums
  if (threadIdx.x < kTeams * kTileRows) {
    const int row = threadIdx.x & (kTileRows - 1);
    const int teams = args.grid * kTeams;
    const int64_t items = static_cast<int64_t>(args.tiles) * args.G4;
    for (int64_t it = static_cast<int64_t>(c) * kTeams + (threadIdx.x / kTileRows); it < items; it += teams) {
      const int t = static_cast<int>(it / args.G4);
      const int g = static_cast<int>(it % args.G4);
      const int n = t * kTileRows + row;
      const int cf = __ldcg(args.tile_first + t), cl = __ldcg(args.tile_last + t);
      float4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        v[k] = cf + k <= cl ? __ldcg(slot4(args.partial, cf + k + t, g, row, args)) : make_float4(0, 0, 0, 0);
      const float4 lora = __ldcg(slot4(args.partial, kMaxGrid + args.tiles + t, g, row, args));
      float4 acc = v[0];
#pragma unroll
      for (int k = 1; k < 4; ++k)
        if (cf + k <= cl) acc = add4(acc, v[k]);
      for (int cs = cf + 4; cs <= cl; ++cs) acc = add4(acc, __ldcg(slot4(args.partial, cs + t, g, row, args)));
      acc = add4(acc, lora);
      if (n < args.N) {
        const float av[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int m = 4 * g + e;
          if (m < args.M) args.Y[static_cast<int64_t>(m) * args.N + n] = bf16_bits(av[e]);
        }
      }
    }
  }
}

template <int MP>
cudaError_t launch_mp(const CUtensorMap& c, const CUtensorMap& x, const CUtensorMap& a, const CUtensorMap& b,
                      const CUtensorMap& t, const SmallMArgs& args, cudaStream_t stream) {
  using L = SmallLayout<MP>;
  static_assert(L::kDynamic <= 232448, "shared memory budget");
  auto kern = smallm_fwd_kernel<MP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynamic);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(args.grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kDynamic;
  cfg.stream = stream;
  // CTAs wait for the T pair that other CTAs of the grid produce: the
  // cooperative launch guarantees that all of them are resident.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, c, x, a, b, t, args);
}

int small_m_pad(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

struct WsParts {
  size_t cnt, t_part, t_l1, partial, total;
};

WsParts ws_parts(int64_t M, int64_t N) {
  const int64_t tiles = (N + kTileRows - 1) / kTileRows;
  const size_t slot = static_cast<size_t>((M + 3) / 4) * 4 * kTileRows * 4;  // bytes per partial slot
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  WsParts p{};
  const size_t n_cnt = static_cast<size_t>(2 * tiles + 4 * kMaxTGroups + 4 + 3);
  p.cnt = 0;
  p.t_part = up(n_cnt * 4);
  p.t_l1 = p.t_part + static_cast<size_t>(kMaxGrid) * slot;
  p.partial = p.t_l1 + static_cast<size_t>(kMaxTGroups) * slot;
  p.total = p.partial + static_cast<size_t>(kMaxGrid + 2 * tiles) * slot;
  return p;
}

}  // namespace

size_t small_m_workspace_bytes(int64_t M, int64_t N, int r) {
  (void)r;
  return ws_parts(M, N).total;
}

cudaError_t launch_small_m_fwd(const uint16_t* X, const uint8_t* codes, const uint8_t* absmax_q,
                               const float* absmax_scale, const uint16_t* A, const uint16_t* B, int64_t M, int64_t K,
                               int64_t N, int r, float scale, uint16_t* Y, float* T_save, uint16_t* Tpair,
                               void* scratch, int* status, const Nf4Params& P, cudaStream_t stream) {
  if (M > kSmallMMax) return cudaErrorInvalidValue;
  const int rp = lora_pad(r);
  const int MP = small_m_pad(M);
  CUtensorMap mC, mX, mA, mB, mT;
  if (!make_map_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 32, kTileRows,
                   CU_TENSOR_MAP_SWIZZLE_32B) ||
      !make_map_2d(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, MP, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, r, K, static_cast<int64_t>(r) * 2, 64, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, r, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Tpair, 2 * rp, M, static_cast<int64_t>(rp) * 4, 64, MP,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  SmallMArgs a{};
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.r = r;
  a.rp = rp;
  a.KB = static_cast<int>(K / 64);
  a.L = 2 * rp / 64;
  a.tiles = static_cast<int>((N + kTileRows - 1) / kTileRows);
  a.W = static_cast<int64_t>(a.KB) * (a.tiles + 1);
  a.grid = static_cast<int>(std::min<int64_t>({static_cast<int64_t>(device_sm_count()), static_cast<int64_t>(kMaxGrid),
                                               std::max<int64_t>(1, a.W / 8)}));
  a.nT = std::min(a.grid, std::max(1, (a.KB + 1) / 2));
  // Every CTA's range must cover its T units; otherwise run on one CTA.
  for (int cc = 0; cc < a.grid; ++cc) {
    if (pos_start(cc + 1, a) - pos_start(cc, a) < t_cum(cc + 1, a) - t_cum(cc, a)) {
      a.grid = 1;
      a.nT = 1;
      break;
    }
  }
  a.scale = scale;
  a.Y = Y;
  a.T_save = T_save;
  a.Tpair = Tpair;
  a.absmax_q = absmax_q;
  a.absmax_scale = absmax_scale;
  const WsParts wp = ws_parts(M, N);
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  int* cnt = reinterpret_cast<int*>(ws + wp.cnt);
  a.G4 = static_cast<int>((M + 3) / 4);
  a.tile_first = cnt;
  a.tile_last = cnt + a.tiles;
  a.t_cnt1 = cnt + 2 * a.tiles;
  a.t_cnt2 = a.t_cnt1 + 4 * kMaxTGroups;
  a.t_ready = a.t_cnt2 + 4;
  a.bar_count = a.t_ready + 1;
  a.bar_gen = a.bar_count + 1;
  a.t_part = reinterpret_cast<float*>(ws + wp.t_part);
  a.t_l1 = reinterpret_cast<float*>(ws + wp.t_l1);
  a.partial = reinterpret_cast<float*>(ws + wp.partial);
  a.status = status;
  a.wait_ns = wait_limit_ns();
  a.nf4 = P;
  switch (MP) {
    case 16: return launch_mp<16>(mC, mX, mA, mB, mT, a, stream);
    case 32: return launch_mp<32>(mC, mX, mA, mB, mT, a, stream);
    case 64: return launch_mp<64>(mC, mX, mA, mB, mT, a, stream);
    default: return launch_mp<128>(mC, mX, mA, mB, mT, a, stream);
  }
}

}  // namespace qlora
