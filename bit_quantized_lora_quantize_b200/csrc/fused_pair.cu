// Fused NF4 dequant-GEMMs on CTA pairs (tcgen05 cta_group::2), sm_100a.
//
// "AI Glossary: QLoRA", second paragraph, and "QLoRA's Working Process":
// the frozen 4-bit weight is turned back into BFloat16 on the fly for each
// product; no bf16 copy of W is stored.
//
//   forward         Y  = X  W'^T + [T_hi | T_lo] [B ; B]      (B operand K-major)
//   input gradient  dX = dY W'   + [U_hi | U_lo] [A^T ; A^T]  (B operand MN-major)
//
// The rank-r intermediate the LoRA stages read (T = s X A in the forward,
// U = s dY B^T in the input gradient) is computed by the same kernel: the
// first tickets of the grid are "rank units", one per 512-row block, that
// stream the same activation rows through the same pipeline against a
// 64-column slice of the adapter matrix per CTA (N = 128 across the pair),
// write the float32 result and its bf16 pair, and raise that block's ready
// count.  Output tiles wait for the count only before their LoRA stages, so
// the rank units run in the time the grid's last wave would leave SMs idle,
// and no separate launch stands between the inputs and the GEMM.
//
// The input-gradient launch also forms the adapter gradients in "tail
// units": dA = X^T U and dB^T = dY^T T, each unit 512 rows of the result
// reduced over all M tokens in TMEM (A operand MN-major: activation columns;
// B operand the [hi | lo] pair, N = 2rp across the pair, the halves added in
// the epilogue).  Tickets go out as: rank units; tiles for the rest of the
// first wave; as many tail units as there are rank units (taken by the pairs
// that finish the shorter rank units first); the remaining tiles; the
// remaining tail units (short jobs that fill the last wave's idle SMs).
//
// Two CTAs of a cluster compute one 512 x 256 output tile.  Each CTA holds
// 2 x 128 rows of the activation tile (one 128-row half of each of two
// M = 256 pair-MMAs) and decodes its own 128-row half of the weight tile; the
// pair's tensor cores read both halves.  Every decoded weight therefore feeds
// 512 output rows, which halves the decode work per tensor-core cycle
// compared with a 256-row single-CTA tile, and a stage is 52 KB so four
// stages fit.
//
// Per CTA: warp 0 issues TMA (activation rows and LoRA tiles signal the
// leader CTA's barrier, packed codes a local one; no multicast loads), warp 1
// allocates TMEM (both CTAs); in the leader only, warps 1 and 2 issue the MMAs
// of the two accumulators and commit them to both CTAs' barriers; warps 4-7
// decode the even stages and
// warps 8-11 the odd ones (one 64-weight block per thread per stage), then
// all eight drain the two 128 x 256 fp32 accumulators.
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

constexpr int kPairRows = 512;    // output rows of a pair tile
constexpr int kPairCols = 256;    // output columns of a pair tile
constexpr int kDepth = 64;
constexpr int kStages = 4;
constexpr int kThreads = 384;
constexpr int kDecWarps = 4;      // decoder warps per stage (warps 4-7 even stages, 8-11 odd)

struct PairArgs {
  int units;        // CTA pairs in the grid
  int tiles_n;      // output tiles along the columns
  int tiles_m;      // output tiles along the rows (512-row blocks)
  int group_rows;   // row blocks per tile group (tile order, see tile_coords)
  // Rank units (one per 512-row block) ahead of the output tiles, or 0 when
  // the bf16 pair comes from the previous kernel in the stream.
  int r_units;
  int* ctr;         // [ticket, done, ready count per row block]; null: units by block index
  int r;            // adapter rank
  float scale;      // LoRA scale s, applied to the rank-r intermediate
  float* r_f32;     // float32 intermediate [rows x r] (forward T) or null
  uint16_t* r_pair; // bf16 pair of the intermediate, read by the LoRA stages
  // Tail units (input gradient only): for each chunk of t_chunk adapter
  // columns, da_units of dA then the dB ones (t_base per chunk).  The first
  // t_first go out after the first `early` tiles, the rest after all tiles.
  int t_units, da_units, early, t_first, t_base, t_chunk;
  int unit_cols;    // adapter columns per CTA of a rank unit (64 or 128)
  int nmb;          // 64-row blocks of M (reduction depth of a tail unit)
  float* dA;        // [K x r]
  float* dB;        // [r x N]
  // Input gradient: the rank units also write the bf16 pair of T (read by
  // the dB tail units) from T as saved by the forward, for their rows.
  const float* t_src;
  uint16_t* t_pair;
  int nkb;          // main 64-deep stages
  int lora_kb;      // LoRA stages (hi and lo halves of the pair)
  int lora_mod;     // rp: LoRA stage lk reads the adapter at (64*lk) mod rp
  int rows, cols;   // output extent
  int64_t ld_out;
  uint16_t* out;
  const uint8_t* absmax_q;
  const float* absmax_scale;
  int64_t w_rows, w_cols;  // N, K of the packed weight
  int abs_tma;             // dX: 8-bit constant codes by TMA
  int* status;
  uint64_t wait_ns;         // limit of every bounded wait
  Nf4Params nf4;
};

// Tensor maps of the tail units: activation columns (64 x 64 boxes) and the
// bf16 pairs they are reduced against.
struct TailMaps {
  CUtensorMap a_da, b_da, a_db, b_db;
};

template <bool MNB>
struct PairSmem {
  static constexpr int kA = 2 * 128 * kDepth * 2;   // 32 KB: two 128-row halves
  static constexpr int kB = 128 * kDepth * 2;       // 16 KB: this CTA's half of the weight tile
  static constexpr int kC = 4096;                   // packed codes of that half
  static constexpr int kAbs = MNB ? 1024 : 0;
  static constexpr int offA = 0;
  static constexpr int offB = offA + kStages * kA;
  static constexpr int offC = offB + kStages * kB;
  static constexpr int offAbs = offC + kStages * kC;
  static constexpr int offLvl2 = offAbs + kStages * kAbs;
  static constexpr int offBar = offLvl2 + 1024;
  // full, cfull, empty, decoded per stage; acc_full; one MMA drain per issuer
  static constexpr int kNumBars = 4 * kStages + 3;
  static constexpr int offSlot = offBar + kNumBars * 8;
  static constexpr int offAbort = offSlot + 4;
  static constexpr int offUnit = offAbort + 4;
  static constexpr int kTotal = offUnit + 4;
  static constexpr int kDynamic = kTotal + 1024;
};

// Output tile order.  Tiles go out in groups of `group_rows` consecutive
// 512-row blocks; inside a group, column by column, each column's row blocks
// in turn.  The activation rows of a group (group_rows x 512 x depth bf16)
// are sized on the host to stay in L2 while the group sweeps its columns, and
// the pairs working at the same time share the packed codes of a few
// columns, so each code tile comes from HBM about once per group instead of
// once per row block.
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int group_rows, int& tm, int& tn) {
  const int per_group = group_rows * tiles_n;
  const int g = tile / per_group;
  const int idx = tile - g * per_group;
  const int r0 = g * group_rows;
  const int rows = min(group_rows, tiles_m - r0);
  tn = idx / rows;
  tm = r0 + (idx - tn * rows);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared::cluster address of the same object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(smem_u32(p)), "r"(rank));
  return d;
}
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t mbar_cluster, void* dst, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ int ld_cluster_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t mbar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(mbar_cluster) : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs once the issued MMAs end.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

template <bool MNB>
__global__ void __launch_bounds__(kThreads, 1)
    fused_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmC,
                      const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                      const __grid_constant__ CUtensorMap tmAbs, const __grid_constant__ CUtensorMap tmR,
                      const __grid_constant__ TailMaps tm, const PairArgs args) {
  using L = PairSmem<MNB>;
  constexpr uint32_t kTmemCols = 512;  // two 128 x 256 fp32 accumulators

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + L::offA;
  uint8_t* sB = smem + L::offB;
  uint8_t* sC = smem + L::offC;
  uint8_t* sAbs = smem + L::offAbs;
  float* lvl2 = reinterpret_cast<float*>(smem + L::offLvl2);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::offBar);  // leader: both CTAs' TMA bytes
  uint64_t* cfull = full + kStages;                                // local: this CTA's codes
  uint64_t* empty = cfull + kStages;                               // local: MMA done with the stage
  uint64_t* decoded = empty + kStages;                             // leader: both CTAs' decoders
  uint64_t* acc_full = decoded + kStages;                          // local: accumulators ready
  uint64_t* mma_drain = acc_full + 1;                              // leader: an issuer's MMAs ended (abort)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::offSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offAbort);
  int* unit_slot = reinterpret_cast<int*>(smem + L::offUnit);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = leader

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&cfull[s], 1);
      mbar_init(&empty[s], 2);  // one commit from each MMA issuer
      mbar_init(&decoded[s], 2 * kDecWarps);
    }
    mbar_init(acc_full, 2);
    mbar_init(&mma_drain[0], 1);
    mbar_init(&mma_drain[1], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmC);
    tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB2);
    if (args.r_units) tma_prefetch_desc(&tmR);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  if (args.ctr) {
    // Units by ticket, so that the rank units (the first tickets) have started
    // before any tile can wait for them.  All inputs may come from the
    // previous kernel in the stream: wait for it before the first load.
    griddep_wait();
    if (threadIdx.x == 0 && rank == 0) *unit_slot = atomicAdd(args.ctr, 1);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's barriers (and ticket) exist before the peer uses them
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;
  int unit = static_cast<int>(blockIdx.x >> 1);
  if (args.ctr) unit = rank == 0 ? *unit_slot : ld_cluster_s32(map_rank(unit_slot, 0));
  // Ticket order: rank units; tiles [0, early); tail units [0, t_first);
  // the other tiles; the other tail units.
  const bool runit = unit < args.r_units;
  const int v = unit - args.r_units;
  const int ntiles = args.units - args.r_units - args.t_units;
  int tile = 0, tj = -1;
  if (!runit) {
    if (v < args.early) tile = v;
    else if (v < args.early + args.t_first) tj = v - args.early;
    else if (v < ntiles + args.t_first) tile = v - args.t_first;
    else tj = v - ntiles;
  }
  const bool tunit = tj >= 0;
  int tile_m = unit, tile_n = 0;
  if (!runit) tile_coords(tile, args.tiles_m, args.tiles_n, args.group_rows, tile_m, tile_n);
  const int total = runit ? args.nkb : (tunit ? args.nmb : args.nkb + args.lora_kb);
  // Without rank units the previous kernel produces only the LoRA
  // intermediate, read in the last stages: everything else may start now.
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const WaitCtx ctx{abort_flag, args.status, 21, args.wait_ns};
      int issued = 0;
      for (int i = 0; i < total; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, ctx)) break;
        const uint32_t full_leader = map_rank(&full[s], 0);
        uint8_t* a_dst = sA + s * L::kA;
        uint8_t* b_dst = sB + s * L::kB;
        const int row0 = tile_m * kPairRows + static_cast<int>(rank) * 128;
        if (tunit) {
          // 64 tokens per stage: this CTA's 2 x 128 result rows of the
          // activation (four 64-column boxes) and its t_chunk columns of the
          // pair (the hi half in the leader, the lo half in the peer).
          const int chunk = tj / args.t_base, tb = tj - chunk * args.t_base;
          const bool is_da = tb < args.da_units;
          if (i == 0) {
            bool ok = true;
            for (int m = 0; m < args.r_units && ok; ++m) ok = wait_count(args.ctr + 2 + m, 2, ctx);
            if (!ok) break;
            fence_proxy_async_global();  // the U and T pairs are written by this launch's rank units
          }
          const CUtensorMap* am = is_da ? &tm.a_da : &tm.a_db;
          const CUtensorMap* bm = is_da ? &tm.b_da : &tm.b_db;
          const int c0 = (is_da ? tb : tb - args.da_units) * kPairRows + static_cast<int>(rank) * 128;
          const int nb = args.t_chunk / 64;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * L::kA + 2 * nb * 8192);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int a = 0; a < 2; ++a)
              tma_load_2d_pair(am, full_leader, a_dst + h * 16384 + a * 8192, c0 + h * 256 + a * 64, i * kDepth);
          for (int b = 0; b < nb; ++b)
            tma_load_2d_pair(bm, full_leader, b_dst + b * 8192,
                             static_cast<int>(rank) * args.lora_mod + chunk * args.t_chunk + b * 64, i * kDepth);
          ++issued;
          continue;
        }
        if (i < args.nkb) {
          const int kb = i;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * L::kA + (runit ? 2 * args.unit_cols * kDepth * 2 : 0));
          tma_load_2d_pair(&tmA, full_leader, a_dst, kb * kDepth, row0);
          tma_load_2d_pair(&tmA, full_leader, a_dst + 16384, kb * kDepth, row0 + 256);
          if (runit) {
            // This CTA's unit_cols adapter columns (64-wide boxes): forward
            // A[K, r] rows of block kb (MN-major B operand), input gradient
            // B[r, N] columns of block kb (K-major).  Columns past r read as
            // zeros.
            for (int b = 0; b < args.unit_cols / 64; ++b) {
              const int col = static_cast<int>(rank) * args.unit_cols + b * 64;
              if (!MNB) tma_load_2d_pair(&tmR, full_leader, b_dst + b * 8192, col, kb * kDepth);
              else tma_load_2d_pair(&tmR, full_leader, b_dst + b * 8192, kb * kDepth, col);
            }
            ++issued;
            continue;
          }
          const bool abs_tma = MNB && args.abs_tma;
          mbar_arrive_expect_tx(&cfull[s], L::kC + (abs_tma ? 1024 : 0));
          if (!MNB) {
            // codes [N, K/2]: this CTA's 128 weight rows x 32 bytes
            tma_load_2d(&tmC, &cfull[s], sC + s * L::kC, kb * 32, tile_n * kPairCols + static_cast<int>(rank) * 128);
          } else {
            // codes: 64 reduction rows x 64 bytes (this CTA's 128 outputs)
            tma_load_2d(&tmC, &cfull[s], sC + s * L::kC, tile_n * 128 + static_cast<int>(rank) * 64, kb * kDepth);
            if (abs_tma)
              tma_load_2d(&tmAbs, &cfull[s], sAbs + s * 1024, ((tile_n * 4) + static_cast<int>(rank) * 2) & ~15,
                          kb * kDepth);
          }
        } else {
          const int lk = i - args.nkb;
          const int lb = (lk * kDepth) % args.lora_mod;
          if (lk == 0) {
            if (args.ctr) {
              // the pair is written by this row block's rank unit
              if (!wait_count(args.ctr + 2 + tile_m, 2, ctx)) break;
              fence_proxy_async_global();
            } else {
              griddep_wait();  // the pair is the previous kernel's output
            }
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (L::kA + L::kB));
          tma_load_2d_pair(&tmA2, full_leader, a_dst, lk * kDepth, row0);
          tma_load_2d_pair(&tmA2, full_leader, a_dst + 16384, lk * kDepth, row0 + 256);
          const int c0 = tile_n * kPairCols + static_cast<int>(rank) * 128;
          if (!MNB) {
            // LoRA B [r, N] (MN-major): this CTA's 128 output columns
            tma_load_2d_pair(&tmB2, full_leader, b_dst, c0, lb);
            tma_load_2d_pair(&tmB2, full_leader, b_dst + 8192, c0 + 64, lb);
          } else {
            // LoRA A [K, r] (K-major): this CTA's 128 output rows of A
            tma_load_2d_pair(&tmB2, full_leader, b_dst, lb, c0);
          }
        }
        ++issued;
      }
      if (*abort_flag) {
        // Let every copy this CTA pair issued land before the CTAs exit (the
        // leader's full barrier counts both CTAs' activation bytes).
        for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i) {
          const int s = i % kStages;
          const uint32_t ph = (i / kStages) & 1;
          const bool codes = i < args.nkb && !runit && !tunit;  // only these stages load codes
          if (codes) mbar_drain(&cfull[s], ph);
          if (rank == 0) mbar_drain(&full[s], ph);
        }
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA (leader)
    // One tcgen05.mma takes its issuing thread about as long as the tensor
    // cores take to execute it at this tile size, so the two M = 256
    // accumulators are fed by two threads: warp 1 issues the first, warp 2 the
    // second; each commits to the stage and accumulator barriers (count 2).
    if (lane == 0 && rank == 0) {
      const int h = warp - 1;
      const WaitCtx ctx{abort_flag, args.status, 22, args.wait_ns};
      // M = 256 across the pair, N = 256 (each CTA supplies 128 columns of B).
      const uint32_t idesc_main = idesc_bf16_f32(256, 256, false, MNB);
      const uint32_t idesc_lora = idesc_bf16_f32(256, 256, false, !MNB);
      const uint32_t idesc_unit = idesc_bf16_f32(256, 2 * args.unit_cols, false, !MNB);
      const uint32_t idesc_tail = idesc_bf16_f32(256, 2 * args.t_chunk, true, true);
      const uint32_t d = tmem_acc + h * 256;
      bool ok = true;
      for (int i = 0; i < total && ok; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        const bool main_stage = i < args.nkb;
        const bool dec_stage = main_stage && !runit && !tunit;  // B is the decoded weight
        if (!mbar_wait(&full[s], ph, ctx)) { ok = false; break; }
        if (dec_stage && !mbar_wait(&decoded[s], ph, ctx)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sA + s * L::kA) + h * 16384;
        const uint32_t b_base = smem_u32(sB + s * L::kB);
        // The B operand is the decoded weight in main stages of output tiles
        // and an adapter matrix or pair otherwise; only tail units read A
        // MN-major.
        const bool b_mn = tunit || (dec_stage ? MNB : !MNB);
        const uint32_t idesc = tunit ? idesc_tail : (runit ? idesc_unit : (main_stage ? idesc_main : idesc_lora));
#pragma unroll
        for (int kk = 0; kk < kDepth / 16; ++kk) {
          const uint64_t bdesc = b_mn ? smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                      : smem_desc_sw128(b_base + kk * 32, 16, 1024);
          const uint64_t adesc = tunit ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                       : smem_desc_sw128(a_base + kk * 32, 16, 1024);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          umma_pair(d, adesc, bdesc, idesc, acc);
        }
        umma_commit_pair(&empty[s]);
      }
      if (ok) {
        umma_commit_pair(acc_full);
      } else {
        // Aborted: wait until the MMAs this thread issued have ended, so that
        // neither CTA frees its TMEM or leaves while they still read the
        // pair's shared memory.
        umma_commit_pair(&mma_drain[h]);
        mbar_drain(&mma_drain[h], 0);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ decoders (warps 4-11)
    // Two groups of four warps take alternate stages; in each group thread d
    // decodes one 64-weight block of this CTA's half of the weight tile.
    {
      const WaitCtx ctx{abort_flag, args.status, 23, args.wait_ns};
      const int grp = (warp - 4) >> 2;          // 0: even stages, 1: odd stages
      const int d = (threadIdx.x - 128) & 127;  // 0..127
      lvl2[threadIdx.x - 128] = level2_value_for(threadIdx.x - 128, args.nf4.centred);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      const int64_t blocks_per_row = args.w_cols / 64;
      const float mu = centred_mu(args.absmax_scale, (args.w_rows * blocks_per_row + 255) / 256, args.nf4.centred);
      if (runit || tunit) {
        // Rank and tail units read no weight.  In the input gradient the
        // rank units' idle decoder threads write the bf16 pair of the saved
        // T for the unit's rows (one row per thread), for the dB tail units.
        if (runit && args.t_pair) {
          const int local = threadIdx.x - 128;  // 0..255
          const int64_t row = static_cast<int64_t>(tile_m) * kPairRows + (local >> 7) * 256 + rank * 128 + (local & 127);
          const int rp = args.lora_mod;
          if (row < args.rows) {
            const float* ts = args.t_src + row * args.r;
            uint16_t* tp = args.t_pair + row * 2 * rp;
#pragma unroll 1
            for (int c0 = 0; c0 < rp; c0 += 8) {
              float tv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
              if (c0 < args.r) {
                const float4 t0 = __ldg(reinterpret_cast<const float4*>(ts + c0));
                const float4 t1 = __ldg(reinterpret_cast<const float4*>(ts + c0 + 4));
                tv[0] = t0.x; tv[1] = t0.y; tv[2] = t0.z; tv[3] = t0.w;
                tv[4] = t1.x; tv[5] = t1.y; tv[6] = t1.z; tv[7] = t1.w;
              }
              uint32_t hi[4], lo[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat16 h0 = __float2bfloat16_rn(tv[2 * e]);
                const __nv_bfloat16 h1 = __float2bfloat16_rn(tv[2 * e + 1]);
                const __nv_bfloat16 l0 = __float2bfloat16_rn(__fsub_rn(tv[2 * e], __bfloat162float(h0)));
                const __nv_bfloat16 l1 = __float2bfloat16_rn(__fsub_rn(tv[2 * e + 1], __bfloat162float(h1)));
                hi[e] = __bfloat16_as_ushort(h0) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
                lo[e] = __bfloat16_as_ushort(l0) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
              }
              *reinterpret_cast<uint4*>(tp + c0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
              *reinterpret_cast<uint4*>(tp + rp + c0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
          }
        }
      } else if (!MNB) {
        // Thread d decodes weight row n (this CTA's half), one block per stage.
        const int64_t n = static_cast<int64_t>(tile_n) * kPairCols + rank * 128 + d;
        const bool row_ok = n < args.w_rows;
        const uint32_t b_row = (d >> 3) * 1024;
        const int r8 = d & 7;
        int64_t blk = n * blocks_per_row + grp;
        uint32_t q2 = 0;
        float c1 = 0.0f;
        if (row_ok && grp < args.nkb) {
          q2 = __ldg(args.absmax_q + blk);
          c1 = __ldg(args.absmax_scale + (blk >> 8));
        }
        for (int i = grp; i < args.nkb; i += 2) {
          const int s = i % kStages;
          const uint32_t ph = (i / kStages) & 1;
          uint32_t q2n = 0;
          float c1n = 0.0f;
          if (row_ok && i + 2 < args.nkb) {
            q2n = __ldg(args.absmax_q + blk + 2);
            c1n = __ldg(args.absmax_scale + ((blk + 2) >> 8));
          }
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&cfull[s], ph, ctx))) break;
          uint8_t* dst = sB + s * L::kB + b_row;
          if (row_ok) {
            // 32-byte rows with the 32-byte swizzle: chunk c at c ^ ((d >> 2) & 1)
            const uint8_t* src = sC + s * L::kC + d * 32;
            const int sw = (d >> 2) & 1;
            const uint4 v0 = *reinterpret_cast<const uint4*>(src + ((0 ^ sw) << 4));
            const uint4 v1 = *reinterpret_cast<const uint4*>(src + ((1 ^ sw) << 4));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const Nf4Lut lut = make_lut(args.nf4, __fadd_rn(__fmul_rn(lvl2[q2], c1), mu));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o[4];
              decode8(lut, w[c], o);
              *reinterpret_cast<uint4*>(dst + sw128_offset(r8, c)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst + sw128_offset(r8, c)) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_rank(&decoded[s], 0));
          q2 = q2n;
          c1 = c1n;
          blk += 2;
        }
      } else {
        // Thread d: reduction row nl of the stage, output atom j (64 outputs).
        const int nl = d & 63;
        const int j = d >> 6;  // 0..1
        const int64_t kob = static_cast<int64_t>(tile_n) * 4 + rank * 2 + j;  // 64-wide output block
        const bool col_ok = kob < blocks_per_row;
        const uint32_t b_off = j * 8192 + (nl >> 3) * 1024;
        const int r8 = nl & 7;
        const bool abs_tma = args.abs_tma != 0;
        const int abs_col = static_cast<int>(kob - ((static_cast<int64_t>(tile_n) * 4 + rank * 2) & ~int64_t(15)));
        auto load_const = [&](int i, uint32_t& q, float& c) {
          const int64_t n = static_cast<int64_t>(i) * 64 + nl;
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
        bool ok_cur = grp < args.nkb ? load_const(grp, q2, c1) : false;
        for (int i = grp; i < args.nkb; i += 2) {
          const int s = i % kStages;
          const uint32_t ph = (i / kStages) & 1;
          uint32_t q2n = 0;
          float c1n = 0.0f;
          const bool ok_next = (i + 2 < args.nkb) ? load_const(i + 2, q2n, c1n) : false;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&cfull[s], ph, ctx))) break;
          uint8_t* dst = sB + s * L::kB + b_off;
          if (ok_cur) {
            // 64-byte rows with the 64-byte swizzle: chunk c at c ^ ((nl >> 1) & 3)
            const uint8_t* row = sC + s * L::kC + nl * 64;
            const int sw = (nl >> 1) & 3;
            const uint4 v0 = *reinterpret_cast<const uint4*>(row + (((2 * j) ^ sw) << 4));
            const uint4 v1 = *reinterpret_cast<const uint4*>(row + (((2 * j + 1) ^ sw) << 4));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            if (abs_tma) q2 = sAbs[s * 1024 + nl * 16 + abs_col];
            const Nf4Lut lut = make_lut(args.nf4, __fadd_rn(__fmul_rn(lvl2[q2], c1), mu));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o[4];
              decode8(lut, w[c], o);
              *reinterpret_cast<uint4*>(dst + sw128_offset(r8, c)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(dst + sw128_offset(r8, c)) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_rank(&decoded[s], 0));
          q2 = q2n;
          c1 = c1n;
          ok_cur = ok_next;
        }
      }
    }
    // ------------------------------------------------------------ epilogue (warps 4-11)
    {
      const WaitCtx ctx{abort_flag, args.status, 24, args.wait_ns};
      const int q = warp & 3;
      const int h = (warp - 4) >> 2;  // accumulator (first or second M = 256 MMA)
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0, ctx));
      tc_fence_after();
      const int row = tile_m * kPairRows + h * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
      const uint32_t t_row = tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + h * 256;
      if (ok && runit) {
        // v = s * acc in float32 (the forward keeps it as T); the pair holds
        // hi = bf16(v) in columns [0, rp) and lo = bf16(v - hi) in [rp, 2rp),
        // zero past r.
        const int rp = args.lora_mod;
#pragma unroll 1
        for (int cc = 0; cc < rp / 32; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + cc * 32, v);
          tmem_wait_ld();
          if (row < args.rows) {
            uint16_t* pr = args.r_pair + static_cast<int64_t>(row) * 2 * rp;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int c0 = cc * 32 + g * 8;
              float sv[8];
              uint32_t hi[4], lo[4];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                sv[e] = (c0 + e < args.r) ? __fmul_rn(args.scale, __uint_as_float(v[g * 8 + e])) : 0.0f;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat16 h0 = __float2bfloat16_rn(sv[2 * e]);
                const __nv_bfloat16 h1 = __float2bfloat16_rn(sv[2 * e + 1]);
                const __nv_bfloat16 l0 = __float2bfloat16_rn(__fsub_rn(sv[2 * e], __bfloat162float(h0)));
                const __nv_bfloat16 l1 = __float2bfloat16_rn(__fsub_rn(sv[2 * e + 1], __bfloat162float(h1)));
                hi[e] = __bfloat16_as_ushort(h0) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
                lo[e] = __bfloat16_as_ushort(l0) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
              }
              *reinterpret_cast<uint4*>(pr + c0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
              *reinterpret_cast<uint4*>(pr + rp + c0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
              if (args.r_f32 && c0 < args.r) {
                float* tf = args.r_f32 + static_cast<int64_t>(row) * args.r + c0;
                *reinterpret_cast<float4*>(tf) = make_float4(sv[0], sv[1], sv[2], sv[3]);
                *reinterpret_cast<float4*>(tf + 4) = make_float4(sv[4], sv[5], sv[6], sv[7]);
              }
            }
          }
        }
      } else if (ok && tunit) {
        // Result rows (k of dA, n of dB) in lanes; columns [0, rc) hold the
        // product with the chunk's hi half of the pair, [rc, 2rc) with its lo
        // half (rc = t_chunk adapter columns, chunk `chunk`).
        const int rc = args.t_chunk;
        const int chunk = tj / args.t_base, tb = tj - chunk * args.t_base;
        const bool is_da = tb < args.da_units;
        const int rrow = (is_da ? tb : tb - args.da_units) * kPairRows + h * 256 + static_cast<int>(rank) * 128 +
                         q * 32 + lane;
        const bool in = rrow < (is_da ? args.w_cols : args.w_rows);
#pragma unroll 1
        for (int cc = 0; cc < rc / 32; ++cc) {
          uint32_t vh[32], vl[32];
          tmem_ld_32x32b_x32(t_row + cc * 32, vh);
          tmem_ld_32x32b_x32(t_row + rc + cc * 32, vl);
          tmem_wait_ld();
          if (in) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const int j = chunk * rc + cc * 32 + e;
              if (j < args.r) {
                const float4 o = make_float4(__fadd_rn(__uint_as_float(vh[e]), __uint_as_float(vl[e])),
                                             __fadd_rn(__uint_as_float(vh[e + 1]), __uint_as_float(vl[e + 1])),
                                             __fadd_rn(__uint_as_float(vh[e + 2]), __uint_as_float(vl[e + 2])),
                                             __fadd_rn(__uint_as_float(vh[e + 3]), __uint_as_float(vl[e + 3])));
                if (is_da) {
                  *reinterpret_cast<float4*>(args.dA + static_cast<int64_t>(rrow) * args.r + j) = o;
                } else {
                  float* col = args.dB + static_cast<int64_t>(j) * args.w_rows + rrow;
                  col[0] = o.x;
                  col[args.w_rows] = o.y;
                  col[2 * args.w_rows] = o.z;
                  col[3 * args.w_rows] = o.w;
                }
              }
            }
          }
        }
      } else if (ok) {
#pragma unroll 1
        for (int cc = 0; cc < kPairCols / 32; ++cc) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + cc * 32, v);
          tmem_wait_ld();
          const int col0 = tile_n * kPairCols + cc * 32;
          if (row < args.rows) {
            uint16_t* out = args.out + static_cast<int64_t>(row) * args.ld_out;
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
        }
      }
      if (runit) {
        // Publish this CTA's half of the row block: stores visible to other
        // CTAs' TMA loads, then one count per CTA (the tiles wait for 2).
        fence_proxy_async_global();
        __threadfence();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (threadIdx.x == 128) atomicAdd(args.ctr + 2 + tile_m, 1);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the pair's MMAs or signals may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_acc, kTmemCols);
  }
  if (args.ctr && threadIdx.x == 0 && rank == 0) {
    // The last pair to finish returns the counters to zero: every pair has
    // taken its ticket and is past its last look at a ready count.
    __threadfence();
    if (atomicAdd(args.ctr + 1, 1) == args.units - 1) {
      for (int m = 0; m < args.r_units; ++m) args.ctr[2 + m] = 0;
      args.ctr[0] = 0;
      args.ctr[1] = 0;
      __threadfence();
    }
  }
}

template <bool MNB>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& c, const CUtensorMap& a2, const CUtensorMap& b2,
                        const CUtensorMap& abs, const CUtensorMap& rmap, const TailMaps& tmaps, const PairArgs& args,
                        cudaStream_t stream) {
  using L = PairSmem<MNB>;
  static_assert(L::kDynamic <= 232448, "shared memory budget");
  auto kern = fused_pair_kernel<MNB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynamic);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * args.units), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kDynamic;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a, c, a2, b2, abs, rmap, tmaps, args);
}

// Row blocks per tile group: as few groups as keep one group's activation
// rows (512 x depth bf16 per row block) within half of L2, balanced.
int group_rows_for(int tiles_m, int64_t depth) {
  const int64_t block_bytes = static_cast<int64_t>(kPairRows) * depth * 2;
  const int64_t budget = device_l2_bytes() / 2;
  const int64_t fit = std::max<int64_t>(1, budget / std::max<int64_t>(1, block_bytes));
  const int64_t groups = (tiles_m + fit - 1) / fit;
  return static_cast<int>((tiles_m + groups - 1) / groups);
}

// Unit count and rank-unit fields shared by both directions.  `depth` is the
// reduction length of the output tiles (K forward, N input gradient).
void plan_units(PairArgs& args, int64_t M, int64_t cols, int64_t depth, int r, float scale, int* ctr,
                float* r_f32, uint16_t* r_pair) {
  const int tiles_n = static_cast<int>((cols + kPairCols - 1) / kPairCols);
  const int tiles_m = static_cast<int>((M + kPairRows - 1) / kPairRows);
  args.tiles_n = tiles_n;
  args.tiles_m = tiles_m;
  args.group_rows = group_rows_for(tiles_m, depth);
  args.r_units = ctr ? tiles_m : 0;
  args.units = tiles_m * tiles_n + args.r_units;
  args.ctr = ctr;
  args.r = r;
  args.scale = scale;
  args.r_f32 = r_f32;
  args.r_pair = r_pair;
  args.early = tiles_m * tiles_n;
  const int rp = lora_pad(r);
  args.unit_cols = rp <= 128 ? 64 : 128;               // N = 2 * unit_cols <= 256 across the pair
  args.t_chunk = rp <= 128 ? rp : (rp % 128 == 0 ? 128 : 64);
}

// CTA pairs resident at once (one 1-CTA-per-SM pair per two SMs).
int resident_pairs() { return std::max(1, device_sm_count() / 2); }

}  // namespace

int fused_ctr_ints(int64_t M) { return 2 + static_cast<int>((M + kPairRows - 1) / kPairRows); }

cudaError_t launch_fused_fwd(const uint16_t* X, const uint8_t* codes, const uint8_t* absmax_q,
                             const float* absmax_scale, uint16_t* Tpair, const uint16_t* B, int64_t M, int64_t K,
                             int64_t N, int r, uint16_t* Y, int* status, const Nf4Params& P, cudaStream_t stream,
                             const uint16_t* A, float* T_save, float scale, int* ctr) {
  const int rp = lora_pad(r);
  CUtensorMap mX, mC, mT, mB, mR;
  if (!make_map_2d(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_32B) ||
      !make_map_2d(&mT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Tpair, 2 * rp, M, static_cast<int64_t>(rp) * 4, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, r, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  mR = mB;
  if (ctr) {
    // A [K, r]: 64 reduction rows x 64 adapter columns per CTA and stage
    if (!A || !T_save ||
        !make_map_2d(&mR, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, r, K, static_cast<int64_t>(r) * 2, 64, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  PairArgs args{};
  plan_units(args, M, N, K, r, scale, ctr, T_save, Tpair);
  args.nkb = static_cast<int>(K / 64);
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
  args.abs_tma = 0;
  args.status = status;
  args.wait_ns = wait_limit_ns();
  args.nf4 = P;
  const TailMaps none{mB, mB, mB, mB};
  return launch_pair<false>(mX, mC, mT, mB, mB, mR, none, args, stream);
}

cudaError_t launch_fused_dx(const uint16_t* dY, const uint8_t* codes, const uint8_t* absmax_q,
                            const float* absmax_scale, uint16_t* Upair, const uint16_t* A, int64_t M, int64_t K,
                            int64_t N, int r, uint16_t* dX, int* status, const Nf4Params& P, cudaStream_t stream,
                            const uint16_t* B, float scale, int* ctr, const uint16_t* X, const float* T_save,
                            uint16_t* Tpair, float* dA, float* dB) {
  const int rp = lora_pad(r);
  CUtensorMap mD, mC, mU, mA, mR;
  if (!make_map_2d(&mD, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, N, M, N * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_2d(&mU, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Upair, 2 * rp, M, static_cast<int64_t>(rp) * 4, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, r, K, static_cast<int64_t>(r) * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  mR = mA;
  if (ctr) {
    // B [r, N]: 64 adapter rows x 64 reduction columns per CTA and stage
    if (!B || !make_map_2d(&mR, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, r, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  CUtensorMap mAbs = mA;
  const bool abs_tma = (K % 1024 == 0) &&
                       make_map_2d(&mAbs, CU_TENSOR_MAP_DATA_TYPE_UINT8, absmax_q, K / 64, N, K / 64, 16, 64,
                                   CU_TENSOR_MAP_SWIZZLE_NONE);
  PairArgs args{};
  plan_units(args, M, K, N, r, scale, ctr, nullptr, Upair);
  TailMaps tails{mA, mA, mA, mA};
  if (ctr && dA && dB) {
    // dA = X^T U and dB^T = dY^T T: 64 tokens x 64 result rows per box
    const int64_t ps = static_cast<int64_t>(rp) * 4;
    if (!X || !T_save || !Tpair ||
        !make_map_2d(&tails.a_da, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tails.b_da, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Upair, 2 * rp, M, ps, 64, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tails.a_db, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, N, M, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tails.b_db, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Tpair, 2 * rp, M, ps, 64, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    args.da_units = static_cast<int>((K + kPairRows - 1) / kPairRows);
    args.t_base = args.da_units + static_cast<int>((N + kPairRows - 1) / kPairRows);
    args.t_units = args.t_base * (rp / args.t_chunk);
    args.early = std::min(args.early, std::max(0, resident_pairs() - args.r_units));
    args.t_first = std::min(args.t_units, args.r_units);
    args.units += args.t_units;
    args.nmb = static_cast<int>((M + 63) / 64);
    args.dA = dA;
    args.dB = dB;
    args.t_src = T_save;
    args.t_pair = Tpair;
  }
  args.nkb = static_cast<int>((N + 63) / 64);
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
  args.abs_tma = abs_tma ? 1 : 0;
  args.status = status;
  args.wait_ns = wait_limit_ns();
  args.nf4 = P;
  return launch_pair<true>(mD, mC, mU, mA, mAbs, mR, tails, args, stream);
}

}  // namespace qlora
