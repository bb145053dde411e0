// Small-M forward of the NF4 LoRA linear layer for M <= 16 tokens, sm_100a.
//
// "QLoRA: Fine-Tuning 65-Billion Parameter Models on a Single Consumer GPU",
// "QLoRA's Working Process" and its closing remark that 4-bit inference is
// still slow: with a handful of tokens the forward is a stream over the packed
// weight.  What bounds such a stream here is the number of bytes in flight
// per SM and the shared-memory traffic of the decode, so this path:
//
//  * streams the codes with TMA in tiles of 256 weight rows x 128 bytes (256
//    inputs, four 64-input blocks) through a 4-stage ring, 128 KB in flight
//    per SM, and brings the matching slice of X with one 5-D TMA whose box
//    lands it in the order the MMA fragments are read in (no multicast);
//  * decodes a code byte with one byte permute, which forms the address of a
//    bf16 level pair in a table with 32 bank-private copies, and one 32-bit
//    shared load;
//  * multiplies with mma.sync m16n8k16 (bf16 in, float32 accumulate): weight
//    rows on the 16-row side, tokens on the 8-column side;
//  * multiplies each 64-input block's partial product by the block constant
//    (float32) instead of scaling every weight;
//  * spreads the (256-row block, 256-input chunk) units evenly over one CTA
//    per SM; each warp stores a float32 partial of every row block it
//    worked on, with no synchronisation, and the epilogue kernel sums a row
//    block's partials in a fixed order.
//
// T = s X A is computed by the same stream: the rows of A^T come first as
// extra row blocks (bf16, no block constant), so that their products with the
// X tiles already on chip are partials of T, which the last warp of each such
// row group sums.  A small kernel launched after the stream (programmatic
// dependent launch) writes Y = bf16(sum of partials + T B).
//
// Rounding.  A block's product is sum_k bf16(q_k) x_k (exact products,
// float32 sums) times the float32 constant a'_b; the other paths multiply by
// the dequantized weight bf16(fp32(q_k) a'_b).  Each form carries one bf16
// rounding of relative size <= 2^-9 per term against the exact q_k a'_b x_k.
#include <algorithm>
#include <atomic>
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

constexpr int kRows = 256;                  // weight rows per unit
constexpr int kKc = 256;                    // inputs per unit (4 blocks, 128 B of codes per row)
constexpr int kStages = 4;
constexpr int kCons = 16;                   // consumer warps: row group w & 7, block pair w >> 3
constexpr int kThreads = (kCons + 1) * 32;  // + one producer warp
constexpr int kCodeStage = kRows * kKc / 2;
constexpr int kMaxGridRd = 160;

template <int NT>
struct RdLayout {
  static constexpr int MP = 8 * NT;                        // tokens, padded
  static constexpr int kXStage = MP * kKc * 2;
  static constexpr int offCodes = 65536;                   // after the 64 KB level-pair table
  static constexpr int offX = offCodes + kStages * kCodeStage;
  static constexpr int offLvl = offX + kStages * kXStage;  // 256 float32 constant levels
  static constexpr int offBar = offLvl + 1024;
  static constexpr int offAbort = offBar + 2 * kStages * 8;
  static constexpr int kDynamic = offAbort + 16;
};
static_assert(RdLayout<2>::kDynamic <= 232448, "shared memory budget");

struct RdArgs {
  int M, N, K, KB, CH, RB, RBT, S2, r;
  int64_t U;             // units = RB * CH; row blocks 0 .. RBT-1 hold the rows of A^T (T = X A)
  int64_t n_scales;      // group scales in absmax_scale (the centred mean follows them)
  const uint8_t* absmax_q;
  const float* absmax_scale;
  float* partial;        // [RB][S2][256][MP] float32: one slot per (contributing CTA, block pair)
  float* T;              // [M x r] float32: T = s X A, finished by the last warp of each A^T row group
  int* tcnt;             // [RBT][2] arrival counters of those row groups
  float scale;
  int* status;
  uint64_t wait_ns;
  Nf4Params nf4;
};

// The dynamic shared window of a kernel without static shared memory starts
// at shared address kSmemBase (after the 1 KB each CTA reserves); the level
// table sits there, so a table offset formed by one byte permute is the
// load's register and the base its immediate.
constexpr uint32_t kSmemBase = 1024;
__device__ __forceinline__ uint32_t lds32_tab(uint32_t off) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1+1024];" : "=r"(v) : "r"(off));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
// D = A B (+ 0) and D += A B, m16n8k16, bf16 inputs, float32 accumulators.
__device__ __forceinline__ void mma_first(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ void mma_acc(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Schedule (identical on host and device): CTA j owns units
// [U j / G, U (j + 1) / G); unit u is (row block u / CH, chunk u % CH).
__host__ __device__ __forceinline__ int64_t unit_start(int j, int64_t U, int G) { return U * j / G; }
__host__ __device__ __forceinline__ int cta_of(int64_t u, int64_t U, int G) {
  return static_cast<int>(((u + 1) * G + U - 1) / U - 1);
}

// ---------------------------------------------------------------- weight stream
template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    smallm_rd_kernel(const __grid_constant__ CUtensorMap mapC, const __grid_constant__ CUtensorMap mapX,
                     const __grid_constant__ CUtensorMap mapA, const RdArgs a) {
  using L = RdLayout<NT>;
  constexpr int MP = L::MP;
  // The kernel has no static shared memory: the dynamic window starts at
  // shared address kSmemBase, aligned for the 128-byte-swizzled TMA tiles.
  extern __shared__ __align__(1024) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::offBar);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::offAbort);
  float* lvl2 = reinterpret_cast<float*>(sm + L::offLvl);
  if (smem_u32(sm) != kSmemBase) {  // table addressing and 1024-byte aligned swizzled copies rely on it
    if (tid == 0 && a.status) atomicCAS(a.status, 0, 0x100 + 62);
    return;
  }

  // Level-pair table: entry e (a code byte; the high nibble is the earlier
  // input) holds bf16(q[e >> 4]) in its low half and bf16(q[e & 15]) in its
  // high half; entry e, copy l sits at byte e * 256 + 4 l, so lane l always
  // reads bank l.  The upper 128 bytes of each 256-byte row stay unused.
  for (int i = tid; i < 256 * 32; i += kThreads) {
    const int e = i >> 5, l = i & 31;
    reinterpret_cast<uint32_t*>(sm)[e * 64 + l] = pack_bf16x2_rn(a.nf4.q[e >> 4], a.nf4.q[e & 15]);
  }
  for (int i = tid; i < 256; i += kThreads) lvl2[i] = level2_value_for(static_cast<uint32_t>(i), a.nf4.centred);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCons);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  griddep_launch_dependents();  // the epilogue kernel may get resident now; it waits for this grid

  const int G = gridDim.x, j = blockIdx.x;
  const int64_t u0 = unit_start(j, a.U, G), u1 = unit_start(j + 1, a.U, G);
  const int nu = static_cast<int>(u1 - u0);
  const int CH = a.CH;

  if (warp == kCons) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const WaitCtx ctx{abort_flag, a.status, 60, a.wait_ns};
      tma_prefetch_desc(&mapC);
      tma_prefetch_desc(&mapX);
      tma_prefetch_desc(&mapA);
      int rb = static_cast<int>(u0 / CH), ch = static_cast<int>(u0 % CH);
      int issued = 0;
      for (int i = 0; i < nu; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, ctx)) break;
        mbar_arrive_expect_tx(&full[s], kCodeStage + L::kXStage);
        if (rb >= a.RBT)
          tma_load_2d(&mapC, &full[s], sm + L::offCodes + s * kCodeStage, ch * 128, (rb - a.RBT) * kRows);
        else  // 64 columns of A x 256 inputs, bf16: the same 32 KB
          tma_load_2d(&mapA, &full[s], sm + L::offCodes + s * kCodeStage, 64 * rb, ch * kKc);
        tma_load_5d_outer(&mapX, &full[s], sm + L::offX + s * L::kXStage, 4 * ch);
        ++issued;
        if (++ch == CH) {
          ch = 0;
          ++rb;
        }
      }
      // After an abort nobody consumes the copies still in flight: they land
      // before the CTA exits.
      if (*abort_flag)
        for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
          mbar_drain(&full[i % kStages], (i / kStages) & 1);
    }
  } else {
    // ------------------------------------------------------------ consumers
    const WaitCtx ctx{abort_flag, a.status, 61, a.wait_ns};
    const int rg = warp & 7, kh = warp >> 3;
    const int g = lane >> 2, c = lane & 3;
    const uint32_t lane4 = static_cast<uint32_t>(lane) * 4u;
    const uint32_t codes0 = smem_u32(sm + L::offCodes), x0 = smem_u32(sm + L::offX);
    const int KB = a.KB;
    const float mu = centred_mu(a.absmax_scale, a.n_scales, a.nf4.centred);
    // Weight rows of a 16-row tile: fragment row g is row 2g, fragment row
    // g + 8 is row 2g + 1.  The 16 lanes of a half-warp then read their code
    // bytes from 8 different 16-byte chunk positions of the 128-byte-swizzled
    // tile (no bank conflict).  This lane loads the constants of row r_own
    // (t = c >> 1, h = c & 1) and hands them to the lanes that need them.
    const int r_own = 32 * rg + 16 * (c >> 1) + 2 * g + (c & 1);
    const bool vec16 = (KB & 15) == 0 && (reinterpret_cast<uintptr_t>(a.absmax_q) & 15u) == 0;
    // Raw 8-bit constants and the two group scales of 16 consecutive blocks.
    auto fetch = [&](int rbx, int gx, uint4& q, float (&sc)[2]) {
      q = make_uint4(0, 0, 0, 0);
      sc[0] = sc[1] = 0.0f;
      const int n = (rbx - a.RBT) * kRows + r_own;
      if (rbx < a.RBT || rbx >= a.RB || n >= a.N) return;
      const int64_t b0 = static_cast<int64_t>(n) * KB + 16 * gx;
      if (vec16) {
        q = __ldg(reinterpret_cast<const uint4*>(a.absmax_q + b0));
      } else {
        uint32_t w4[4] = {0, 0, 0, 0};
        for (int e = 0; e < 16 && 16 * gx + e < KB; ++e)
          w4[e >> 2] |= static_cast<uint32_t>(__ldg(a.absmax_q + b0 + e)) << (8 * (e & 3));
        q = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      const int64_t i0 = b0 >> 8;
      sc[0] = __ldg(a.absmax_scale + i0);
      sc[1] = __ldg(a.absmax_scale + (i0 + 1 < a.n_scales ? i0 + 1 : i0));
    };
    auto next_group = [&](int rbx, int gx, int& nrb, int& ng) {
      nrb = rbx;
      ng = gx + 1;
      if (ng * 4 >= CH) {
        ng = 0;
        ++nrb;
      }
    };
    int rb = static_cast<int>(u0 / CH), ch = static_cast<int>(u0 % CH);
    uint4 gq, gq_n;
    float gs[2], gs_n[2];
    fetch(rb, ch >> 2, gq, gs);
    {
      int nrb, ng;
      next_group(rb, ch >> 2, nrb, ng);
      fetch(nrb, ng, gq_n, gs_n);
    }
    float acc[2][NT][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][nt][e] = 0.0f;

    for (int i = 0; i < nu; ++i) {
      const int s = i % kStages;
      // Constants of this unit's two blocks for row r_own.
      float aown[2];
      {
        const int sb = (ch & 3) * 4 + 2 * kh;
        const uint32_t word = sb < 4 ? gq.x : sb < 8 ? gq.y : sb < 12 ? gq.z : gq.w;
        const int n = (rb - a.RBT) * kRows + r_own;  // negative in the A^T row blocks
        const bool wrow = rb >= a.RBT && n < a.N;
        const int64_t bl0 = static_cast<int64_t>(wrow ? n : 0) * KB + 16 * (ch >> 2);
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const uint32_t q = (word >> (8 * ((sb + bb) & 3))) & 255u;
          const float sc = ((bl0 + sb + bb) >> 8) == (bl0 >> 8) ? gs[0] : gs[1];
          const bool live = wrow && ch * 4 + 2 * kh + bb < KB;
          aown[bb] = live ? __fadd_rn(__fmul_rn(lvl2[q], sc), mu) : 0.0f;
        }
      }
      int nrb = rb, nch = ch + 1;
      if (nch == CH) {
        nch = 0;
        ++nrb;
      }
      if ((nch & 3) == 0) {  // the next unit starts the next group: rotate, fetch the one after
        gq = gq_n;
        gs[0] = gs_n[0];
        gs[1] = gs_n[1];
        int rr, ng;
        next_group(nrb, nch >> 2, rr, ng);
        fetch(rr, ng, gq_n, gs_n);
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (i / kStages) & 1, ctx))) break;

      const uint32_t cs = codes0 + s * kCodeStage, xs = x0 + s * L::kXStage;
      if (rb < a.RBT) {
        // Rows of A^T: the stage holds A[256 inputs][64 columns] bf16 with the
        // 128-byte swizzle.  One transposing matrix load gives a tile's
        // fragment: lane i addresses input row k(i) of 8x8 matrix i / 8 (rows
        // 2c + e <- inputs 16c + 4 s4 + e, +2 for matrices 2 and 3; columns
        // +8 for matrices 1 and 3), so lane (g, c) receives A^T rows j0 + g
        // (+8) at exactly the inputs its X fragment holds.  No block
        // constant.  Row groups 0 and 1 cover the 64 columns.
        if (rg < 2) {
          const int mq = lane >> 3, ii = lane & 7;
#pragma unroll
          for (int s4 = 0; s4 < 4; ++s4) {
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
              const int b = 2 * kh + bb;
              const int k = 64 * b + 16 * (ii >> 1) + 4 * s4 + (ii & 1) + 2 * (mq >> 1);
              uint32_t A[2][4];
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                const int chunk = 4 * rg + 2 * t + (mq & 1);
                const uint32_t addr = cs + k * 128 + (((chunk ^ (k & 7)) & 7) << 4);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(A[t][0]), "=r"(A[t][1]), "=r"(A[t][2]), "=r"(A[t][3])
                             : "r"(addr));
              }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const uint2 xb = lds64(xs + (((b * 2 + (s4 >> 1)) * MP + 8 * nt + g) * 4 + c) * 16 + 8 * (s4 & 1));
                mma_acc(acc[0][nt], A[0], xb.x, xb.y);
                mma_acc(acc[1][nt], A[1], xb.x, xb.y);
              }
            }
          }
        }
      } else {
      float av[2][2][2];  // [t][h][bb]
#pragma unroll
      for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int h = 0; h < 2; ++h) av[t][h][bb] = __shfl_sync(0xFFFFFFFFu, aown[bb], g * 4 + t * 2 + h);
      // This lane's 8 code bytes per (block, row): inputs 16c .. 16c + 15 of
      // the block; the 128-byte swizzle puts 16-byte chunk k of row r at k ^ (r & 7).
      uint2 w[2][2][2];  // [bb][t][h]
#pragma unroll
      for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int r = 32 * rg + 16 * t + 2 * g + h, b = 2 * kh + bb;
            w[bb][t][h] = lds64(cs + r * 128 + ((((2 * b + (c >> 1)) ^ r) & 7) << 4) + 8 * (c & 1));
          }
      float bl[2][2][NT][4];  // [bb][t][nt]
#pragma unroll
      for (int s4 = 0; s4 < 4; ++s4) {
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
          const int b = 2 * kh + bb;
          // MMA k-slots 2c, 2c+1 <- inputs 16c + 4 s4 + {0, 1} (code byte 2 s4),
          // slots 2c+8, 2c+9 <- inputs 16c + 4 s4 + {2, 3} (code byte 2 s4 + 1).
          const uint32_t j0 = (2 * s4) & 3;
          uint32_t A[2][4];
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t w0 = s4 < 2 ? w[bb][t][0].x : w[bb][t][0].y;
            const uint32_t w1 = s4 < 2 ? w[bb][t][1].x : w[bb][t][1].y;
            A[t][0] = lds32_tab(prmt(w0, lane4, 0x5504u | (j0 << 4)));
            A[t][1] = lds32_tab(prmt(w1, lane4, 0x5504u | (j0 << 4)));
            A[t][2] = lds32_tab(prmt(w0, lane4, 0x5504u | ((j0 + 1) << 4)));
            A[t][3] = lds32_tab(prmt(w1, lane4, 0x5504u | ((j0 + 1) << 4)));
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            // X tile layout [block][s4 / 2][token][c][8 inputs].
            const uint2 xb = lds64(xs + (((b * 2 + (s4 >> 1)) * MP + 8 * nt + g) * 4 + c) * 16 + 8 * (s4 & 1));
            if (s4 == 0) {
              mma_first(bl[bb][0][nt], A[0], xb.x, xb.y);
              mma_first(bl[bb][1][nt], A[1], xb.x, xb.y);
            } else {
              mma_acc(bl[bb][0][nt], A[0], xb.x, xb.y);
              mma_acc(bl[bb][1][nt], A[1], xb.x, xb.y);
            }
          }
        }
      }
      // Block constant times the block's partial product, two accumulators
      // (same row, two tokens) per packed float32 multiply-add.
#pragma unroll
      for (int bb = 0; bb < 2; ++bb)
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float2 a0 = make_float2(av[t][0][bb], av[t][0][bb]);
            const float2 a1 = make_float2(av[t][1][bb], av[t][1][bb]);
            const float2 r0 = __ffma2_rn(a0, make_float2(bl[bb][t][nt][0], bl[bb][t][nt][1]),
                                         make_float2(acc[t][nt][0], acc[t][nt][1]));
            const float2 r1 = __ffma2_rn(a1, make_float2(bl[bb][t][nt][2], bl[bb][t][nt][3]),
                                         make_float2(acc[t][nt][2], acc[t][nt][3]));
            acc[t][nt][0] = r0.x;
            acc[t][nt][1] = r0.y;
            acc[t][nt][2] = r1.x;
            acc[t][nt][3] = r1.y;
          }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      if (nrb != rb || i + 1 == nu) {
        // Row block rb ends here for this warp: store its part of row group
        // rg in the slot of (this CTA, block pair); the epilogue kernel sums
        // the slots of each row block in order.
        const int jf = cta_of(static_cast<int64_t>(rb) * CH, a.U, G);
        if (rb >= a.RBT || rg < 2) {
          const int slot = 2 * (j - jf) + kh;
          float* my = a.partial + ((static_cast<int64_t>(rb) * a.S2 + slot) * kRows + 32 * rg) * MP;
          // Rows of fragment rows g and g + 8 (A^T tiles keep the plain order).
          const bool tb = rb < a.RBT;
          const int r0 = tb ? g : 2 * g, r1 = tb ? g + 8 : 2 * g + 1;
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              *reinterpret_cast<float2*>(my + (16 * t + r0) * MP + 8 * nt + 2 * c) =
                  make_float2(acc[t][nt][0], acc[t][nt][1]);
              *reinterpret_cast<float2*>(my + (16 * t + r1) * MP + 8 * nt + 2 * c) =
                  make_float2(acc[t][nt][2], acc[t][nt][3]);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[t][nt][e] = 0.0f;
            }
          if (rb < a.RBT) {
            // A row group of A^T: the last of its 2 * (contributing CTAs)
            // warps sums the slots in order into T (once per call, by the
            // first CTAs of the grid, early in their ranges).
            const int jl = cta_of(static_cast<int64_t>(rb + 1) * CH - 1, a.U, G);
            const int nparts = 2 * (jl - jf + 1);
            __threadfence();
            __syncwarp();
            int old = 0;
            if (lane == 0) old = atomicAdd(a.tcnt + rb * 2 + rg, 1);
            old = __shfl_sync(0xFFFFFFFFu, old, 0);
            if (old == nparts - 1) {
              __threadfence();
              const float* base = a.partial + (static_cast<int64_t>(rb) * a.S2 * kRows + 32 * rg) * MP;
#pragma unroll
              for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int row = 16 * t + 8 * h + g, col = 64 * rb + 32 * rg + row;
#pragma unroll
                  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                      const int m = 8 * nt + 2 * c + e;
                      float v = 0.0f;
                      for (int p = 0; p < nparts; ++p)
                        v += __ldcg(base + (static_cast<int64_t>(p) * kRows + row) * MP + m);
                      if (m < a.M && col < a.r) a.T[static_cast<int64_t>(m) * a.r + col] = __fmul_rn(a.scale, v);
                    }
                }
              if (lane == 0) a.tcnt[rb * 2 + rg] = 0;
            }
          }
        }
      }
      rb = nrb;
      ch = nch;
    }
  }
}

// ---------------------------------------------------------------- Y = bf16(partials + T B)
// Warp: 8 adjacent outputs n (four pairs) of four tokens.  Lane (pair p,
// slice q) sums the partial slots q, q + 8, ... of the output's row block and
// ranks q r/8 .. (q + 1) r/8 - 1 of T B, then a fixed butterfly over the 8
// slices completes the sum.
struct UpArgs {
  int M, N, r, CH, G, S2, MP, RBT;
  int64_t U;
};

__global__ void __launch_bounds__(256) lora_up_kernel(const float* __restrict__ T, const uint16_t* __restrict__ B,
                                                      const float* __restrict__ partial, const UpArgs u,
                                                      uint16_t* __restrict__ Y) {
  const int lane = threadIdx.x & 31, q = lane & 7, p = lane >> 3;
  const int n = (blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * 8 + 2 * p;
  const int m0 = blockIdx.y * 4;
  const bool live = n < u.N;
  const int rs = u.r / 8;  // r is a multiple of 8, at most 128
  // B is an input of the call: read it before waiting for the stream.
  uint32_t bw[16];
#pragma unroll
  for (int e = 0; e < 16; ++e)
    bw[e] = live && e < rs ? __ldg(reinterpret_cast<const uint32_t*>(B + static_cast<int64_t>(q * rs + e) * u.N + n)) : 0u;
  griddep_wait();  // the weight stream (which also finished T) has completed
  // This CTA's four rows of T, staged once; the partial slots of Y are read
  // in the same round.
  __shared__ float Ts[4][128];
  for (int i = threadIdx.x; i < 4 * u.r; i += blockDim.x) {
    const int mm = i / u.r, jj = i % u.r;
    Ts[mm][jj] = m0 + mm < u.M ? __ldcg(T + static_cast<int64_t>(m0 + mm) * u.r + jj) : 0.0f;
  }
  float z[4][2];
#pragma unroll
  for (int mm = 0; mm < 4; ++mm) z[mm][0] = z[mm][1] = 0.0f;
  if (live) {
    const int rb = u.RBT + n / kRows, row = n % kRows;
    const int jf = cta_of(static_cast<int64_t>(rb) * u.CH, u.U, u.G);
    const int jl = cta_of(static_cast<int64_t>(rb + 1) * u.CH - 1, u.U, u.G);
    const int nparts = 2 * (jl - jf + 1);
    for (int s = q; s < nparts; s += 8) {
      const float* ps = partial + ((static_cast<int64_t>(rb) * u.S2 + s) * kRows + row) * u.MP + m0;
      const float4 v0 = __ldcg(reinterpret_cast<const float4*>(ps));
      const float4 v1 = __ldcg(reinterpret_cast<const float4*>(ps + u.MP));
      z[0][0] += v0.x; z[1][0] += v0.y; z[2][0] += v0.z; z[3][0] += v0.w;
      z[0][1] += v1.x; z[1][1] += v1.y; z[2][1] += v1.z; z[3][1] += v1.w;
    }
  }
  __syncthreads();
  if (live) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      if (e < rs) {
        const float b0 = __uint_as_float(bw[e] << 16), b1 = __uint_as_float(bw[e] & 0xFFFF0000u);
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) {
          const float t = Ts[mm][q * rs + e];
          z[mm][0] = fmaf(t, b0, z[mm][0]);
          z[mm][1] = fmaf(t, b1, z[mm][1]);
        }
      }
    }
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1)
#pragma unroll
    for (int mm = 0; mm < 4; ++mm) {
      z[mm][0] += __shfl_xor_sync(0xFFFFFFFFu, z[mm][0], o);
      z[mm][1] += __shfl_xor_sync(0xFFFFFFFFu, z[mm][1], o);
    }
  if (!live || q != 0) return;
#pragma unroll
  for (int mm = 0; mm < 4; ++mm) {
    const int m = m0 + mm;
    if (m < u.M) *reinterpret_cast<uint32_t*>(Y + static_cast<int64_t>(m) * u.N + n) = pack_bf16x2_rn(z[mm][0], z[mm][1]);
  }
}

struct RdPlan {
  int KB, CH, RB, RBT, G, S2, MP;
  int64_t U;
  size_t off_partial, off_tcnt, total;
};

size_t r256(size_t x) { return (x + 255) / 256 * 256; }

RdPlan rd_plan(int64_t M, int64_t K, int64_t N, int r, int sms) {
  RdPlan p{};
  p.KB = static_cast<int>(K / 64);
  p.CH = static_cast<int>((K + kKc - 1) / kKc);
  p.RBT = (r + 63) / 64;  // the rows of A^T, 64 per block, first
  p.RB = p.RBT + static_cast<int>((N + kRows - 1) / kRows);
  p.U = static_cast<int64_t>(p.RB) * p.CH;
  p.G = static_cast<int>(std::min<int64_t>({static_cast<int64_t>(sms), static_cast<int64_t>(kMaxGridRd), p.U}));
  // A row block spans at most ceil(CH / (U / G)) + 1 CTAs.
  const int64_t per = p.U / p.G;  // >= 1
  const int maxc = static_cast<int>(std::min<int64_t>(p.G, (p.CH + per - 1) / per + 1));
  p.S2 = 2 * maxc;
  p.MP = M <= 8 ? 8 : 16;
  size_t o = 0;
  p.off_partial = o;
  o += r256(static_cast<size_t>(p.RB) * p.S2 * kRows * p.MP * 4);
  p.off_tcnt = o;
  o += r256(static_cast<size_t>(p.RBT) * 2 * 4);
  p.total = o;
  return p;
}

template <int NT>
cudaError_t launch_rd_main(const CUtensorMap& mC, const CUtensorMap& mX, const CUtensorMap& mA, const RdArgs& args,
                           int grid, cudaStream_t stream) {
  using L = RdLayout<NT>;
  auto kern = smallm_rd_kernel<NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kDynamic);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kDynamic;
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, kern, mC, mX, mA, args);
}

}  // namespace

size_t small_m_rd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r) {
  // Sized for the largest grid any device here uses.
  return rd_plan(M, K, N, r, kMaxGridRd).total;
}

cudaError_t launch_small_m_rd(const uint16_t* X, const uint8_t* codes, const uint8_t* absmax_q,
                              const float* absmax_scale, const uint16_t* A, const uint16_t* B, int64_t M, int64_t K,
                              int64_t N, int r, float scale, uint16_t* Y, float* T_save, void* scratch, int* status,
                              const Nf4Params& P, cudaStream_t stream) {
  if (M < 1 || M > kSmallMRdMax || r > 128) return cudaErrorInvalidValue;
  const RdPlan p = rd_plan(M, K, N, r, device_sm_count());
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  CUtensorMap mC, mX, mA;
  if (!make_map_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 128, kRows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  // A [K x r] bf16 in tiles of 256 inputs x 64 columns (the A^T row blocks).
  if (!make_map_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, r, K, static_cast<int64_t>(r) * 2, 64, kKc,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  {
    // X viewed as [K/64 blocks][2][M tokens][4][8] bf16 (outermost first):
    // input k = 64 d4 + 16 d1 + 8 d3 + d0 of token d2.
    const uint64_t dims[5] = {8, 4, static_cast<uint64_t>(M), 2, static_cast<uint64_t>(K / 64)};
    const uint64_t strides[4] = {32, static_cast<uint64_t>(K) * 2, 16, 128};
    const uint32_t box[5] = {8, 4, static_cast<uint32_t>(p.MP), 2, 4};
    if (!make_map_nd(&mX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, 5, dims, strides, box)) return cudaErrorInvalidValue;
  }
  // The epilogue asks for the whole shared-memory carveout, as the stream
  // does: its CTAs then start on an SM as soon as the stream CTA leaves it.
  // A preference, set once per device (a failure only costs that overlap).
  {
    static std::atomic<uint64_t> carveout_set{0};
    int dev = 0;
    const bool known = cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64;
    const uint64_t bit = known ? (uint64_t(1) << dev) : 0;
    if (!known || !(carveout_set.load(std::memory_order_relaxed) & bit)) {
      if (cudaFuncSetAttribute(lora_up_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared) == cudaSuccess)
        carveout_set.fetch_or(bit, std::memory_order_relaxed);
      else
        cudaGetLastError();  // the preference is optional: drop its recorded error
    }
  }

  RdArgs args{};
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.KB = p.KB;
  args.CH = p.CH;
  args.RB = p.RB;
  args.RBT = p.RBT;
  args.r = r;
  args.T = T_save;
  args.tcnt = reinterpret_cast<int*>(ws + p.off_tcnt);
  args.scale = scale;
  args.S2 = p.S2;
  args.U = p.U;
  args.n_scales = (N * p.KB + 255) / 256;
  args.absmax_q = absmax_q;
  args.absmax_scale = absmax_scale;
  args.partial = reinterpret_cast<float*>(ws + p.off_partial);
  args.status = status;
  args.wait_ns = wait_limit_ns();
  args.nf4 = P;
  cudaError_t e = p.MP == 8 ? launch_rd_main<1>(mC, mX, mA, args, p.G, stream)
                            : launch_rd_main<2>(mC, mX, mA, args, p.G, stream);
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((N + 63) / 64), static_cast<unsigned>((M + 3) / 4), 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  UpArgs ua{};
  ua.M = static_cast<int>(M);
  ua.N = static_cast<int>(N);
  ua.r = r;
  ua.CH = p.CH;
  ua.G = p.G;
  ua.S2 = p.S2;
  ua.MP = p.MP;
  ua.RBT = p.RBT;
  ua.U = p.U;
  return cudaLaunchKernelEx(&cfg, lora_up_kernel, static_cast<const float*>(T_save), B,
                            static_cast<const float*>(args.partial), ua, Y);
}

}  // namespace qlora
