// C ABI of the library: argument validation, workspace layout and the
// sequence of kernel launches for each call (declared in include/qlora.h).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/qlora.h"
#include "abi_internal.h"
#include "kernels.h"
#include "nf4_host.h"
#include "tensor_map.h"

namespace qlora {

namespace {

thread_local std::string g_last_cuda_error;

// Limit of every bounded wait in the kernels (qlora_set_wait_timeout).
std::atomic<uint64_t> g_wait_ns{kWaitTimeoutNs};

constexpr size_t kStatusBytes = 256;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// The kernels take ranks that are multiples of 8 (the adapter rows are copied
// by TMA, whose row strides are multiples of 16 bytes); other ranks run with
// the adapter padded by zero columns to r8 in the workspace.
int rank8(int r) { return (r + 7) / 8 * 8; }

// The weight-streaming forward holds rank indices in one 128-row MMA tile.
bool small_m_path(int64_t M, int r) { return M <= kSmallMMax && rank8(r) <= 128; }

// Up to 8 tokens the forward decodes into register fragments of mma.sync
// (smallm_rd.cu), and up to 16 when the weight has 2^27 elements or more;
// otherwise, up to 128 tokens, into tensor memory (smallm.cu).  Measured at
// 16 tokens: 44.0 against 38.9 us for 8192 x 8192, 62.5 against 72.7 us for
// 22016 x 8192.
bool small_m_rd_path(int64_t M, int64_t K, int64_t N, int r) {
  if (rank8(r) > 128 || M > kSmallMRdMax) return false;
  return M <= 8 || N * K >= (int64_t(1) << 27);
}

// Workspace: [status word (256 B)][counters of the forward and input-gradient
// GEMMs][T pair: bf16 M x 2rp][U pair: bf16 M x 2rp]; when a small-M
// forward runs, [its counters, partials and float32 partial of Y]; when
// r % 8 != 0, [A, B, T, dA, dB padded to r8].
struct WsLayout {
  size_t cf_off, cd_off, t_off, u_off, sm_off, pad_off;
  size_t pa_off, pb_off, pt_off, pda_off, pdb_off, total;
};

WsLayout ws_layout(int64_t M, int64_t K, int64_t N, int r) {
  WsLayout w{};
  const int r8 = rank8(r);
  const size_t pair_bytes = round_up(static_cast<size_t>(M) * 2 * lora_pad(r8) * 2, 256);
  const size_t ctr_bytes = round_up(static_cast<size_t>(fused_ctr_ints(M)) * 4, 256);
  w.cf_off = kStatusBytes;
  w.cd_off = w.cf_off + ctr_bytes;
  w.t_off = w.cd_off + ctr_bytes;
  w.u_off = w.t_off + pair_bytes;
  w.sm_off = w.u_off + pair_bytes;
  size_t sm_bytes = 0;
  if (small_m_rd_path(M, K, N, r))
    sm_bytes = small_m_rd_workspace_bytes(M, K, N, r8);
  else if (small_m_path(M, r))
    sm_bytes = small_m_workspace_bytes(M, N, r8);
  w.pad_off = w.sm_off + round_up(sm_bytes, 256);
  size_t o = w.pad_off;
  if (r8 != r) {
    w.pa_off = o; o += round_up(static_cast<size_t>(K) * r8 * 2, 256);
    w.pb_off = o; o += round_up(static_cast<size_t>(r8) * N * 2, 256);
    w.pt_off = o; o += round_up(static_cast<size_t>(M) * r8 * 4, 256);
    w.pda_off = o; o += round_up(static_cast<size_t>(K) * r8 * 4, 256);
    w.pdb_off = o; o += round_up(static_cast<size_t>(r8) * N * 4, 256);
  }
  w.total = o;
  return w;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// ---------------------------------------------------------------- profiling
// Optional per-launch timing with CUDA events recorded on the caller's
// stream around each kernel (or kernel pair) of a call.  Off by default.
struct ProfRec {
  const char* name;
  int launches;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

// The levels and constant scheme of a qlora_code value (4-bit code in the
// low byte, QLORA_DQ_CENTRED_FP8 as a flag); false for an unknown value.
bool resolve_code(int32_t code, Nf4Params* P) {
  if (code & ~(0xFF | QLORA_DQ_CENTRED_FP8)) return false;
  const Nf4Params* base = code_params_or_null(code & 0xFF);
  if (!base) return false;
  *P = *base;
  P->centred = (code & QLORA_DQ_CENTRED_FP8) ? 1 : 0;
  return true;
}

qlora_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = cudaGetErrorString(e);
  return QLORA_ERR_CUDA;
}

qlora_status check_linear_shape(int64_t M, int64_t K, int64_t N, int32_t r) {
  if (M <= 0 || K <= 0 || N <= 0 || r <= 0) return QLORA_ERR_INVALID_ARG;
  if (M >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31)) return QLORA_ERR_UNSUPPORTED;
  if (K % 64 != 0 || N % 8 != 0 || r > 256) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_l2_bytes[kMaxDevices];

// Attribute `what` of the current device, read once per device; `fallback`
// when the device or the attribute cannot be read.
int cached_attribute(std::atomic<int>* cache, cudaDeviceAttr what, int fallback) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return fallback;
  int v = dev < kMaxDevices ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, what, dev) != cudaSuccess || v <= 0) return fallback;
  if (dev < kMaxDevices) cache[dev].store(v, std::memory_order_relaxed);
  return v;
}
}  // namespace

int device_sm_count() { return cached_attribute(g_sm_count, cudaDevAttrMultiProcessorCount, 148); }

int device_l2_bytes() { return cached_attribute(g_l2_bytes, cudaDevAttrL2CacheSize, 126 << 20); }

ProfScope::ProfScope(cudaStream_t s, const char* n, int l) : on(false), st(s), name(n), launches(l) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  on = g_prof_on;
  if (on) {
    a = prof_event();
    cudaEventRecord(a, st);
  }
}

void ProfScope::done() {
  if (!on) return;
  std::lock_guard<std::mutex> g(g_prof_mu);
  cudaEvent_t b = prof_event();
  cudaEventRecord(b, st);
  g_prof_recs.push_back({name, launches, a, b});
  on = false;
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner, int64_t rows,
                 int64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_bytes)};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_nd(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = static_cast<cuuint64_t>(dims[i]);
    b[i] = static_cast<cuuint32_t>(box[i]);
    e[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = static_cast<cuuint64_t>(strides_bytes[i]);
  return fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, b, e,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace qlora

using namespace qlora;

extern "C" {

qlora_status qlora_quantize_4bit(const uint16_t* W, int64_t numel, int32_t code, uint8_t* codes, uint8_t* absmax_q,
                                 float* absmax_scale, void* stream) {
  if (!W || !codes || !absmax_q || !absmax_scale || numel <= 0) return QLORA_ERR_INVALID_ARG;
  Nf4Params Pv;
  if (!resolve_code(code, &Pv)) return QLORA_ERR_INVALID_ARG;
  const Nf4Params* P = &Pv;
  if (!aligned16(W) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(absmax_scale) & 3u))
    return QLORA_ERR_ALIGNMENT;
  if (numel > (int64_t(1) << 46)) return QLORA_ERR_UNSUPPORTED;
  if (Pv.centred && numel > (int64_t(1) << 38)) return QLORA_ERR_UNSUPPORTED;  // the mean divides by NB < 2^32
  ProfScope p(static_cast<cudaStream_t>(stream), "quantize_nf4", Pv.centred ? 3 : 1);
  const cudaError_t e = launch_quantize_nf4(W, numel, codes, absmax_q, absmax_scale, *P,
                                            static_cast<cudaStream_t>(stream));
  p.done();
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

qlora_status qlora_quantize_nf4(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* absmax_q,
                                float* absmax_scale, void* stream) {
  return qlora_quantize_4bit(W, numel, QLORA_CODE_NF4, codes, absmax_q, absmax_scale, stream);
}

qlora_status qlora_dequantize_4bit(const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                                   int64_t numel, int32_t code, uint16_t* W_out, void* stream) {
  if (!codes || !absmax_q || !absmax_scale || !W_out || numel <= 0) return QLORA_ERR_INVALID_ARG;
  Nf4Params Pv;
  if (!resolve_code(code, &Pv)) return QLORA_ERR_INVALID_ARG;
  const Nf4Params* P = &Pv;
  if (!aligned16(codes) || !aligned16(W_out) || (reinterpret_cast<uintptr_t>(absmax_scale) & 3u))
    return QLORA_ERR_ALIGNMENT;
  if (numel > (int64_t(1) << 46)) return QLORA_ERR_UNSUPPORTED;
  ProfScope p(static_cast<cudaStream_t>(stream), "dequantize_nf4", 1);
  const cudaError_t e = launch_dequantize_nf4(codes, absmax_q, absmax_scale, numel, W_out, *P,
                                              static_cast<cudaStream_t>(stream));
  p.done();
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

qlora_status qlora_dequantize_nf4(const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                                  int64_t numel, uint16_t* W_out, void* stream) {
  return qlora_dequantize_4bit(codes, absmax_q, absmax_scale, numel, QLORA_CODE_NF4, W_out, stream);
}

size_t qlora_workspace_bytes(int64_t M, int64_t K, int64_t N, int32_t r) {
  if (check_linear_shape(M, K, N, r) != QLORA_OK) return 0;
  return ws_layout(M, K, N, r).total;
}

qlora_status qlora_linear_fwd_4bit(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* codes,
                                   const uint8_t* absmax_q, const float* absmax_scale, int32_t code,
                                   const uint16_t* A, const uint16_t* B, int32_t r, float scale, uint16_t* Y,
                                   float* T_save, void* workspace, size_t ws_bytes, void* stream) {
  if (!X || !codes || !absmax_q || !absmax_scale || !A || !B || !Y || !T_save) return QLORA_ERR_INVALID_ARG;
  Nf4Params Pv;
  if (!resolve_code(code, &Pv)) return QLORA_ERR_INVALID_ARG;
  const Nf4Params* Pc = &Pv;
  if (!std::isfinite(scale)) return QLORA_ERR_INVALID_ARG;
  const qlora_status sh = check_linear_shape(M, K, N, r);
  if (sh != QLORA_OK) return sh;
  if (!aligned16(X) || !aligned16(codes) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || !aligned16(T_save) ||
      (reinterpret_cast<uintptr_t>(absmax_scale) & 3u))
    return QLORA_ERR_ALIGNMENT;
  const WsLayout wl = ws_layout(M, K, N, r);
  if (!workspace || ws_bytes < wl.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Nf4Params& P = *Pc;

  uint16_t* Tpair = reinterpret_cast<uint16_t*>(ws + wl.t_off);
  const int r8 = rank8(r);
  const uint16_t* Ak = A;
  const uint16_t* Bk = B;
  float* Tk = T_save;
  if (r8 != r) {
    // The adapter padded with zero columns (A) and rows (B) to r8; T comes
    // back through a padded buffer.
    uint16_t* Ap = reinterpret_cast<uint16_t*>(ws + wl.pa_off);
    uint16_t* Bp = reinterpret_cast<uint16_t*>(ws + wl.pb_off);
    cudaError_t e = launch_pad_copy(A, K, r, r, Ap, r8, r8, 2, st);
    if (e == cudaSuccess) e = launch_pad_copy(B, r, N, N, Bp, N, N, 2, st, r8);
    if (e != cudaSuccess) return cuda_fail(e);
    Ak = Ap;
    Bk = Bp;
    Tk = reinterpret_cast<float*>(ws + wl.pt_off);
  }
  cudaError_t e;
  if (small_m_rd_path(M, K, N, r)) {
    // Three launches: T, the weight stream, Y = bf16(stream + T B).
    ProfScope p0(st, "small_m_nf4_fwd", 3);
    e = launch_small_m_rd(X, codes, absmax_q, absmax_scale, Ak, Bk, M, K, N, r8, scale, Y, Tk, ws + wl.sm_off, status,
                          P, st);
    p0.done();
  } else if (small_m_path(M, r)) {
    // One launch: T, its pair and Y.
    ProfScope p0(st, "small_m_nf4_fwd", 1);
    e = launch_small_m_fwd(X, codes, absmax_q, absmax_scale, Ak, Bk, M, K, N, r8, scale, Y, Tk, Tpair,
                           ws + wl.sm_off, status, P, st);
    p0.done();
  } else {
    // One launch: T = s X A (T_save and its pair) in the kernel's first
    // units, then the output tiles.
    ProfScope p2(st, "fused_nf4_fwd", 1);
    e = launch_fused_fwd(X, codes, absmax_q, absmax_scale, Tpair, Bk, M, K, N, r8, Y, status, P, st, Ak, Tk, scale,
                         reinterpret_cast<int*>(ws + wl.cf_off));
    p2.done();
  }
  if (e == cudaSuccess && r8 != r) e = launch_pad_copy(Tk, M, r8, r8, T_save, r, r, 4, st);
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

qlora_status qlora_linear_fwd(const uint16_t* X, int64_t M, int64_t K, int64_t N, const uint8_t* codes,
                              const uint8_t* absmax_q, const float* absmax_scale, const uint16_t* A,
                              const uint16_t* B, int32_t r, float scale, uint16_t* Y, float* T_save,
                              void* workspace, size_t ws_bytes, void* stream) {
  return qlora_linear_fwd_4bit(X, M, K, N, codes, absmax_q, absmax_scale, QLORA_CODE_NF4, A, B, r, scale, Y, T_save,
                               workspace, ws_bytes, stream);
}

qlora_status qlora_linear_bwd_4bit(const uint16_t* dY, const uint16_t* X, const float* T_save, int64_t M, int64_t K,
                                   int64_t N, const uint8_t* codes, const uint8_t* absmax_q,
                                   const float* absmax_scale, int32_t code, const uint16_t* A, const uint16_t* B,
                                   int32_t r, float scale, uint16_t* dX, float* dA, float* dB, void* workspace,
                                   size_t ws_bytes, void* stream) {
  if (!dY || !X || !T_save || !codes || !absmax_q || !absmax_scale || !A || !B || !dX || !dA || !dB)
    return QLORA_ERR_INVALID_ARG;
  Nf4Params Pv;
  if (!resolve_code(code, &Pv)) return QLORA_ERR_INVALID_ARG;
  const Nf4Params* Pc = &Pv;
  if (!std::isfinite(scale)) return QLORA_ERR_INVALID_ARG;
  const qlora_status sh = check_linear_shape(M, K, N, r);
  if (sh != QLORA_OK) return sh;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(T_save) || !aligned16(codes) || !aligned16(A) ||
      !aligned16(B) || !aligned16(dX) || !aligned16(dA) || !aligned16(dB) ||
      (reinterpret_cast<uintptr_t>(absmax_scale) & 3u))
    return QLORA_ERR_ALIGNMENT;
  const WsLayout wl = ws_layout(M, K, N, r);
  if (!workspace || ws_bytes < wl.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  uint16_t* Tpair = reinterpret_cast<uint16_t*>(ws + wl.t_off);
  uint16_t* Upair = reinterpret_cast<uint16_t*>(ws + wl.u_off);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Nf4Params& P = *Pc;

  const int r8 = rank8(r);
  const uint16_t* Ak = A;
  const uint16_t* Bk = B;
  const float* Tk = T_save;
  float* dAk = dA;
  float* dBk = dB;
  cudaError_t e = cudaSuccess;
  if (r8 != r) {
    uint16_t* Ap = reinterpret_cast<uint16_t*>(ws + wl.pa_off);
    uint16_t* Bp = reinterpret_cast<uint16_t*>(ws + wl.pb_off);
    float* Tp = reinterpret_cast<float*>(ws + wl.pt_off);
    e = launch_pad_copy(A, K, r, r, Ap, r8, r8, 2, st);
    if (e == cudaSuccess) e = launch_pad_copy(B, r, N, N, Bp, N, N, 2, st, r8);
    if (e == cudaSuccess) e = launch_pad_copy(T_save, M, r, r, Tp, r8, r8, 4, st);
    if (e != cudaSuccess) return cuda_fail(e);
    Ak = Ap;
    Bk = Bp;
    Tk = Tp;
    dAk = reinterpret_cast<float*>(ws + wl.pda_off);
    dBk = reinterpret_cast<float*>(ws + wl.pdb_off);
  }
  // One launch: U = s dY B^T (and the bf16 pair of T) in the first units,
  // the dX tiles, and dA = X^T U and dB = T^T dY in units that fill the SMs
  // the last wave of tiles leaves idle.
  ProfScope p2(st, "fused_nf4_dx", 1);
  e = launch_fused_dx(dY, codes, absmax_q, absmax_scale, Upair, Ak, M, K, N, r8, dX, status, P, st, Bk, scale,
                      reinterpret_cast<int*>(ws + wl.cd_off), X, Tk, Tpair, dAk, dBk);
  p2.done();
  if (e == cudaSuccess && r8 != r) {
    e = launch_pad_copy(dAk, K, r8, r8, dA, r, r, 4, st);
    if (e == cudaSuccess) e = launch_pad_copy(dBk, r, N, N, dB, N, N, 4, st);
  }
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

qlora_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, const float* T_save, int64_t M, int64_t K,
                              int64_t N, const uint8_t* codes, const uint8_t* absmax_q, const float* absmax_scale,
                              const uint16_t* A, const uint16_t* B, int32_t r, float scale, uint16_t* dX, float* dA,
                              float* dB, void* workspace, size_t ws_bytes, void* stream) {
  return qlora_linear_bwd_4bit(dY, X, T_save, M, K, N, codes, absmax_q, absmax_scale, QLORA_CODE_NF4, A, B, r, scale,
                               dX, dA, dB, workspace, ws_bytes, stream);
}

qlora_status qlora_silu_gate_fwd(const uint16_t* G, const uint16_t* U, uint16_t* H, int64_t n, void* stream) {
  if (!G || !U || !H || n <= 0) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(U) || !aligned16(H)) return QLORA_ERR_ALIGNMENT;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope p(st, "silu_gate_fwd", 1);
  const cudaError_t e = launch_silu_gate_fwd(G, U, H, n, st);
  p.done();
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

qlora_status qlora_silu_gate_bwd(const uint16_t* G, const uint16_t* U, const uint16_t* dH, uint16_t* dG,
                                 uint16_t* dU, int64_t n, void* stream) {
  if (!G || !U || !dH || !dG || !dU || n <= 0) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(G) || !aligned16(U) || !aligned16(dH) || !aligned16(dG) || !aligned16(dU)) return QLORA_ERR_ALIGNMENT;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope p(st, "silu_gate_bwd", 1);
  const cudaError_t e = launch_silu_gate_bwd(G, U, dH, dG, dU, n, st);
  p.done();
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

qlora_status qlora_check_status(void* workspace, void* stream) {
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  bool timed_out = false;
  if (workspace) {
    int word = 0;
    e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    if (word != 0) {
      timed_out = true;
      e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
      if (e == cudaSuccess) e = cudaStreamSynchronize(st);
      if (e != cudaSuccess) return cuda_fail(e);
    }
  }
  // The status words inside the library (quantization, allocation-free
  // forward) on the current device.
  int word = 0;
  e = codec_status_take(st, &word);
  if (e != cudaSuccess) return cuda_fail(e);
  timed_out |= word != 0;
  e = noalloc_status_take(st, &word);
  if (e != cudaSuccess) return cuda_fail(e);
  timed_out |= word != 0;
  return timed_out ? QLORA_ERR_TIMEOUT : QLORA_OK;
}

qlora_status qlora_set_wait_timeout(uint64_t timeout_ns) {
  if (timeout_ns > kMaxWaitTimeoutNs) return QLORA_ERR_INVALID_ARG;
  g_wait_ns.store(timeout_ns == 0 ? kWaitTimeoutNs : timeout_ns, std::memory_order_relaxed);
  return QLORA_OK;
}

uint64_t qlora_get_wait_timeout(void) { return wait_limit_ns(); }

void qlora_nf4_codebook(float out[16]) {
  if (!out) return;
  const Nf4Params& P = nf4_params();
  std::memcpy(out, P.q, sizeof(P.q));
}

qlora_status qlora_codebook(int32_t code, float out[16]) {
  const Nf4Params* P = code_params_or_null(code & ~QLORA_DQ_CENTRED_FP8);
  if (!P || !out) return QLORA_ERR_INVALID_ARG;
  std::memcpy(out, P->q, sizeof(P->q));
  return QLORA_OK;
}

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case QLORA_ERR_UNSUPPORTED: return "unsupported shape";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "kernel pipeline wait timed out";
  }
  return "unknown status";
}

const char* qlora_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

void qlora_profile_start(void) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  for (auto& r : g_prof_recs) {
    g_prof_pool.push_back(r.a);
    g_prof_pool.push_back(r.b);
  }
  g_prof_recs.clear();
  g_prof_on = true;
}

int qlora_profile_stop(int max_entries, char* names, float* total_ms, int* calls, int* launches) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = false;
  std::map<std::string, std::pair<double, std::pair<int, int>>> agg;
  for (auto& r : g_prof_recs) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      auto& e = agg[r.name];
      e.first += ms;
      e.second.first += 1;
      e.second.second += r.launches;
    }
    g_prof_pool.push_back(r.a);
    g_prof_pool.push_back(r.b);
  }
  g_prof_recs.clear();
  int n = 0;
  for (auto& kv : agg) {
    if (n >= max_entries) break;
    if (names) {
      std::strncpy(names + 48 * n, kv.first.c_str(), 47);
      names[48 * n + 47] = 0;
    }
    if (total_ms) total_ms[n] = static_cast<float>(kv.second.first);
    if (calls) calls[n] = kv.second.second.first;
    if (launches) launches[n] = kv.second.second.second;
    ++n;
  }
  return n;
}

}  // extern "C"
