// Forward of the LoRA linear layer for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: code that
// runs where the allocator must not be touched (inside a memory-pool or
// allocator callback, under a framework that forbids allocation on its hot
// path, or in an embedding that owns all device memory up front).  They can
// still pass their own inputs and outputs, but not the workspace that
// qlora_linear_fwd needs.  qlora_linear_fwd_noalloc gives them the same
// forward with its scratch taken from one fixed array in this file instead.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes; every
// GPU that loads this library keeps it for the life of the process.  Host
// code cannot use the array's name as a device address, so the first call on
// each device (with that device current) asks the runtime for the address
// with cudaGetSymbolAddress and keeps it; that first call should therefore
// come before any stream capture on that device.  All calls on a device share
// the array and it keeps the previous call's contents: each call clears the
// counters it needs at zero and overwrites everything else it reads, and
// calls that overlap on the GPU (different streams, or different host threads
// without ordering) race on it.  The first 256 bytes hold the status word: a
// pipeline wait that gave up sets it, and qlora_check_status reports and
// clears it (calls leave it alone, so a timeout stays visible until then).
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/qlora.h"
#include "abi_internal.h"
#include "kernels.h"
#include "nf4_host.h"

namespace qlora {

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;
constexpr size_t kStatusBytes = 256;

__device__ __align__(256) unsigned char g_fwd_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices] = {};

size_t round_up256(size_t v) { return (v + 255) / 256 * 256; }

// Device address of the scratch array on the current device (set up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fwd_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

cudaError_t noalloc_status_take(cudaStream_t stream, int* word) {
  *word = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> g(g_setup_mu);
    if (dev >= 0 && dev < kMaxDevices) base = g_scratch_ptr[dev];
  }
  if (!base) return cudaSuccess;  // no allocation-free call ran on this device
  e = cudaMemcpyAsync(word, base, sizeof(int), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && *word != 0) {
    e = cudaMemsetAsync(base, 0, sizeof(int), stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  }
  return e;
}

}  // namespace qlora

using namespace qlora;

extern "C" qlora_status qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, int64_t K, int64_t N,
                                                 const uint8_t* codes, const uint8_t* absmax_q,
                                                 const float* absmax_scale, const uint16_t* A, const uint16_t* B,
                                                 int32_t r, float scale, uint16_t* Y, float* T_save, void* stream) {
  if (!X || !codes || !absmax_q || !absmax_scale || !A || !B || !Y || !T_save) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return QLORA_ERR_INVALID_ARG;
  const qlora_status sh = check_linear_shape(M, K, N, r);
  if (sh != QLORA_OK) return sh;
  if (r % 8 != 0) return QLORA_ERR_UNSUPPORTED;  // no room for the padded adapter here
  if (!aligned16(X) || !aligned16(codes) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || !aligned16(T_save) ||
      (reinterpret_cast<uintptr_t>(absmax_scale) & 3u))
    return QLORA_ERR_ALIGNMENT;

  // Scratch layout: [status word][counters of the GEMM launch][T pair: bf16 M x 2rp].
  const size_t ctr_bytes = round_up256(static_cast<size_t>(fused_ctr_ints(M)) * 4);
  const size_t pair_bytes = round_up256(static_cast<size_t>(M) * 2 * lora_pad(r) * 2);
  if (kStatusBytes + ctr_bytes + pair_bytes > kNoAllocScratchBytes) return QLORA_ERR_WORKSPACE;

  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned char* ws = static_cast<unsigned char*>(base);
  int* status = reinterpret_cast<int*>(ws);
  int* ctr = reinterpret_cast<int*>(ws + kStatusBytes);
  uint16_t* Tpair = reinterpret_cast<uint16_t*>(ws + kStatusBytes + ctr_bytes);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);

  // Clear the counters (a call that timed out earlier may have left them
  // set), then the one GEMM launch: T = s X A in its first units, then the
  // output tiles.  For every M this is the pair GEMM of the large-M forward.
  e = cudaMemsetAsync(ctr, 0, ctr_bytes, st);
  if (e != cudaSuccess) return cuda_fail(e);
  ProfScope p(st, "fused_nf4_fwd", 1);
  e = launch_fused_fwd(X, codes, absmax_q, absmax_scale, Tpair, B, M, K, N, r, Y, status, nf4_params(), st, A,
                       T_save, scale, ctr);
  p.done();
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}
