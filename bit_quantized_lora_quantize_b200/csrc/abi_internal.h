// Host-side helpers shared by the C-ABI entry points (abi.cu, noalloc.cu):
// argument checks, error recording and the optional per-launch timing.  Not
// part of the public header.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/qlora.h"

namespace qlora {

// Records the CUDA error string for qlora_last_cuda_error and returns
// QLORA_ERR_CUDA.
qlora_status cuda_fail(cudaError_t e);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape rules of the linear calls (include/qlora.h): QLORA_OK, or the status
// an unsupported or invalid shape returns.
qlora_status check_linear_shape(int64_t M, int64_t K, int64_t N, int32_t r);

// Optional per-launch timing: when qlora_profile_start is active, records a
// pair of CUDA events on the stream around the launches between construction
// and done().
struct ProfScope {
  bool on;
  cudaStream_t st;
  const char* name;
  int launches;
  cudaEvent_t a = nullptr;
  ProfScope(cudaStream_t s, const char* n, int l);
  void done();
};

}  // namespace qlora
