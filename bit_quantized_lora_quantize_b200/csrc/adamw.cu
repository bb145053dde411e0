// Paged AdamW for the LoRA parameters.
//
// "QLoRA: Fine-Tuning 65-Billion Parameter Models on a Single Consumer GPU",
// "3. Paged Optimizers", and "AI Glossary: QLoRA", second paragraph: only the
// LoRA matrices are trained, and their optimizer states live in NVIDIA
// unified memory so that they can move between GPU and CPU memory when a
// memory spike needs the room.  Here the states (float32 master parameters,
// first and second moments) are allocated with cudaMallocManaged by
// qlora_paged_malloc; qlora_paged_prefetch moves them to the host before a
// spike and back to the GPU before the step; a step that finds them on the
// host still runs and pages them in on demand.
//
// The step is the textbook AdamW (decoupled weight decay, bias correction),
// one pass over the flattened parameters: 16 bytes read and 12 written per
// parameter (parameter, gradient, two moments), plus the bf16 copy of the
// updated parameter that the linear layer reads (2 bytes).  HBM-bound:
// 16-byte vector accesses, a grid of a few resident CTAs per SM striding over
// the vector.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/qlora.h"
#include "abi_internal.h"
#include "kernels.h"

namespace qlora {

namespace {

constexpr int kAdamThreads = 256;

struct AdamArgs {
  float lr, b1, b2, eps, wd;
  float inv_bc1, inv_bc2;  // 1 / (1 - b1^t), 1 / (1 - b2^t)
};

__device__ __forceinline__ float adam_update(float& p, float g, float& m, float& v, const AdamArgs& a) {
  m = a.b1 * m + (1.0f - a.b1) * g;
  v = a.b2 * v + (1.0f - a.b2) * (g * g);
  const float mh = m * a.inv_bc1;
  const float vh = v * a.inv_bc2;
  p = p - a.lr * (mh / (sqrtf(vh) + a.eps) + a.wd * p);
  return p;
}

__global__ void __launch_bounds__(kAdamThreads) adamw_kernel(float* __restrict__ p, uint16_t* __restrict__ pb,
                                                             const float* __restrict__ g, float* __restrict__ m,
                                                             float* __restrict__ v, int64_t n, int vec,
                                                             AdamArgs a) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (vec) {
    const int64_t n4 = n / 4;
    for (int64_t i = t0; i < n4; i += stride) {
      float4 pp = reinterpret_cast<float4*>(p)[i];
      const float4 gg = __ldcs(reinterpret_cast<const float4*>(g) + i);
      float4 mm = reinterpret_cast<float4*>(m)[i];
      float4 vv = reinterpret_cast<float4*>(v)[i];
      adam_update(pp.x, gg.x, mm.x, vv.x, a);
      adam_update(pp.y, gg.y, mm.y, vv.y, a);
      adam_update(pp.z, gg.z, mm.z, vv.z, a);
      adam_update(pp.w, gg.w, mm.w, vv.w, a);
      reinterpret_cast<float4*>(p)[i] = pp;
      reinterpret_cast<float4*>(m)[i] = mm;
      reinterpret_cast<float4*>(v)[i] = vv;
      if (pb) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(pp.x, pp.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(pp.z, pp.w);
        reinterpret_cast<uint2*>(pb)[i] =
            make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
      }
    }
    for (int64_t i = n4 * 4 + t0; i < n; i += stride) {
      float pp = p[i], mm = m[i], vv = v[i];
      adam_update(pp, g[i], mm, vv, a);
      p[i] = pp;
      m[i] = mm;
      v[i] = vv;
      if (pb) pb[i] = __bfloat16_as_ushort(__float2bfloat16_rn(pp));
    }
  } else {
    for (int64_t i = t0; i < n; i += stride) {
      float pp = p[i], mm = m[i], vv = v[i];
      adam_update(pp, g[i], mm, vv, a);
      p[i] = pp;
      m[i] = mm;
      v[i] = vv;
      if (pb) pb[i] = __bfloat16_as_ushort(__float2bfloat16_rn(pp));
    }
  }
}

int adam_grid(int64_t work) {
  const int64_t want = (work + kAdamThreads - 1) / kAdamThreads;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(device_sm_count()) * 8)));
}

}  // namespace

}  // namespace qlora

using namespace qlora;

extern "C" {

void* qlora_paged_malloc(size_t size, int device, void* stream) {
  (void)stream;
  int prev = 0;
  cudaError_t e = cudaGetDevice(&prev);
  if (e == cudaSuccess && device >= 0 && device != prev) e = cudaSetDevice(device);
  if (e != cudaSuccess) {
    cuda_fail(e);  // qlora_last_cuda_error says why the result is null
    return nullptr;
  }
  void* p = nullptr;
  e = cudaMallocManaged(&p, size > 0 ? size : 1, cudaMemAttachGlobal);
  if (device >= 0 && device != prev) cudaSetDevice(prev);
  if (e != cudaSuccess) {
    cuda_fail(e);
    return nullptr;
  }
  return p;
}

void qlora_paged_free(void* ptr, size_t size, int device, void* stream) {
  (void)size;
  (void)device;
  if (!ptr) return;
  // The memory may still be in use by work queued on `stream`.
  if (stream) cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  cudaFree(ptr);
}

qlora_status qlora_paged_prefetch(const void* ptr, size_t bytes, int32_t to_device, void* stream) {
  if (!ptr || bytes == 0) return QLORA_ERR_INVALID_ARG;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const int dst = to_device ? dev : cudaCpuDeviceId;
  e = cudaMemPrefetchAsync(ptr, bytes, dst, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

qlora_status qlora_paged_location(const void* ptr, size_t bytes, int32_t* location) {
  if (!ptr || bytes == 0 || !location) return QLORA_ERR_INVALID_ARG;
  int loc = 0;
  const cudaError_t e =
      cudaMemRangeGetAttribute(&loc, sizeof(loc), cudaMemRangeAttributeLastPrefetchLocation, ptr, bytes);
  if (e != cudaSuccess) return cuda_fail(e);
  *location = loc;
  return QLORA_OK;
}

qlora_status qlora_adamw_step(float* param, uint16_t* param_bf16, const float* grad, float* m, float* v, int64_t n,
                              int32_t step, float lr, float beta1, float beta2, float eps, float weight_decay,
                              void* stream) {
  if (!param || !grad || !m || !v || n <= 0 || step < 1) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(lr) || !std::isfinite(eps) || !std::isfinite(weight_decay) || !(beta1 >= 0.0f) ||
      !(beta1 < 1.0f) || !(beta2 >= 0.0f) || !(beta2 < 1.0f))
    return QLORA_ERR_INVALID_ARG;
  const auto al4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
  if (!al4(param) || !al4(grad) || !al4(m) || !al4(v) || (param_bf16 && (reinterpret_cast<uintptr_t>(param_bf16) & 1u)))
    return QLORA_ERR_ALIGNMENT;
  const bool vec = aligned16(param) && aligned16(grad) && aligned16(m) && aligned16(v) &&
                   (!param_bf16 || (reinterpret_cast<uintptr_t>(param_bf16) & 7u) == 0);
  AdamArgs a{};
  a.lr = lr;
  a.b1 = beta1;
  a.b2 = beta2;
  a.eps = eps;
  a.wd = weight_decay;
  // Bias corrections in double, once per step.
  a.inv_bc1 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(beta1), step)));
  a.inv_bc2 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(beta2), step)));
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope prof(st, "adamw_step", 1);
  adamw_kernel<<<adam_grid(vec ? n / 4 : n), kAdamThreads, 0, st>>>(param, param_bf16, grad, m, v, n, vec ? 1 : 0,
                                                                    a);
  const cudaError_t e = cudaGetLastError();
  prof.done();
  return e == cudaSuccess ? QLORA_OK : cuda_fail(e);
}

}  // extern "C"
