// Shared device helpers for the FastMKA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mka {

using bf16 = __nv_bfloat16;

// Device status codes (mirror mka_status_t in mka.h).
constexpr int kStatusOk = 0;
constexpr int kStatusCapacity = -4;
constexpr int kStatusTimeout = -5;
constexpr int kStatusBounds = -6;

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// The status block every kernel receives (16 bytes, 16-byte aligned): word 0 is the device
// status code above; word 1 a mask of the wait classes that take the limit in words 2-3 (an
// unsigned 64-bit count of nanoseconds; 0 = none) in place of their built-in limit.  Only the
// host writes words 1-3, and only while no kernel of the library runs.
constexpr int kWaitPipeline = 1;  // mbarrier waits of the TMA / tensor-core pipelines
constexpr int kWaitGrid = 2;      // grid barriers of the cooperative decode step
__device__ __forceinline__ unsigned long long wait_limit(const int* status, int wait_class,
                                                         unsigned long long builtin_ns) {
  if (!status || !(status[1] & wait_class)) return builtin_ns;
  const unsigned long long o = *(const unsigned long long*)(status + 2);
  return o ? o : builtin_ns;
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

template <typename T> __device__ __forceinline__ double to_d(T v) { return (double)to_f<T>(v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// GELU(x) = x * Phi(x), Phi(x) = 0.5 * erfc(-x / sqrt(2)).
__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * erfcf(-x * 0.70710678118654752f); }

// Routing gate over the three memory sources from the router logits (notes §2), with the
// routing variant and the active tiers of the layer configuration (abstract page, Tables 9
// and 10).  mode: 0 soft = softmax over the active tiers; 1 fixed = equal weights over them;
// 2 top-1 = all weight on the largest active logit; 3 top-2 = softmax over the two largest
// active logits.  Ties go to the lower tier index.  tiers: bit 0 L1, bit 1 L2, bit 2 L3
// (never 0 here).  Inactive tiers get 0.
__device__ __forceinline__ void route_gate(float z0, float z1, float z2, int mode, int tiers, float* l) {
  const float z[3] = {z0, z1, z2};
  int i1 = -1, i2 = -1, n = 0;  // the two largest active logits, in (value desc, index asc) order
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    if (!((tiers >> i) & 1)) continue;
    ++n;
    if (i1 < 0 || z[i] > z[i1]) {
      i2 = i1;
      i1 = i;
    } else if (i2 < 0 || z[i] > z[i2]) {
      i2 = i;
    }
  }
  l[0] = l[1] = l[2] = 0.f;
  if (mode == 1) {
    const float w = 1.f / (float)n;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      if ((tiers >> i) & 1) l[i] = w;
  } else if (mode == 2 || (mode == 3 && i2 < 0)) {
    l[i1] = 1.f;
  } else if (mode == 3) {
    const float e = expf(z[i2] - z[i1]);
    const float inv = 1.f / (1.f + e);
    l[i1] = inv;
    l[i2] = e * inv;
  } else {
    const float m = z[i1];
    float e[3], sum = 0.f;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      e[i] = ((tiers >> i) & 1) ? expf(z[i] - m) : 0.f;
      sum += e[i];
    }
    const float inv = 1.f / sum;
#pragma unroll
    for (int i = 0; i < 3; ++i) l[i] = e[i] * inv;
  }
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Raise a kernel's dynamic shared memory limit.  Skipped while `s` is being
// captured into a CUDA graph: the attribute persists, and an eager call made
// before the capture has already set it.
template <typename F>
inline cudaError_t set_max_smem(F* func, size_t bytes, cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) == cudaSuccess && st != cudaStreamCaptureStatusNone) return cudaSuccess;
  return cudaFuncSetAttribute((const void*)func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace mka
