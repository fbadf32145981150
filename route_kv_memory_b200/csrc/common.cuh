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
