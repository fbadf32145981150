// CUDA-core pieces of the dense projections: the float32 FFMA GEMM (float32
// workloads, where tensor-core TF32 would break the float32 tolerance, and the
// one-time fold W_q W_r1), the shared epilogue store, and weight packing
// (transposes, bf16 hi/lo split).  The bf16 GEMM runs on tcgen05 (tc_gemm.cu).
#include "common.cuh"
#include "kernels.h"

namespace mka {

// ---------------------------------------------------------------- epilogue store
__device__ __forceinline__ void ep_store1(const Epilogue& ep, int m, int n, float v) {
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    if (s >= ep.nseg) break;
    const OutSeg& g = ep.seg[s];
    if (n >= g.n_begin && n < g.n_end) {
      size_t off = (size_t)m * g.ld + (n - g.n_begin);
      if (g.is_bf16) ((bf16*)g.ptr)[off] = __float2bfloat16_rn(v);
      else ((float*)g.ptr)[off] = v;
      return;
    }
  }
}

// Stores columns n and n+1 of row m (n+1 may fall in the next segment or past N).
__device__ __forceinline__ void ep_store2(const Epilogue& ep, int m, int n, float v0, float v1, int M, int N) {
  if (m >= M) return;
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    if (s >= ep.nseg) break;
    const OutSeg& g = ep.seg[s];
    if (n >= g.n_begin && n < g.n_end) {
      size_t off = (size_t)m * g.ld + (n - g.n_begin);
      if (n + 1 < g.n_end && (off & 1) == 0) {
        if (g.is_bf16) *(__nv_bfloat162*)((bf16*)g.ptr + off) = __floats2bfloat162_rn(v0, v1);
        else *(float2*)((float*)g.ptr + off) = make_float2(v0, v1);
        return;
      }
      if (g.is_bf16) ((bf16*)g.ptr)[off] = __float2bfloat16_rn(v0);
      else ((float*)g.ptr)[off] = v0;
      if (n + 1 < N) ep_store1(ep, m, n + 1, v1);
      return;
    }
  }
  if (n + 1 < N) ep_store1(ep, m, n + 1, v1);
}

// ---------------------------------------------------------------- FFMA GEMM (float32 workloads, weight folding)
namespace ff {
constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

template <typename TA, typename TB>
__global__ void __launch_bounds__(NT) gemm_tn_ffma_kernel(const TA* __restrict__ A, int lda, const TB* __restrict__ B,
                                                          int ldb, int M, int N, int K, Epilogue ep) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int e = tid + i * NT, r = e >> 4, kk = e & 15;
      int gm = m0 + r, gn = n0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < K) ? to_f<TA>(A[(size_t)gm * lda + gk]) : 0.f;
      Bs[kk][r] = (gn < N && gk < K) ? to_f<TB>(B[(size_t)gn * ldb + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
      if (n < N) ep_store2(ep, m, n, acc[i][j], acc[i][j + 1], M, N);
    }
}
}  // namespace ff

cudaError_t gemm_tn_ffma(const void* A, int lda, int a_bf16, const void* B, int ldb, int b_bf16, int M, int N, int K,
                         const Epilogue& ep, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + ff::BN - 1) / ff::BN, (M + ff::BM - 1) / ff::BM);
  if (a_bf16 && b_bf16)
    ff::gemm_tn_ffma_kernel<bf16, bf16><<<grid, ff::NT, 0, s>>>((const bf16*)A, lda, (const bf16*)B, ldb, M, N, K, ep);
  else if (!a_bf16 && !b_bf16)
    ff::gemm_tn_ffma_kernel<float, float><<<grid, ff::NT, 0, s>>>((const float*)A, lda, (const float*)B, ldb, M, N, K, ep);
  else if (a_bf16)
    ff::gemm_tn_ffma_kernel<bf16, float><<<grid, ff::NT, 0, s>>>((const bf16*)A, lda, (const float*)B, ldb, M, N, K, ep);
  else
    ff::gemm_tn_ffma_kernel<float, bf16><<<grid, ff::NT, 0, s>>>((const float*)A, lda, (const bf16*)B, ldb, M, N, K, ep);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- small packing kernels
template <typename Tin, typename Tout>
__global__ void transpose_kernel(const Tin* __restrict__ in, int rows, int cols, int ld_in, Tout* __restrict__ out,
                                 int ld_out) {
  __shared__ float tile[32][33];
  int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = to_f<Tin>(in[(size_t)r * ld_in + c]);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[(size_t)c * ld_out + r] = (Tout)tile[threadIdx.x][i];
  }
}
// bf16 -> bf16 transpose of 64 x 64 tiles with 16-byte loads and stores (rows, cols, ld_in, ld_out
// multiples of 8, both pointers 16-byte aligned); 256 threads.
__global__ void __launch_bounds__(256) transpose_bf16_v8_kernel(const bf16* __restrict__ in, int rows, int cols,
                                                                int ld_in, bf16* __restrict__ out, int ld_out) {
  __shared__ bf16 tile[64][64 + 8];
  const int c0 = blockIdx.x * 64, r0 = blockIdx.y * 64;
#pragma unroll
  for (int k = 0; k < 2; ++k) {  // 512 vectors of 8 elements
    const int v = threadIdx.x + 256 * k, r = v >> 3, c = (v & 7) * 8;
    if (r0 + r < rows && c0 + c < cols)
      *(uint4*)&tile[r][c] = *(const uint4*)(in + (size_t)(r0 + r) * ld_in + c0 + c);
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int v = threadIdx.x + 256 * k, oc = v >> 3, orow = (v & 7) * 8;  // out row c0 + oc, columns r0 + orow..+7
    if (c0 + oc < cols && r0 + orow < rows) {
      uint4 u;
      bf16* e = (bf16*)&u;
#pragma unroll
      for (int i = 0; i < 8; ++i) e[i] = tile[orow + i][oc];
      *(uint4*)(out + (size_t)(c0 + oc) * ld_out + r0 + orow) = u;
    }
  }
}
template <typename Tin>
__global__ void transpose_bf16_out_kernel(const Tin* __restrict__ in, int rows, int cols, int ld_in,
                                          bf16* __restrict__ out, int ld_out) {
  __shared__ float tile[32][33];
  int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = to_f<Tin>(in[(size_t)r * ld_in + c]);
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[(size_t)c * ld_out + r] = __float2bfloat16_rn(tile[threadIdx.x][i]);
  }
}

cudaError_t transpose(const void* in, int rows, int cols, int ld_in, void* out, int ld_out, int elem, int to_f64,
                      cudaStream_t s) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  if (to_f64) {
    if (elem == 2) transpose_kernel<bf16, double><<<grid, block, 0, s>>>((const bf16*)in, rows, cols, ld_in, (double*)out, ld_out);
    else transpose_kernel<float, double><<<grid, block, 0, s>>>((const float*)in, rows, cols, ld_in, (double*)out, ld_out);
  } else if (elem == 2 && rows % 8 == 0 && cols % 8 == 0 && ld_in % 8 == 0 && ld_out % 8 == 0 &&
             ((uintptr_t)in & 15) == 0 && ((uintptr_t)out & 15) == 0) {
    transpose_bf16_v8_kernel<<<dim3((cols + 63) / 64, (rows + 63) / 64), 256, 0, s>>>((const bf16*)in, rows, cols,
                                                                                      ld_in, (bf16*)out, ld_out);
  } else if (elem == 2) {
    transpose_bf16_out_kernel<bf16><<<grid, block, 0, s>>>((const bf16*)in, rows, cols, ld_in, (bf16*)out, ld_out);
  } else {
    transpose_kernel<float, float><<<grid, block, 0, s>>>((const float*)in, rows, cols, ld_in, (float*)out, ld_out);
  }
  return cudaGetLastError();
}

__global__ void split_hi_lo_kernel(const float* __restrict__ w, int n, bf16* __restrict__ hi, bf16* __restrict__ lo) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    float v = w[i];
    bf16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}
cudaError_t split_hi_lo(const float* w, int n, void* hi, void* lo, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  split_hi_lo_kernel<<<(n + 255) / 256, 256, 0, s>>>(w, n, (bf16*)hi, (bf16*)lo);
  return cudaGetLastError();
}

__global__ void split_hi_lo_interleaved_kernel(const float* __restrict__ w, int rh, int d, bf16* __restrict__ dst) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)rh * d) return;
  const int u = (int)(i / d), col = (int)(i % d);
  const float v = w[i];
  const bf16 h = __float2bfloat16_rn(v);
  const size_t row_hi = (size_t)(u / 128) * 256 + (u % 128);
  dst[row_hi * d + col] = h;
  dst[(row_hi + 128) * d + col] = __float2bfloat16_rn(v - __bfloat162float(h));
}
cudaError_t split_hi_lo_interleaved(const float* w, int rh, int d, void* dst, cudaStream_t s) {
  const size_t n = (size_t)rh * d;
  if (n == 0) return cudaSuccess;
  split_hi_lo_interleaved_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w, rh, d, (bf16*)dst);
  return cudaGetLastError();
}

template <typename T>
__global__ void widen_pad32_kernel(const T* __restrict__ in, int rows, int cols, double* __restrict__ out) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * 32) return;
  int r = i >> 5, c = i & 31;
  out[i] = c < cols ? (double)to_f<T>(in[(size_t)r * cols + c]) : 0.0;
}
cudaError_t widen_pad32_f64(const void* in, int rows, int cols, int in_bf16, double* out, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  int n = rows * 32;
  if (in_bf16) widen_pad32_kernel<bf16><<<(n + 255) / 256, 256, 0, s>>>((const bf16*)in, rows, cols, out);
  else widen_pad32_kernel<float><<<(n + 255) / 256, 256, 0, s>>>((const float*)in, rows, cols, out);
  return cudaGetLastError();
}

template <typename T>
__global__ void widen_kernel(const T* __restrict__ in, int n, float* __restrict__ out) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = to_f<T>(in[i]);
}
cudaError_t widen_f32(const void* in, int n, int in_bf16, float* out, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (in_bf16) widen_kernel<bf16><<<(n + 255) / 256, 256, 0, s>>>((const bf16*)in, n, out);
  else widen_kernel<float><<<(n + 255) / 256, 256, 0, s>>>((const float*)in, n, out);
  return cudaGetLastError();
}

}  // namespace mka
