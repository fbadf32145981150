// Router tail, L2 session EMA, L3 long-term recall and the route-fuse of the
// FastMKA layer ("MKA: Memory-Keyed Attention for Efficient Long-Context
// Reasoning", paper-notes page §1-§3).  All bandwidth-bound: float4 row
// streaming, warp-level reductions, per-block parallel scans.
//
// Projected space: K = X_fused W_k = l1 (X W_k) + l2 (M2 W_k) + l3 (M3 W_k), and
// both M2 (an EMA) and M3 (a mean of block means) commute with the projection,
// so the session and long-term memories run on the 2*dkv projected columns of
// each token instead of its d_model columns.
#include "common.cuh"
#include "kernels.h"

namespace mka {

// ---------------------------------------------------------------- router tail
// lambda = softmax(GELU(h) W_r2) per token (notes §2); h = h1 (+ h2) when the
// first layer was applied as a bf16 hi/lo pair.
__global__ void router_tail_kernel(const float* __restrict__ h1, const float* __restrict__ h2, int ldh, int T, int rh,
                                   const float* __restrict__ w_r2, int mode, int tiers, float* __restrict__ lam) {
  extern __shared__ float sw[];
  for (int i = threadIdx.x; i < rh * 3; i += blockDim.x) sw[i] = w_r2[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  float z0 = 0.f, z1 = 0.f, z2 = 0.f;
  const float* a = h1 + (size_t)t * ldh;
  const float* b = h2 ? h2 + (size_t)t * ldh : nullptr;
  for (int j = lane; j < rh; j += 32) {
    float h = a[j];
    if (b) h += b[j];
    float g = gelu_erf(h);
    z0 = fmaf(g, sw[j * 3 + 0], z0);
    z1 = fmaf(g, sw[j * 3 + 1], z1);
    z2 = fmaf(g, sw[j * 3 + 2], z2);
  }
  z0 = warp_sum(z0);
  z1 = warp_sum(z1);
  z2 = warp_sum(z2);
  if (lane == 0) {
    float l[3];
    route_gate(z0, z1, z2, mode, tiers, l);
    lam[(size_t)t * 3 + 0] = l[0];
    lam[(size_t)t * 3 + 1] = l[1];
    lam[(size_t)t * 3 + 2] = l[2];
  }
}

cudaError_t router_tail(const float* h1, const float* h2, int ldh, int T, int rh, const float* w_r2, int mode,
                        int tiers, float* lam, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  router_tail_kernel<<<(T + 7) / 8, 256, rh * 3 * sizeof(float), s>>>(h1, h2, ldh, T, rh, w_r2, mode, tiers, lam);
  return cudaGetLastError();
}

template <typename T> struct Vec4;
template <> struct Vec4<float> {
  static __device__ __forceinline__ float4 load(const float* p) { return *(const float4*)p; }
};
template <> struct Vec4<bf16> {
  static __device__ __forceinline__ float4 load(const bf16* p) {
    uint2 u = *(const uint2*)p;
    __nv_bfloat162 a = *(__nv_bfloat162*)&u.x, b = *(__nv_bfloat162*)&u.y;
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
};
__global__ void router_softmax_kernel(const float* __restrict__ zpart, int nparts, int T, int mode, int tiers,
                                      float* __restrict__ lam) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float z0 = 0.f, z1 = 0.f, z2 = 0.f;
  for (int r = 0; r < nparts; ++r) {
    const float4 v = *(const float4*)(zpart + ((size_t)r * T + t) * 4);
    z0 += v.x;
    z1 += v.y;
    z2 += v.z;
  }
  float l[3];
  route_gate(z0, z1, z2, mode, tiers, l);
  lam[(size_t)t * 3 + 0] = l[0];
  lam[(size_t)t * 3 + 1] = l[1];
  lam[(size_t)t * 3 + 2] = l[2];
}

cudaError_t router_softmax(const float* zpart, int nparts, int T, int mode, int tiers, float* lam, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  router_softmax_kernel<<<(T + 255) / 256, 256, 0, s>>>(zpart, nparts, T, mode, tiers, lam);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- L3 sign codes
// The float32 projection p = x . P_k (a tensor-core or FFMA dot product of
// length K) carries a rounding error below about K/16 * 2^-23 * |partial sum|
// per step-accumulation, i.e. under K * 2^-23 * rms_k(p) for partial sums of a
// few standard deviations (rms_k(p) estimates that scale).  Signs of
// projections within eps = K * 2^-21 * rms_k(p) of zero (a 4x margin) are
// decided again from an exact float64 dot product, so every code bit equals
// the sign of the exact projection.
template <typename T>
__device__ __forceinline__ double dot_row_f64(const T* __restrict__ x, const double* __restrict__ p, int d, int lane) {
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
  int i = lane * 4;
  for (; i + 3 < d; i += 128) {  // d is a multiple of 64: each lane takes 4 consecutive elements
    float4 v = Vec4<T>::load(x + i);
    const double2 p01 = *(const double2*)(p + i), p23 = *(const double2*)(p + i + 2);
    a0 = fma((double)v.x, p01.x, a0);
    a1 = fma((double)v.y, p01.y, a1);
    a2 = fma((double)v.z, p23.x, a2);
    a3 = fma((double)v.w, p23.y, a3);
  }
  return warp_sum_d((a0 + a1) + (a2 + a3));
}

template <typename T>
__global__ void token_codes_kernel(HashArgs a, int T_, uint32_t* __restrict__ codes) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T_) return;
  float p = lane < a.nb ? a.proj[(size_t)t * a.ldp + lane] : 0.f;
  float rms = sqrtf(warp_sum(p * p) / (float)a.nb);
  float e = (float)a.K * 0x1p-21f * rms;
  bool bit = p > 0.f;
  unsigned doubt = __ballot_sync(0xffffffffu, lane < a.nb && fabsf(p) <= e);
  const T* xr = (const T*)a.x + (size_t)t * a.d;
  while (doubt) {
    int k = __ffs(doubt) - 1;
    doubt &= doubt - 1;
    double v = dot_row_f64<T>(xr, a.pT64 + (size_t)k * a.d, a.d, lane);
    if (lane == k) bit = v > 0.0;
  }
  unsigned code = __ballot_sync(0xffffffffu, bit && lane < a.nb);
  if (lane == 0) codes[t] = code;
}

cudaError_t token_codes(const HashArgs& a, int T, uint32_t* codes, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (a.x_bf16) token_codes_kernel<bf16><<<(T + 7) / 8, 256, 0, s>>>(a, T, codes);
  else token_codes_kernel<float><<<(T + 7) / 8, 256, 0, s>>>(a, T, codes);
  return cudaGetLastError();
}

// Block codes.  The code of block j is the sign pattern of (sum of its rows) P,
// the same signs as (block mean) P.  Both are formed in float64 from the exact
// inputs: the block's column sums in d_model space (sums of at most a few
// hundred bf16 or float32 values), then dot products with P.  No float32
// rounding enters the decision.
//
// Pass 1: CTA (64-column chunk c, sequence b, group of blocks).  For each block it
// sums the block's rows over the chunk (16 row groups x 16 four-column threads),
// then 32 x 8 threads form the 64-long partial dot products with P's chunk.
// Pass 2: per block and bit, the partials are summed over the chunks in order.
constexpr int kXChunk = 64;
#ifndef MKA_BP_UNROLL
#define MKA_BP_UNROLL 4
#endif
constexpr int kBpUnroll = MKA_BP_UNROLL;

template <typename T>
__global__ void __launch_bounds__(256) block_proj_partial_kernel(const T* __restrict__ x, int d, int S, int blk,
                                                                  int nblk, int blocks_per_group,
                                                                  const double* __restrict__ P64, int nb,
                                                                  double* __restrict__ part) {
  __shared__ double Ps[kXChunk][33];
  __shared__ double xs[16][kXChunk];
  __shared__ double xt[kXChunk];
  const int chunk = blockIdx.x, nchunk = gridDim.x, bi = blockIdx.y;
  const int c0 = chunk * kXChunk;
  const int tid = threadIdx.x;
  for (int i = tid; i < kXChunk * 32; i += 256) {
    int c = i >> 5, k = i & 31;
    Ps[c][k] = (k < nb && c0 + c < d) ? P64[(size_t)(c0 + c) * 32 + k] : 0.0;
  }
  const int cq = tid & 15, rg = tid >> 4;
  const int col = c0 + cq * 4;
  const int per = (blk + 15) / 16;
  const int ra = min(rg * per, blk), rb = min(ra + per, blk);
  const int j0 = blockIdx.z * blocks_per_group, j1 = min(nblk, j0 + blocks_per_group);
  const int k = tid >> 3, sub = tid & 7;
  for (int j = j0; j < j1; ++j) {
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    if (col < d) {
      const T* p = x + ((size_t)bi * S + (size_t)j * blk) * d + col;
#pragma unroll kBpUnroll
      for (int r = ra; r < rb; ++r) {
        float4 v = Vec4<T>::load(p + (size_t)r * d);
        a0 += v.x;
        a1 += v.y;
        a2 += v.z;
        a3 += v.w;
      }
    }
    xs[rg][cq * 4 + 0] = a0;
    xs[rg][cq * 4 + 1] = a1;
    xs[rg][cq * 4 + 2] = a2;
    xs[rg][cq * 4 + 3] = a3;
    __syncthreads();
    if (tid < kXChunk) {
      double t = 0.0;
#pragma unroll
      for (int g = 0; g < 16; ++g) t += xs[g][tid];
      xt[tid] = t;
    }
    __syncthreads();
    double v = 0.0;
#pragma unroll
    for (int c = sub; c < kXChunk; c += 8) v = fma(xt[c], Ps[c][k], v);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (sub == 0) part[(((size_t)bi * nblk + j) * nchunk + chunk) * 32 + k] = v;
    __syncthreads();
  }
}

__global__ void block_codes_kernel(const double* __restrict__ part, int nchunk, int nb, int nblk,
                                   uint32_t* __restrict__ codes, int code_bstride) {
  const int j = blockIdx.x, bi = blockIdx.y, lane = threadIdx.x;
  const double* p = part + ((size_t)bi * nblk + j) * nchunk * 32 + lane;
  double v = 0.0;
  for (int c = 0; c < nchunk; ++c) v += p[(size_t)c * 32];
  unsigned code = __ballot_sync(0xffffffffu, lane < nb && v > 0.0);
  if (lane == 0) codes[(size_t)bi * code_bstride + j] = code;
}

size_t summary_codes_scratch(int d, int B, int nblk) {
  return (size_t)B * nblk * ((d + kXChunk - 1) / kXChunk) * 32 * sizeof(double);
}

cudaError_t summary_codes(const void* x, int x_bf16, int d, int B, int S, int nblk, int blk, const double* P64,
                          int nb, double* part, uint32_t* codes, int code_bstride, cudaStream_t s) {
  if (B <= 0 || nblk <= 0) return cudaSuccess;
  const int nchunk = (d + kXChunk - 1) / kXChunk;
  // enough CTAs to stream X at full bandwidth: about MKA_BP_WAVES waves over the SMs
#ifndef MKA_BP_WAVES
#define MKA_BP_WAVES 16
#endif
  int groups = (MKA_BP_WAVES * 148 + nchunk * B - 1) / (nchunk * B);
  groups = groups < 1 ? 1 : (groups > nblk ? nblk : groups);
  const int bpg = (nblk + groups - 1) / groups;
  groups = (nblk + bpg - 1) / bpg;
  dim3 g1(nchunk, B, groups);
  if (x_bf16)
    block_proj_partial_kernel<bf16><<<g1, 256, 0, s>>>((const bf16*)x, d, S, blk, nblk, bpg, P64, nb, part);
  else
    block_proj_partial_kernel<float><<<g1, 256, 0, s>>>((const float*)x, d, S, blk, nblk, bpg, P64, nb, part);
  block_codes_kernel<<<dim3(nblk, B), 32, 0, s>>>(part, nchunk, nb, nblk, codes, code_bstride);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- block sums + EMA end states
__device__ __forceinline__ float4 f4_fma(float a, float4 x, float4 y) {
  return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}
__device__ __forceinline__ float4 f4_add(float4 x, float4 y) { return make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w); }
__device__ __forceinline__ float4 f4_scale(float a, float4 x) { return make_float4(a * x.x, a * x.y, a * x.z, a * x.w); }
// One EMA step m <- a*m + (1-a)*x.
__device__ __forceinline__ float4 ema_step(float al, float om, float4 m, float4 x) {
  return make_float4(fmaf(al, m.x, om * x.x), fmaf(al, m.y, om * x.y), fmaf(al, m.z, om * x.z), fmaf(al, m.w, om * x.w));
}

constexpr int kRG = 8;  // row groups per block in block_reduce and fuse_kv

// Rows [ra, rb) of row group g of a block of `blk` rows.
__device__ __forceinline__ void group_rows(int g, int blk, int& ra, int& rb) {
  const int per = (blk + kRG - 1) / kRG;
  ra = min(g * per, blk);
  rb = min(ra + per, blk);
}

template <typename T>
__global__ void __launch_bounds__(512) block_reduce_kernel(const T* __restrict__ x, int ld, int width, int S, int nblk,
                                                            int blk, float alpha, float* __restrict__ bsum,
                                                            long long bsum_bstride, float* __restrict__ bend,
                                                            float* __restrict__ gend) {
  __shared__ float4 ssum[kRG][64], send[kRG][64];
  const int bi = blockIdx.z, j = blockIdx.y;
  const int cl = threadIdx.x & 63, rg = threadIdx.x >> 6;
  const int c = (blockIdx.x * 64 + cl) * 4;
  int ra, rb;
  group_rows(rg, blk, ra, rb);
  const float om = 1.f - alpha;
  float4 s = make_float4(0, 0, 0, 0), e = s;
  if (c < width) {
    const T* p = x + ((size_t)bi * S + (size_t)j * blk) * ld + c;
#pragma unroll 4
    for (int r = ra; r < rb; ++r) {
      float4 v = Vec4<T>::load(p + (size_t)r * ld);
      s = f4_add(s, v);
      e = ema_step(alpha, om, e, v);
    }
    if (gend) *(float4*)(gend + (((size_t)bi * nblk + j) * kRG + rg) * width + c) = e;
  }
  ssum[rg][cl] = s;
  send[rg][cl] = e;
  __syncthreads();
  if (rg == 0 && c < width) {
    float4 S4 = ssum[0][cl], E4 = send[0][cl];
    for (int g = 1; g < kRG; ++g) {
      int ga, gb;
      group_rows(g, blk, ga, gb);
      float ap = 1.f;
      for (int i = ga; i < gb; ++i) ap *= alpha;  // a^(rows of group g)
      S4 = f4_add(S4, ssum[g][cl]);
      E4 = f4_add(f4_scale(ap, E4), send[g][cl]);
    }
    if (bsum) *(float4*)(bsum + (size_t)bi * bsum_bstride + (size_t)j * width + c) = S4;
    if (bend) *(float4*)(bend + ((size_t)bi * nblk + j) * width + c) = E4;
  }
}

cudaError_t block_reduce(const void* x, int x_bf16, int ld, int width, int B, int S, int nblk, int blk, float alpha,
                         float* bsum, long long bsum_bstride, float* bend, float* gend, cudaStream_t s) {
  if (B <= 0 || nblk <= 0) return cudaSuccess;
  dim3 grid((width / 4 + 63) / 64, nblk, B);
  if (x_bf16)
    block_reduce_kernel<bf16><<<grid, 64 * kRG, 0, s>>>((const bf16*)x, ld, width, S, nblk, blk, alpha, bsum,
                                                         bsum_bstride, bend, gend);
  else
    block_reduce_kernel<float><<<grid, 64 * kRG, 0, s>>>((const float*)x, ld, width, S, nblk, blk, alpha, bsum,
                                                          bsum_bstride, bend, gend);
  return cudaGetLastError();
}

// carry[b][0] = carry_in (or 0); carry[b][j+1] = A * carry[b][j] + bend[b][j], A = a^blk.
// CTA = (32 columns, sequence b), 32 warps: warp w scans blocks [w*cpw, (w+1)*cpw) from a
// zero carry (lanes = columns, coalesced), the 32 chunk end states are chained in order
// (A^len * c + end), then every warp rescans its chunk from its true carry-in.
__global__ void __launch_bounds__(1024) ema_carry_kernel(const float* __restrict__ bend, int width, int nblk,
                                                          float apb, const float* __restrict__ carry_in,
                                                          float* __restrict__ carry) {
  __shared__ float sA[32][33], sL[32][33], sC[33][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int bi = blockIdx.y, c = blockIdx.x * 32 + lane;
  const int cpw = (nblk + 31) / 32;
  const int j0 = min(nblk, w * cpw), j1 = min(nblk, j0 + cpw);
  const bool ok = c < width;
  const float* e = bend + (size_t)bi * nblk * width + c;
  float L = 0.f, A = 1.f;
  if (ok)
    for (int j = j0; j < j1; ++j) {
      L = fmaf(apb, L, e[(size_t)j * width]);
      A *= apb;
    }
  sA[w][lane] = A;
  sL[w][lane] = L;
  __syncthreads();
  if (w == 0) {
    float cur = (ok && carry_in) ? carry_in[(size_t)bi * width + c] : 0.f;
    for (int k = 0; k < 32; ++k) {
      sC[k][lane] = cur;
      cur = fmaf(sA[k][lane], cur, sL[k][lane]);
    }
    sC[32][lane] = cur;
  }
  __syncthreads();
  if (!ok) return;
  float* out = carry + (size_t)bi * (nblk + 1) * width + c;
  float cur = sC[w][lane];
  for (int j = j0; j < j1; ++j) {
    out[(size_t)j * width] = cur;
    cur = fmaf(apb, cur, e[(size_t)j * width]);
  }
  if (w == 31) out[(size_t)nblk * width] = sC[32][lane];
}

cudaError_t ema_carry(const float* bend, int width, int B, int nblk, float alpha_pow_b, const float* carry_in,
                      float* carry, cudaStream_t s) {
  if (B <= 0 || width <= 0) return cudaSuccess;
  dim3 grid((width + 31) / 32, B);
  ema_carry_kernel<<<grid, 1024, 0, s>>>(bend, width, nblk, alpha_pow_b, carry_in, carry);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- top-R recall
// One warp per token.  Distances take at most 33 values, so the (distance,
// index) order is built by counting: a histogram gives each distance's first
// output slot, and a pass in index order places equal-distance blocks by rank
// (__match_any_sync groups the lanes that share a distance).  Deterministic, no
// sort, every output position written exactly once.
__global__ void __launch_bounds__(256) recall_kernel(const uint32_t* __restrict__ tok, const uint32_t* __restrict__ blkc,
                                                     int bstride, int B, int S, int nblk, int blk, int R,
                                                     int* __restrict__ idx, int* __restrict__ count) {
  __shared__ int base[8][34];
  __shared__ int run[8][34];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tg = (long long)blockIdx.x * 8 + w;
  if (tg >= (long long)B * S) return;
  const int bi = (int)(tg / S), t = (int)(tg % S);
  const int n = min(t / blk, nblk);
  const int cnt = min(R, n);
  const uint32_t code = tok[tg];
  const uint32_t* bc = blkc + (size_t)bi * bstride;
  int* out = idx + tg * R;
  for (int i = lane; i < 34; i += 32) {
    base[w][i] = 0;
    run[w][i] = 0;
  }
  __syncwarp();
  for (int j0 = 0; j0 < n; j0 += 32) {
    int j = j0 + lane;
    if (j < n) atomicAdd(&base[w][__popc(code ^ bc[j])], 1);
  }
  __syncwarp();
  if (lane == 0) {
    int acc = 0;
    for (int dd = 0; dd < 34; ++dd) {
      int h = base[w][dd];
      base[w][dd] = acc;
      acc += h;
    }
  }
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  for (int j0 = 0; j0 < n; j0 += 32) {
    int j = j0 + lane;
    bool valid = j < n;
    int dist = valid ? __popc(code ^ bc[j]) : 64 + lane;
    unsigned grp = __match_any_sync(0xffffffffu, dist);
    int rank = __popc(grp & lt);
    int pos = valid ? base[w][dist] + run[w][dist] + rank : R;
    __syncwarp();
    if (valid && pos < R) out[pos] = j;
    if (valid && rank == 0) run[w][dist] += __popc(grp);
    __syncwarp();
  }
  for (int p = cnt + lane; p < R; p += 32) out[p] = -1;
  if (lane == 0 && count) count[tg] = cnt;
}

cudaError_t recall_select(const uint32_t* tok_codes, const uint32_t* blk_codes, int blk_codes_bstride, int B, int S,
                          int nblk, int blk, int R, int* idx, int* count, cudaStream_t s) {
  long long T = (long long)B * S;
  if (T <= 0) return cudaSuccess;
  recall_kernel<<<(unsigned)((T + 7) / 8), 256, 0, s>>>(tok_codes, blk_codes, blk_codes_bstride, B, S, nblk, blk, R, idx,
                                                        count);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- route-fuse -> K, V
// notes §3: X_fused = l1*X + l2*M2 + l3*M3, applied to the projected columns.
// One CTA per (sequence, block, 256 columns); rows of the block run in order
// (the EMA recurrence), starting from the block's carried EMA value.
template <typename OutT>
__device__ __forceinline__ void store4(OutT* p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float* p, float4 v) { *(float4*)p = v; }
template <> __device__ __forceinline__ void store4<bf16>(bf16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *(uint32_t*)&a;
  u.y = *(uint32_t*)&b;
  *(uint2*)p = u;
}

template <typename OutT>
__global__ void __launch_bounds__(64 * kRG) fuse_kernel(FuseArgs a) {
  extern __shared__ float sm[];
  float* slam = sm;                                   // [blk*3]
  int* sidx = (int*)(slam + a.blk * 3);               // [blk*R]
  int* scnt = sidx + a.blk * a.R;                     // [blk]
  const int bi = blockIdx.z, j = blockIdx.y;
  const int r0 = j * a.blk, r1 = min(r0 + a.blk, a.S), nr = r1 - r0;
  const size_t tg0 = (size_t)bi * a.S + r0;
  for (int i = threadIdx.x; i < nr * 3; i += blockDim.x) slam[i] = a.lam[tg0 * 3 + i];
  for (int i = threadIdx.x; i < nr * a.R; i += blockDim.x) sidx[i] = a.idx[tg0 * a.R + i];
  for (int i = threadIdx.x; i < nr; i += blockDim.x) scnt[i] = a.count[tg0 + i];
  __syncthreads();
  const int cl = threadIdx.x & 63, rg = threadIdx.x >> 6;
  const int c = (blockIdx.x * 64 + cl) * 4;
  if (c >= a.width) return;
  const float om = 1.f - a.alpha;
  // EMA value at the first row of this thread's row group: the block's carry advanced
  // over the preceding groups (their zero-carry end states come from block_reduce).
  float4 m2 = *(const float4*)(a.carry + ((size_t)bi * (a.nblk + 1) + j) * a.width + c);
  int ra, rb;
  if (j < a.nblk) {
    group_rows(rg, a.blk, ra, rb);
    for (int g = 0; g < rg; ++g) {
      int ga, gb;
      group_rows(g, a.blk, ga, gb);
      float ap = 1.f;
      for (int i = ga; i < gb; ++i) ap *= a.alpha;
      float4 ge = *(const float4*)(a.gend + (((size_t)bi * a.nblk + j) * kRG + g) * a.width + c);
      m2 = f4_add(f4_scale(ap, m2), ge);
    }
  } else {  // the unfinished last block: one group walks all its rows
    ra = 0;
    rb = rg == 0 ? nr : 0;
  }
  const float* bs = a.bsum + (size_t)bi * a.bsum_bstride + c;
  const bool is_k = c < a.dkv;
  OutT* dst = (OutT*)(is_k ? a.k_out : a.v_out) + (size_t)bi * a.kv_bstride + (size_t)r0 * a.dkv + (is_k ? c : c - a.dkv);
  const float* xp = a.xkv + tg0 * a.ld + c;
  const float invb = 1.f / (float)a.blk;
  if (a.v2_out) {  // full MKA: raw K/V of the tokens and the L2 value, no fusion
    float* v2 = is_k ? nullptr : a.v2_out + tg0 * a.dkv + (c - a.dkv);
    for (int r = ra; r < rb; ++r) {
      const float4 x = *(const float4*)(xp + (size_t)r * a.ld);
      store4<OutT>(dst + (size_t)r * a.dkv, x);
      if (v2) *(float4*)(v2 + (size_t)r * a.dkv) = m2;
      m2 = ema_step(a.alpha, om, m2, x);
    }
    if (r1 == a.S && rb == nr && rb > ra && a.state_ema) *(float4*)(a.state_ema + (size_t)bi * a.width + c) = m2;
    return;
  }
  for (int r = ra; r < rb; ++r) {
    float4 x = *(const float4*)(xp + (size_t)r * a.ld);
    int cnt = scnt[r];
    float4 m3 = make_float4(0, 0, 0, 0);
    for (int q = 0; q < cnt; ++q) m3 = f4_add(m3, *(const float4*)(bs + (size_t)sidx[r * a.R + q] * a.width));
    float s3 = cnt ? invb / (float)cnt : 0.f;
    float l0 = slam[r * 3], l1 = slam[r * 3 + 1], l2 = slam[r * 3 + 2];
    float4 o = f4_fma(l0, x, f4_fma(l1, m2, f4_scale(l2 * s3, m3)));
    store4<OutT>(dst + (size_t)r * a.dkv, o);
    m2 = ema_step(a.alpha, om, m2, x);
  }
  if (r1 == a.S && rb == nr && rb > ra && a.state_ema) *(float4*)(a.state_ema + (size_t)bi * a.width + c) = m2;
}

// ---------------------------------------------------------------- route-fuse with staged summaries
// The same fuse, organised around the recalled-block gather.  A CTA owns one sequence, a 64-column
// slice of the projected sources and a range of blocks.  It first stages that slice of the mean of
// every block its tokens can recall (the blocks before its last one) in shared memory, so the
// R-way gather-mean of each token reads shared memory instead of L2.  bf16 layers stage the means
// in bf16: 2^-9 relative on M3, the size of the rounding of the K/V it feeds; float32 layers stage
// float32.  Threads: 8 columns each, 8 threads per row, the kRG row groups of a block (EMA carried
// in from block_reduce's group end states), kFsBlocks blocks at a time; the projected rows, counts
// and gates are loaded two rows ahead.
constexpr int kFsCols = 64, kFsLaneCols = 8, kFsLanes = kFsCols / kFsLaneCols;
constexpr int kFsThreads = 256, kFsBlocks = kFsThreads / (kFsLanes * kRG), kFsBlocksPerCta = kFsBlocks;
constexpr size_t kFsMaxSmem = 200 * 1024;
constexpr int kFsBatch = 8;  // staging loads in flight per thread

template <typename ST> struct Staged8;
template <> struct Staged8<bf16> {
  static __device__ __forceinline__ void put(bf16* p, float4 a, float4 b, float sc) {
    __nv_bfloat162 h0 = __floats2bfloat162_rn(a.x * sc, a.y * sc), h1 = __floats2bfloat162_rn(a.z * sc, a.w * sc);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(b.x * sc, b.y * sc), h3 = __floats2bfloat162_rn(b.z * sc, b.w * sc);
    *(uint4*)p = make_uint4(*(uint32_t*)&h0, *(uint32_t*)&h1, *(uint32_t*)&h2, *(uint32_t*)&h3);
  }
  // a row's 8 staged columns, loaded before they are added so that several gathers are in flight
  using V = uint4;
  static __device__ __forceinline__ V load(const bf16* p) { return *(const uint4*)p; }
  static __device__ __forceinline__ V zero() { return make_uint4(0, 0, 0, 0); }
  // sm_100 mixed-precision adds: each bf16 half of a word goes straight into its fp32 sum (the
  // same round-to-nearest fp32 sum as widening first), one instruction per element
  static __device__ __forceinline__ void accum(V u, float2* acc) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
          "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
          : "+f"(acc[i].x), "+f"(acc[i].y)
          : "r"(w[i]));
  }
};
template <> struct Staged8<float> {
  static __device__ __forceinline__ void put(float* p, float4 a, float4 b, float sc) {
    *(float4*)p = f4_scale(sc, a);
    *(float4*)(p + 4) = f4_scale(sc, b);
  }
  struct V {
    float4 a, b;
  };
  static __device__ __forceinline__ V load(const float* p) { return {*(const float4*)p, *(const float4*)(p + 4)}; }
  static __device__ __forceinline__ V zero() { return {make_float4(0, 0, 0, 0), make_float4(0, 0, 0, 0)}; }
  static __device__ __forceinline__ void accum(const V& v, float2* acc) {
    acc[0] = __fadd2_rn(acc[0], make_float2(v.a.x, v.a.y));
    acc[1] = __fadd2_rn(acc[1], make_float2(v.a.z, v.a.w));
    acc[2] = __fadd2_rn(acc[2], make_float2(v.b.x, v.b.y));
    acc[3] = __fadd2_rn(acc[3], make_float2(v.b.z, v.b.w));
  }
};

template <typename OutT> __device__ __forceinline__ void store8(OutT* p, const float* v);
template <> __device__ __forceinline__ void store8<float>(float* p, const float* v) {
  *(float4*)p = make_float4(v[0], v[1], v[2], v[3]);
  *(float4*)(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
template <> __device__ __forceinline__ void store8<bf16>(bf16* p, const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *(uint32_t*)&h;
  }
  *(uint4*)p = make_uint4(w[0], w[1], w[2], w[3]);
}

// Shared memory of one CTA: the staged means of every block, then one ring per row group of
// kFsDepth rows in flight: the projected columns of its 8 lanes and the row's recalled indices,
// gates and count (cp.async, no registers held while the copies fly).
constexpr int kFsDepth = 4;
constexpr int kFsInflight = 8;  // gathers of one row in flight per lane
constexpr int kFsGroups = kFsThreads / kFsLanes;  // row groups of a CTA
template <typename ST>
__host__ __device__ __forceinline__ size_t fs_mean_bytes(int nblk) {
  return ((size_t)nblk * kFsCols * sizeof(ST) + 15) & ~(size_t)15;
}
// idx[R], lam[3], cnt, rounded up to 4 words: at least R rounded up to kFsInflight
__host__ __device__ __forceinline__ int fs_meta(int R) { return (R + 4 + 3) & ~3; }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename OutT, typename ST>
__global__ void __launch_bounds__(kFsThreads, 2) fuse_staged_kernel(FuseArgs a, int blocks_per_cta) {
  extern __shared__ __align__(16) uint8_t fs_smem[];
  const int bi = blockIdx.z, c0 = blockIdx.x * kFsCols;
  const int nb_all = (a.S + a.blk - 1) / a.blk;  // the unfinished block included
  const int J0 = blockIdx.y * blocks_per_cta, J1 = min(nb_all, J0 + blocks_per_cta);
  if (J0 >= J1) return;
  const int nstage = min(J1 - 1, a.nblk);  // a token of block j recalls blocks < j only
  ST* smean = (ST*)fs_smem;                // [nstage][kFsCols] block means of this slice
  const int meta = fs_meta(a.R);
  float* ring_x = (float*)(fs_smem + fs_mean_bytes<ST>(a.nblk));        // [groups][depth][kFsCols]
  uint32_t* ring_m = (uint32_t*)(ring_x + kFsGroups * kFsDepth * kFsCols);  // [groups][depth][meta]
  const float invb = 1.f / (float)a.blk;
  const float* bs = a.bsum + (size_t)bi * a.bsum_bstride + c0;
  // staging loads are batched (kFsBatch per thread in flight before any store)
  for (int i0 = 0; i0 < nstage * kFsLanes; i0 += kFsBatch * kFsThreads) {
    float4 va[kFsBatch], vb[kFsBatch];
#pragma unroll
    for (int u = 0; u < kFsBatch; ++u) {
      const int i = i0 + u * kFsThreads + (int)threadIdx.x;
      if (i < nstage * kFsLanes) {
        const float* src = bs + (size_t)(i / kFsLanes) * a.width + (i % kFsLanes) * kFsLaneCols;
        va[u] = *(const float4*)src;
        vb[u] = *(const float4*)(src + 4);
      }
    }
#pragma unroll
    for (int u = 0; u < kFsBatch; ++u) {
      const int i = i0 + u * kFsThreads + (int)threadIdx.x;
      if (i < nstage * kFsLanes)
        Staged8<ST>::put(smean + (i / kFsLanes) * kFsCols + (i % kFsLanes) * kFsLaneCols, va[u], vb[u], invb);
    }
  }
  __syncthreads();
  const int lane = threadIdx.x % kFsLanes, gid = threadIdx.x / kFsLanes;
  const int rg = gid % kRG, bl = gid / kRG;
  const unsigned gmask = 0xffu << (8 * (gid & 3));  // this group's 8 lanes within the warp
  const int cs = lane * kFsLaneCols, c = c0 + cs;
  const bool is_k = c < a.dkv;
  const float al = a.alpha, om = 1.f - a.alpha;
  float* gx = ring_x + (size_t)gid * kFsDepth * kFsCols;
  uint32_t* gm = ring_m + (size_t)gid * kFsDepth * meta;
  for (int j = J0 + bl; j < J1; j += kFsBlocks) {
    const int r0 = j * a.blk, nr = min(a.blk, a.S - r0);
    int ra, rb;
    if (j < a.nblk) {
      group_rows(rg, a.blk, ra, rb);
    } else {  // the unfinished last block: one group walks all its rows
      ra = 0;
      rb = rg == 0 ? nr : 0;
    }
    const size_t tg0 = (size_t)bi * a.S + r0;
    OutT* dst = (OutT*)(is_k ? a.k_out : a.v_out) + (size_t)bi * a.kv_bstride + (size_t)r0 * a.dkv +
                (is_k ? c : c - a.dkv);
    // row r into ring slot (r - ra) % kFsDepth: each lane its 8 columns, the indices, gates and
    // count shared out over the 8 lanes
    auto issue = [&](int r) {
      if (r < rb) {
        const size_t t = tg0 + r;
        const int slot = (r - ra) % kFsDepth;
        const float* xp = a.xkv + t * a.ld + c;
        cp_async16(gx + slot * kFsCols + cs, xp);
        cp_async16(gx + slot * kFsCols + cs + 4, xp + 4);
        uint32_t* m = gm + slot * meta;
        for (int k = lane; k < a.R + 4; k += kFsLanes) {
          const void* src = k < a.R ? (const void*)(a.idx + t * a.R + k)
                            : k < a.R + 3 ? (const void*)(a.lam + t * 3 + (k - a.R)) : (const void*)(a.count + t);
          cp_async4(m + k, src);
        }
      }
      cp_commit();  // one group per row (empty past the end), so the waits below count rows
    };
#pragma unroll
    for (int d = 0; d < kFsDepth; ++d) issue(ra + d);
    // EMA value at this group's first row: the block's carry advanced over the preceding groups
    const float* cp = a.carry + ((size_t)bi * (a.nblk + 1) + j) * a.width + c;
    float4 ma = *(const float4*)cp, mb = *(const float4*)(cp + 4);
    if (j < a.nblk) {
#pragma unroll
      for (int g = 0; g < kRG - 1; ++g) {
        if (g < rg) {
          int ga, gb;
          group_rows(g, a.blk, ga, gb);
          float ap = 1.f;
          for (int i = ga; i < gb; ++i) ap *= al;
          const float* ge = a.gend + (((size_t)bi * a.nblk + j) * kRG + g) * a.width + c;
          ma = f4_add(f4_scale(ap, ma), *(const float4*)ge);
          mb = f4_add(f4_scale(ap, mb), *(const float4*)(ge + 4));
        }
      }
    }
    float m2[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
    for (int r = ra; r < rb; ++r) {
      cp_wait<kFsDepth - 1>();  // row r landed (this lane's copies)
      __syncwarp(gmask);        // and the other lanes' share of its indices
      const int slot = (r - ra) % kFsDepth;
      const float* xs = gx + slot * kFsCols + cs;
      const uint32_t* m = gm + slot * meta;
      const int cnt = (int)m[a.R + 3];
      const float l0 = __uint_as_float(m[a.R]), l1 = __uint_as_float(m[a.R + 1]), l2 = __uint_as_float(m[a.R + 2]);
      float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // kFsInflight gathers issued before their adds; indices read four at a time (a slot's meta
      // words run to a multiple of 4 past R, so the reads stay in the slot; entries past cnt and
      // indices outside the staged blocks add nothing)
      for (int q0 = 0; q0 < cnt; q0 += kFsInflight) {
        typename Staged8<ST>::V v[kFsInflight];
#pragma unroll
        for (int k = 0; k < kFsInflight; k += 4) {
          const uint4 j4 = *(const uint4*)(m + q0 + k);
          const uint32_t jj[4] = {j4.x, j4.y, j4.z, j4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
            v[k + u] = q0 + k + u < cnt && jj[u] < (uint32_t)nstage ? Staged8<ST>::load(smean + jj[u] * kFsCols + cs)
                                                                    : Staged8<ST>::zero();
        }
#pragma unroll
        for (int k = 0; k < kFsInflight; ++k) Staged8<ST>::accum(v[k], acc2);
      }
      const float acc[8] = {acc2[0].x, acc2[0].y, acc2[1].x, acc2[1].y, acc2[2].x, acc2[2].y, acc2[3].x, acc2[3].y};
      const float4 xa = *(const float4*)xs, xb = *(const float4*)(xs + 4);
      const float x[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      const float s3 = cnt ? l2 / (float)cnt : 0.f;
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o[i] = fmaf(l0, x[i], fmaf(l1, m2[i], s3 * acc[i]));
        m2[i] = fmaf(al, m2[i], om * x[i]);
      }
      store8<OutT>(dst + (size_t)r * a.dkv, o);
      __syncwarp(gmask);  // the slot is read by all 8 lanes before it is refilled
      issue(r + kFsDepth);
    }
    cp_wait<0>();
    if (r0 + rb == a.S && rb > ra && a.state_ema) {
      float* se = a.state_ema + (size_t)bi * a.width + c;
      *(float4*)se = make_float4(m2[0], m2[1], m2[2], m2[3]);
      *(float4*)(se + 4) = make_float4(m2[4], m2[5], m2[6], m2[7]);
    }
  }
}

// Shared-memory bytes of the staged fuse (0: it does not apply, use fuse_kernel).  Staging pays
// when a token's gather is large: the unstaged kernel reads R * width floats per token from L2
// (17 GB at 1 x 131072 with R = 16 and width 2048, where it is L2-bound), while the staged one
// spends about two instructions per gathered element (bf16 unpack and add) and is issue-bound.
// Measured crossover: staged 1.16 ms against 1.24 at R * width = 32768; unstaged 0.187 ms
// against 0.217 at R * width = 8192 (2 x 32768 tokens).
constexpr int kFsMinGather = 16384;
size_t fuse_staged_smem(const FuseArgs& a) {
  if (a.v2_out || a.width % kFsCols || a.dkv % kFsCols || a.R > 64) return 0;
  if ((long long)a.R * a.width < kFsMinGather) return 0;
  const size_t means = a.out_bf16 ? fs_mean_bytes<bf16>(a.nblk) : fs_mean_bytes<float>(a.nblk);
  const size_t rings = (size_t)kFsGroups * kFsDepth * (kFsCols + fs_meta(a.R)) * 4;
  const size_t b = means + rings;
  return b <= kFsMaxSmem ? b : 0;
}

cudaError_t fuse_kv(const FuseArgs& a, cudaStream_t s) {
  if (a.B <= 0 || a.S <= 0) return cudaSuccess;
  int nb_all = (a.S + a.blk - 1) / a.blk;
  if (const size_t fsm = fuse_staged_smem(a)) {
    // many short CTAs (one pass of kFsBlocks blocks of one column slice each) balance the SMs;
    // two are resident per SM, so one stages while the other streams
    const int slices = a.width / kFsCols;
    const int bpc = kFsBlocksPerCta;
    const int nchunk = (nb_all + bpc - 1) / bpc;
    dim3 grid(slices, nchunk, a.B);
    cudaError_t e;
    if (a.out_bf16) {
      e = set_max_smem(fuse_staged_kernel<bf16, bf16>, fsm, s);
      if (e != cudaSuccess) return e;
      fuse_staged_kernel<bf16, bf16><<<grid, kFsThreads, fsm, s>>>(a, bpc);
    } else {
      e = set_max_smem(fuse_staged_kernel<float, float>, fsm, s);
      if (e != cudaSuccess) return e;
      fuse_staged_kernel<float, float><<<grid, kFsThreads, fsm, s>>>(a, bpc);
    }
    return cudaGetLastError();
  }
  dim3 grid((a.width / 4 + 63) / 64, nb_all, a.B);
  size_t sm = (size_t)a.blk * (3 * sizeof(float) + (a.R + 1) * sizeof(int));
  if (a.out_bf16) {
    cudaError_t e = set_max_smem(fuse_kernel<bf16>, sm, s);
    if (e != cudaSuccess) return e;
    fuse_kernel<bf16><<<grid, 64 * kRG, sm, s>>>(a);
  } else {
    cudaError_t e = set_max_smem(fuse_kernel<float>, sm, s);
    if (e != cudaSuccess) return e;
    fuse_kernel<float><<<grid, 64 * kRG, sm, s>>>(a);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- standalone d-space pieces
template <typename T>
__global__ void __launch_bounds__(64) ema_apply_kernel(const T* __restrict__ x, int width, int S, int nblk, int blk,
                                                        float alpha, const float* __restrict__ carry,
                                                        float* __restrict__ m2, float* __restrict__ carry_out) {
  const int bi = blockIdx.z, j = blockIdx.y;
  const int c = (blockIdx.x * 64 + threadIdx.x) * 4;
  if (c >= width) return;
  const int r0 = j * blk, r1 = min(r0 + blk, S);
  const float om = 1.f - alpha;
  float4 m = *(const float4*)(carry + ((size_t)bi * (nblk + 1) + j) * width + c);
  const size_t base = ((size_t)bi * S + r0) * width + c;
  for (int r = 0; r < r1 - r0; ++r) {
    *(float4*)(m2 + base + (size_t)r * width) = m;
    m = ema_step(alpha, om, m, Vec4<T>::load(x + base + (size_t)r * width));
  }
  if (r1 == S && carry_out) *(float4*)(carry_out + (size_t)bi * width + c) = m;
}

cudaError_t ema_apply(const void* x, int x_bf16, int width, int B, int S, int nblk, int blk, float alpha,
                      const float* carry, float* m2, float* carry_out, cudaStream_t s) {
  if (B <= 0 || S <= 0) return cudaSuccess;
  dim3 grid((width / 4 + 63) / 64, (S + blk - 1) / blk, B);
  if (x_bf16) ema_apply_kernel<bf16><<<grid, 64, 0, s>>>((const bf16*)x, width, S, nblk, blk, alpha, carry, m2, carry_out);
  else ema_apply_kernel<float><<<grid, 64, 0, s>>>((const float*)x, width, S, nblk, blk, alpha, carry, m2, carry_out);
  return cudaGetLastError();
}

// m3[t] = (1 / (count * blk)) * sum_q bsum[idx[t][q]]  (mean of the recalled block means).
__global__ void gather_mean_kernel(const int* __restrict__ idx, const int* __restrict__ count, int R,
                                   const float* __restrict__ bsum, int nblk, int width, int blk, int S,
                                   float* __restrict__ m3) {
  const size_t tg = blockIdx.x;
  const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
  if (c >= width) return;
  const int bi = (int)(tg / S);
  const int cnt = count[tg];
  const float* bs = bsum + (size_t)bi * nblk * width + c;
  float4 acc = make_float4(0, 0, 0, 0);
  for (int q = 0; q < cnt; ++q) acc = f4_add(acc, *(const float4*)(bs + (size_t)idx[tg * R + q] * width));
  float sc = cnt ? 1.f / ((float)cnt * (float)blk) : 0.f;
  *(float4*)(m3 + tg * width + c) = f4_scale(sc, acc);
}

cudaError_t gather_mean(const int* idx, const int* count, int R, const float* bsum, int nblk, int width, int blk,
                        int B, int S, float* m3, cudaStream_t s) {
  if (B <= 0 || S <= 0) return cudaSuccess;
  dim3 grid(B * S, (width / 4 + 127) / 128);
  gather_mean_kernel<<<grid, 128, 0, s>>>(idx, count, R, bsum, nblk, width, blk, S, m3);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- decode state after a prefill
// The unfinished last block of each sequence: its projected-row sums and its exact float64
// d_model-space sum (from which decode forms the block's code once the block is complete).
template <typename T>
__global__ void prefill_tail_kernel(const float* __restrict__ xkv, int ld, int width, const T* __restrict__ x, int d,
                                    int S, int blk, float* blk_sum, double* blk_x, int* pos) {
  const int bi = blockIdx.x;
  const int r0 = (S / blk) * blk;  // first row of the unfinished block
  const size_t t0 = (size_t)bi * S;
  for (int c = threadIdx.x; c < width; c += blockDim.x) {
    float s = 0.f;
    for (int r = r0; r < S; ++r) s += xkv[(t0 + r) * ld + c];
    blk_sum[(size_t)bi * width + c] = s;
  }
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    double s = 0.0;
    for (int r = r0; r < S; ++r) s += to_d<T>(x[(t0 + r) * d + i]);
    blk_x[(size_t)bi * d + i] = s;
  }
  if (threadIdx.x == 0) pos[bi] = S;
}

cudaError_t prefill_tail_state(const float* xkv, int ld, int width, const void* x, int x_bf16, int d, int B, int S,
                               int blk, float* blk_sum, double* blk_x, int* pos, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  if (x_bf16)
    prefill_tail_kernel<bf16><<<B, 256, 0, s>>>(xkv, ld, width, (const bf16*)x, d, S, blk, blk_sum, blk_x, pos);
  else
    prefill_tail_kernel<float><<<B, 256, 0, s>>>(xkv, ld, width, (const float*)x, d, S, blk, blk_sum, blk_x, pos);
  return cudaGetLastError();
}

}  // namespace mka
