// Block-gathered attention around the tcgen05 kernel: the per-block token lists it walks and the
// merge of its per-block partial results.
//
// Block-MKA (MKA paper notes §4-5) lets a token attend to keys of its own L3 block and of the R
// blocks its hash recall picked; full MKA's third path (notes §2) lets it attend to the recalled
// blocks alone.  Recall is per token, so the query rows that need one block's keys are scattered:
// block_lists() lists, for every block (b, j), the tokens that recalled it (after the block's own
// tokens when those are attended too), the gathered attention runs each list's rows against that
// block's keys on the tensor cores, and merge_partials() combines each row's per-block softmax
// results exactly as the online max-shift does (notes §4): with lse_s = m_s + log2(l_s) in log2
// units, o = sum_s 2^(lse_s - M) (O_s / l_s) / sum_s 2^(lse_s - M), M = max_s lse_s.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace mka {
namespace {

constexpr int kListThreads = 256;

// Tokens of batch b that recalled each block, counted in shared memory first.
__global__ void __launch_bounds__(kListThreads) block_count_kernel(const int* __restrict__ idx,
                                                                   const int* __restrict__ cnt, int S, int R,
                                                                   int nblk, int* __restrict__ nrec) {
  extern __shared__ int hist[];
  const int b = blockIdx.y;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < S; t += gridDim.x * blockDim.x) {
    const size_t tok = (size_t)b * S + t;
    const int c = min(cnt[tok], R);
    for (int r = 0; r < c; ++r) {
      const int j = idx[tok * R + r];
      if (j >= 0 && j < nblk) atomicAdd(&hist[j], 1);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nblk; i += blockDim.x)
    if (hist[i]) atomicAdd(&nrec[b * nblk + i], hist[i]);
}

// Exclusive scans over the B*nblk blocks (one CTA): where each block's entries start, and its
// first tile pair (entries = own tokens + recalling tokens, tiles of tpt tokens, pairs of tiles).
__global__ void __launch_bounds__(1024) block_scan_kernel(const int* __restrict__ nrec, int nbj, int nblk,
                                                          int blk, int S, int own, int tpt,
                                                          int* __restrict__ recoff, int* __restrict__ pairoff,
                                                          int* __restrict__ cursor, int* __restrict__ pairbj) {
  __shared__ int wsum[2][32];
  __shared__ int carry[2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  if (threadIdx.x == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  for (int base = 0; base < nbj; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int n = 0, pairs = 0;
    if (i < nbj) {
      n = nrec[i];
      const int j = i % nblk;
      const int entries = (own ? min(blk, S - j * blk) : 0) + n;
      pairs = ((entries + tpt - 1) / tpt + 1) / 2;
      cursor[i] = 0;
    }
    int xn = n, xp = pairs;  // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yn = __shfl_up_sync(0xffffffffu, xn, o), yp = __shfl_up_sync(0xffffffffu, xp, o);
      if (lane >= o) {
        xn += yn;
        xp += yp;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = xn;
      wsum[1][warp] = xp;
    }
    __syncthreads();
    if (warp == 0) {
      int sn = lane < nwarps ? wsum[0][lane] : 0, sp = lane < nwarps ? wsum[1][lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yn = __shfl_up_sync(0xffffffffu, sn, o), yp = __shfl_up_sync(0xffffffffu, sp, o);
        if (lane >= o) {
          sn += yn;
          sp += yp;
        }
      }
      if (lane < nwarps) {  // exclusive prefix of the warps
        wsum[0][lane] = sn - wsum[0][lane];
        wsum[1][lane] = sp - wsum[1][lane];
      }
    }
    __syncthreads();
    if (i < nbj) {
      recoff[i] = carry[0] + wsum[0][warp] + xn - n;
      const int p0 = carry[1] + wsum[1][warp] + xp - pairs;
      pairoff[i] = p0;
      for (int p = 0; p < pairs; ++p) pairbj[p0 + p] = i;
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) {
      carry[0] += wsum[0][warp] + xn;
      carry[1] += wsum[1][warp] + xp;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) pairoff[nbj] = carry[1];
}

// Appends (t << 5) | (r + slot_base) to the list of block idx[t][r].  The order inside a list is
// whatever the atomics give: each row's result does not depend on the other rows of its tile.
__global__ void __launch_bounds__(kListThreads) block_fill_kernel(const int* __restrict__ idx,
                                                                  const int* __restrict__ cnt, int S, int R,
                                                                  int nblk, int slot_base,
                                                                  const int* __restrict__ recoff,
                                                                  int* __restrict__ cursor, int* __restrict__ list) {
  const int b = blockIdx.y;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < S; t += gridDim.x * blockDim.x) {
    const size_t tok = (size_t)b * S + t;
    const int c = min(cnt[tok], R);
    for (int r = 0; r < c; ++r) {
      const int j = idx[tok * R + r];
      if (j < 0 || j >= nblk) continue;
      const int pos = atomicAdd(&cursor[b * nblk + j], 1);
      list[recoff[b * nblk + j] + pos] = (t << 5) | (r + slot_base);
    }
  }
}

// Per tile pair P (persistent CTAs over the pairs): its block with a flag for a second tile, and its
// 2 tpt list entries, the block's own tokens first (own), then the recalling tokens' entries.
__global__ void __launch_bounds__(256) pair_tokens_kernel(const int* __restrict__ nrec, const int* __restrict__ recoff,
                                                          const int* __restrict__ list, const int* __restrict__ pairoff,
                                                          const int* __restrict__ pairbj, int nbj, int nblk, int blk,
                                                          int S, int own, int tpt, int* __restrict__ ptok,
                                                          int* __restrict__ pinfo) {
  const int npairs = pairoff[nbj];
  for (int P = blockIdx.x; P < npairs; P += gridDim.x) {
    const int bj = pairbj[P], j = bj % nblk, p = P - pairoff[bj];
    const int nown = own ? min(blk, S - j * blk) : 0, entries = nown + nrec[bj], e0 = 2 * p * tpt;
    for (int i = threadIdx.x; i < 2 * tpt; i += blockDim.x) {
      const int e = e0 + i;
      ptok[(size_t)P * 2 * tpt + i] = e >= entries ? -1 : e < nown ? ((j * blk + e) << 5) : list[recoff[bj] + e - nown];
    }
    if (threadIdx.x == 0) pinfo[P] = bj | ((e0 + tpt < entries) ? (1 << 30) : 0);
  }
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// One CTA per token (grid-stride); each thread owns 8 consecutive output columns of one head.
__global__ void __launch_bounds__(512) merge_kernel(MergeArgs m) {
  const int dq = m.Hq * m.dh, G = m.Hq / m.Hkv;
  const long long T = (long long)m.B * m.S;
  const bf16* po = (const bf16*)m.part_o;
  for (long long tok = blockIdx.x; tok < T; tok += gridDim.x) {
    const int b = (int)(tok / m.S), t = (int)(tok - (long long)b * m.S);
    const int ns = min(m.cnt[tok], m.nslot - m.own) + m.own;
    bf16* orow = (bf16*)m.o + (size_t)b * m.o_bstride + (size_t)t * m.o_ld;
    for (int cc = threadIdx.x; cc < dq / 8; cc += blockDim.x) {
      const int h = cc * 8 / m.dh;
      const float* lse = m.part_lse + (size_t)tok * m.nslot * m.Hq + h;
      float mx = -INFINITY;
      for (int s = 0; s < ns; ++s) mx = fmaxf(mx, lse[(size_t)s * m.Hq]);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, wsum = 0.f;
      const bf16* src = po + (size_t)tok * m.nslot * dq + cc * 8;
#pragma unroll 4
      for (int s = 0; s < ns; ++s) {
        const float w = ex2f(lse[(size_t)s * m.Hq] - mx);
        const uint4 u = *(const uint4*)(src + (size_t)s * dq);
        const __nv_bfloat162* p2 = (const __nv_bfloat162*)&u;
        wsum += w;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(p2[e]);
          acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
        }
      }
      const float inv = ns > 0 ? 1.f / wsum : 0.f;
      uint4 out;
      uint32_t* ow = (uint32_t*)&out;
      if (m.lam) {  // full MKA: lam0 * causal output + lam1 * L2 value + lam2 * recalled-block output
        const float l0 = m.lam[tok * 3], l1 = m.lam[tok * 3 + 1], l2 = m.lam[tok * 3 + 2];
        const uint4 o1 = *(const uint4*)(orow + cc * 8);
        const __nv_bfloat162* o12 = (const __nv_bfloat162*)&o1;
        const float* v2 = m.v2 + (size_t)tok * (m.Hkv * m.dh) + (size_t)(h / G) * m.dh + (cc * 8 - h * m.dh);
        const float4 va = *(const float4*)v2, vb = *(const float4*)(v2 + 4);
        const float v2e[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(o12[e]);
          __nv_bfloat162 r = __floats2bfloat162_rn(fmaf(l0, f.x, fmaf(l1, v2e[2 * e], l2 * acc[2 * e] * inv)),
                                                   fmaf(l0, f.y, fmaf(l1, v2e[2 * e + 1], l2 * acc[2 * e + 1] * inv)));
          ow[e] = *(uint32_t*)&r;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          __nv_bfloat162 r = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
          ow[e] = *(uint32_t*)&r;
        }
      }
      *(uint4*)(orow + cc * 8) = out;
    }
  }
}

}  // namespace

cudaError_t block_lists(const int* idx, const int* cnt, int B, int S, int R, int blk, int nblk, int own,
                        int slot_base, int tpt, int* nrec, int* recoff, int* cursor, int* pairoff, int* pairbj,
                        int* list, int* ptok, int* pinfo, cudaStream_t s) {
  if (B <= 0 || S <= 0) return cudaSuccess;
  if (R < 1 || R + slot_base > 31 || blk <= 0 || nblk <= 0 || tpt <= 0 || S >= (1 << 26))
    return cudaErrorInvalidValue;
  const size_t hist = (size_t)nblk * sizeof(int);
  if (hist > 48 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(nrec, 0, (size_t)B * nblk * sizeof(int), s);
  if (e != cudaSuccess) return e;
  const int gx = min((S + kListThreads - 1) / kListThreads, 64);
  block_count_kernel<<<dim3(gx, B), kListThreads, hist, s>>>(idx, cnt, S, R, nblk, nrec);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  block_scan_kernel<<<1, 1024, 0, s>>>(nrec, B * nblk, nblk, blk, S, own, tpt, recoff, pairoff, cursor, pairbj);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  block_fill_kernel<<<dim3(gx, B), kListThreads, 0, s>>>(idx, cnt, S, R, nblk, slot_base, recoff, cursor, list);
  if ((e = cudaGetLastError()) != cudaSuccess || !ptok) return e;
  if (B * nblk >= (1 << 30)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  pair_tokens_kernel<<<sms * 4, 256, 0, s>>>(nrec, recoff, list, pairoff, pairbj, B * nblk, nblk, blk, S, own, tpt,
                                              ptok, pinfo);
  return cudaGetLastError();
}

cudaError_t merge_partials(const MergeArgs& m, cudaStream_t s) {
  if (m.B <= 0 || m.S <= 0) return cudaSuccess;
  const int dq = m.Hq * m.dh;
  if (dq % 8 || m.dh % 8 || m.o_ld % 8 || m.o_bstride % 8 || m.nslot < 1 || m.own < 0 || m.own > 1 ||
      (m.lam && !m.v2))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long T = (long long)m.B * m.S;
  const int threads = min(512, ((dq / 8 + 31) / 32) * 32);
  const long long grid = min(T, (long long)sms * 8);
  merge_kernel<<<(int)grid, threads, 0, s>>>(m);
  return cudaGetLastError();
}

}  // namespace mka
