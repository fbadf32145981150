// Layer backward around the attention backward: the row sums D = rowsum(dO * O), the routing
// gate and router MLP backward, and the adjoints of the L2 EMA and the L3 recalled means, all in
// the projected space of the forward (columns of X [W_k | W_v], width 2 dkv).
//
// With dY = [dK | dV] per token and the forward's projected sources xkv = X [W_k | W_v],
// E = EMA(xkv) (the L2 value) and M = mean of the recalled block means of xkv (the L3 value):
//   dlam_l = <dY, source_l>                                   (notes §3, fuse)
//   U = lam1 dY + EMA^T(lam2 dY) + M^T(lam3 dY)               (so dX = U [W_k | W_v]^T and
//                                                              [dW_k | dW_v] = X^T U, by linearity)
//   EMA^T:  c_t = lam2[t] dY[t] + a c_{t+1},  U[t-1] += (1 - a) c_t        (notes §1, L2)
//   M^T:    block j collects G_j = sum over the tokens t that recalled it of lam3[t] dY[t] / count[t],
//           and every row of block j gets G_j / b                          (notes §1, L3; the
//           recalled blocks held fixed)
//   router: dz = gate Jacobian^T dlam, dh = (dz W_r2^T) * GELU'(h), dW_r2 = GELU(h)^T dz  (notes §2)
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace mka {
namespace {

__device__ __forceinline__ float warp_sum32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// D[(b * Hq + h) * ld + t] = sum_i dO[b, t, h, i] * O[b, t, h, i]; one warp per token row, 16 lanes
// per head (dh / 8 16-byte pieces each), the head's sum by shuffles within its 16 lanes.
__global__ void __launch_bounds__(256) attn_dsum_kernel(const bf16* __restrict__ dout, const bf16* __restrict__ o,
                                                        int B, int S, int Hq, int dh, int ld, float* __restrict__ dsum) {
  const int lane = threadIdx.x & 31;
  const long long tok = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (tok >= (long long)B * S) return;
  const int row = Hq * dh, per = dh / 8;  // 16-byte pieces per head (8 or 16)
  const uint4* a = (const uint4*)(dout + tok * (size_t)row);
  const uint4* c = (const uint4*)(o + tok * (size_t)row);
  const int b = (int)(tok / S), t = (int)(tok % S);
  for (int p0 = 0; p0 < row / 8; p0 += 32) {  // 32 pieces (512 bytes) per step: 2 or 4 heads
    float acc = 0.f;
    if (p0 + lane < row / 8) {
      const uint4 x = a[p0 + lane], y = c[p0 + lane];
      const __nv_bfloat162* x2 = (const __nv_bfloat162*)&x;
      const __nv_bfloat162* y2 = (const __nv_bfloat162*)&y;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fx = __bfloat1622float2(x2[e]), fy = __bfloat1622float2(y2[e]);
        acc = fmaf(fx.x, fy.x, fmaf(fx.y, fy.y, acc));
      }
    }
    for (int o2 = per / 2; o2 > 0; o2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
    const int piece = p0 + lane;
    if (lane % per == 0 && piece < row / 8) dsum[((size_t)b * Hq + piece / per) * ld + t] = acc;
  }
}

// dL/dz of the routing gate (route_gate in common.cuh) from lam and dL/dlam: where lam is a softmax
// over a set A (the active tiers for soft, the two chosen logits for top-2, read off lam > 0),
// dz_i = lam_i (dlam_i - sum_{k in A} lam_k dlam_k); fixed and top-1 weights are constants.
__device__ __forceinline__ void route_gate_grad(const float* lam, const float* dlam, int mode, int tiers, float* dz) {
  bool in[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) in[i] = mode == 0 ? ((tiers >> i) & 1) != 0 : (mode == 3 && lam[i] > 0.f);
  float inner = 0.f;
#pragma unroll
  for (int i = 0; i < 3; ++i) inner += in[i] ? lam[i] * dlam[i] : 0.f;
#pragma unroll
  for (int i = 0; i < 3; ++i) dz[i] = in[i] ? lam[i] * (dlam[i] - inner) : 0.f;
}

// One warp per token (grid-stride): dlam from dY and the three sources, the gate and router-MLP
// backward; dh (bf16) for the dq and dW_r1 products, dW_r2 summed in registers then atomically.
// hrec: the router pre-activation X (W_q W_r1) as bf16 hi and lo parts, per 256 columns 128 hi
// then 128 lo (interleaved) or all hi then all lo.
constexpr int kMaxRhPerLane = 16;  // rh <= 512
__global__ void __launch_bounds__(256) router_bwd_kernel(RouterBwdArgs a) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, nw = (gridDim.x * blockDim.x) >> 5;
  const long long T = (long long)a.B * a.S;
  const int nu = a.rh / 32;  // hidden units per lane: u = lane + 32 k
  float gw[kMaxRhPerLane][3];
#pragma unroll
  for (int k = 0; k < kMaxRhPerLane; ++k) gw[k][0] = gw[k][1] = gw[k][2] = 0.f;
  for (long long t = warp; t < T; t += nw) {
    // dlam_l = <dY, source_l>, sources xkv, E, M
    float d0 = 0.f, d1 = 0.f, d2 = 0.f;
    const float* dy = a.dy + t * a.width;
    for (int c = lane * 4; c < a.width; c += 128) {
      const float4 g = *(const float4*)(dy + c);
      const float4 x = *(const float4*)(a.xkv + t * a.ld_xkv + c);
      const float4 e = *(const float4*)(a.ema + t * a.width + c);
      const float4 m = *(const float4*)(a.m3 + t * a.width + c);
      d0 += g.x * x.x + g.y * x.y + g.z * x.z + g.w * x.w;
      d1 += g.x * e.x + g.y * e.y + g.z * e.z + g.w * e.w;
      d2 += g.x * m.x + g.y * m.y + g.z * m.z + g.w * m.w;
    }
    float dl[3] = {warp_sum32(d0), warp_sum32(d1), warp_sum32(d2)};
    const float lam[3] = {a.lam[t * 3], a.lam[t * 3 + 1], a.lam[t * 3 + 2]};
    if (lane == 0 && a.dlam) {
      a.dlam[t * 3] = dl[0];
      a.dlam[t * 3 + 1] = dl[1];
      a.dlam[t * 3 + 2] = dl[2];
    }
    float dz[3];
    route_gate_grad(lam, dl, a.route_mode, a.tiers, dz);
#pragma unroll
    for (int k = 0; k < kMaxRhPerLane; ++k) {
      if (k >= nu) break;
      const int u = lane + 32 * k;
      const int chi = a.r_inter ? (u >> 7) * 256 + (u & 127) : u;
      const int clo = a.r_inter ? chi + 128 : u + a.rh;
      const float h = a.hrec[t * (2 * a.rh) + chi] + a.hrec[t * (2 * a.rh) + clo];
      const float g = gelu_erf(h);
      const float dgelu = 0.5f * erfcf(-h * 0.70710678118654752f) + h * 0.3989422804014327f * expf(-0.5f * h * h);
      const float* w2 = a.w_r2 + u * 3;
      const float dg = dz[0] * w2[0] + dz[1] * w2[1] + dz[2] * w2[2];
      ((bf16*)a.dh)[t * a.rh + u] = __float2bfloat16_rn(dg * dgelu);
      gw[k][0] = fmaf(g, dz[0], gw[k][0]);
      gw[k][1] = fmaf(g, dz[1], gw[k][1]);
      gw[k][2] = fmaf(g, dz[2], gw[k][2]);
    }
  }
  // the CTA's warps add into shared memory first: one atomic per weight and CTA
  __shared__ float red[kMaxRhPerLane * 32 * 3];
  for (int i = threadIdx.x; i < a.rh * 3; i += blockDim.x) red[i] = 0.f;
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kMaxRhPerLane; ++k) {
    if (k >= nu) break;
    const int u = lane + 32 * k;
    atomicAdd(&red[u * 3], gw[k][0]);
    atomicAdd(&red[u * 3 + 1], gw[k][1]);
    atomicAdd(&red[u * 3 + 2], gw[k][2]);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < a.rh * 3; i += blockDim.x) atomicAdd(&a.dw_r2[i], red[i]);
}

// G[b][j] += sum over one 64-entry chunk of block j's recall list of lam3[t] dY[t] / count[t]
// (chunk -> block from block_lists' pair table, built with 32 tokens per tile); persistent CTAs,
// the chunk's tokens and weights staged in shared memory, then independent row loads.
constexpr int kChunk = 64;
__global__ void __launch_bounds__(256) recall_grad_kernel(const float* __restrict__ dy, int width,
                                                          const float* __restrict__ lam, const int* __restrict__ cnt,
                                                          const int* __restrict__ nrec, const int* __restrict__ recoff,
                                                          const int* __restrict__ list, const int* __restrict__ pairoff,
                                                          const int* __restrict__ pairbj, int nbj, int S, int nblk,
                                                          float* __restrict__ gsum) {
  __shared__ int stok[kChunk];
  __shared__ float swt[kChunk];
  const int nchunks = pairoff[nbj];
  for (int w = blockIdx.x; w < nchunks; w += gridDim.x) {
    const int bj = pairbj[w], b = bj / nblk;
    const int e0 = (w - pairoff[bj]) * kChunk, m = min(kChunk, nrec[bj] - e0);
    __syncthreads();  // the previous chunk's readers are done with stok / swt
    if (threadIdx.x < m) {
      const size_t tok = (size_t)b * S + (list[recoff[bj] + e0 + threadIdx.x] >> 5);
      stok[threadIdx.x] = (int)tok;
      swt[threadIdx.x] = lam[tok * 3 + 2] / (float)cnt[tok];
    }
    __syncthreads();
    for (int c = threadIdx.x * 4; c < width; c += blockDim.x * 4) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int i = 0; i < m; ++i) {
        const float wt = swt[i];
        const float4 g = *(const float4*)(dy + (size_t)stok[i] * width + c);
        acc.x = fmaf(wt, g.x, acc.x);
        acc.y = fmaf(wt, g.y, acc.y);
        acc.z = fmaf(wt, g.z, acc.z);
        acc.w = fmaf(wt, g.w, acc.w);
      }
      atomicAdd((float4*)(gsum + (size_t)bj * width + c), acc);
    }
  }
}

// EMA adjoint, pass 1: per block of blk rows, rsum = sum_{t in block} a^(t - start) lam2[t] dY[t]
// (the adjoint state at the block start with nothing to its right).
__global__ void __launch_bounds__(64) ema_adj_block_kernel(const float* __restrict__ dy, int width,
                                                           const float* __restrict__ lam, int S, int nball, int blk,
                                                           float alpha, float* __restrict__ rsum) {
  const int b = blockIdx.z, j = blockIdx.y, c = (blockIdx.x * 64 + threadIdx.x) * 4;
  if (c >= width) return;
  const int r0 = j * blk, r1 = min(r0 + blk, S);
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int t = r1 - 1; t >= r0; --t) {
    const size_t tok = (size_t)b * S + t;
    const float l2 = lam[tok * 3 + 1];
    const float4 g = *(const float4*)(dy + tok * width + c);
    r = make_float4(fmaf(l2, g.x, alpha * r.x), fmaf(l2, g.y, alpha * r.y), fmaf(l2, g.z, alpha * r.z),
                    fmaf(l2, g.w, alpha * r.w));
  }
  *(float4*)(rsum + ((size_t)b * nball + j) * width + c) = r;
}

// Pass 2: carries from the right, cs[j] = rsum[j] + a^len(j) cs[j+1], cs[nball] = 0.
__global__ void ema_adj_carry_kernel(const float* __restrict__ rsum, int width, int S, int nball, int blk,
                                     float alpha, float* __restrict__ cs) {
  const int b = blockIdx.y, c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= width) return;
  float v = 0.f;
  cs[((size_t)b * (nball + 1) + nball) * width + c] = 0.f;
  for (int j = nball - 1; j >= 0; --j) {
    const int len = min(blk, S - j * blk);
    v = rsum[((size_t)b * nball + j) * width + c] + powf(alpha, (float)len) * v;
    cs[((size_t)b * (nball + 1) + j) * width + c] = v;
  }
}

// Pass 3: U[t] = lam1[t] dY[t] + (1 - a) c_{t+1} + G[block(t)] / blk, c_t = lam2[t] dY[t] + a c_{t+1},
// walking each block from its end with c = cs[j + 1]; U goes to `u` (bf16, row stride ldu).
__global__ void __launch_bounds__(64) ema_adj_apply_kernel(const float* __restrict__ dy, int width,
                                                           const float* __restrict__ lam, int S, int nball, int nblk,
                                                           int blk, float alpha, const float* __restrict__ cs,
                                                           const float* __restrict__ gsum, bf16* __restrict__ u,
                                                           int ldu) {
  const int b = blockIdx.z, j = blockIdx.y, c = (blockIdx.x * 64 + threadIdx.x) * 4;
  if (c >= width) return;
  const int r0 = j * blk, r1 = min(r0 + blk, S);
  const float om = 1.f - alpha;
  float4 cc = *(const float4*)(cs + ((size_t)b * (nball + 1) + j + 1) * width + c);
  float4 gj = make_float4(0.f, 0.f, 0.f, 0.f);
  if (j < nblk) {  // full blocks are the ones that can be recalled
    const float4 g = *(const float4*)(gsum + ((size_t)b * nblk + j) * width + c);
    const float ib = 1.f / (float)blk;
    gj = make_float4(g.x * ib, g.y * ib, g.z * ib, g.w * ib);
  }
  for (int t = r1 - 1; t >= r0; --t) {
    const size_t tok = (size_t)b * S + t;
    const float l1 = lam[tok * 3], l2 = lam[tok * 3 + 1];
    const float4 g = *(const float4*)(dy + tok * width + c);
    const float4 v = make_float4(fmaf(l1, g.x, fmaf(om, cc.x, gj.x)), fmaf(l1, g.y, fmaf(om, cc.y, gj.y)),
                                 fmaf(l1, g.z, fmaf(om, cc.z, gj.z)), fmaf(l1, g.w, fmaf(om, cc.w, gj.w)));
    __nv_bfloat162 p0 = __floats2bfloat162_rn(v.x, v.y), p1 = __floats2bfloat162_rn(v.z, v.w);
    uint2 pk;
    pk.x = *(uint32_t*)&p0;
    pk.y = *(uint32_t*)&p1;
    *(uint2*)(u + tok * (size_t)ldu + c) = pk;
    cc = make_float4(fmaf(l2, g.x, alpha * cc.x), fmaf(l2, g.y, alpha * cc.y), fmaf(l2, g.z, alpha * cc.z),
                     fmaf(l2, g.w, alpha * cc.w));
  }
}

}  // namespace

cudaError_t attention_dsum(const void* dout, const void* o, int B, int S, int Hq, int dh, int ld, float* dsum,
                           cudaStream_t s) {
  const long long n = (long long)B * S * Hq;
  if (n <= 0) return cudaSuccess;
  if (dh % 8) return cudaErrorInvalidValue;
  const long long warps = (long long)B * S;
  attn_dsum_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, s>>>((const bf16*)dout, (const bf16*)o, B, S, Hq,
                                                                          dh, ld, dsum);
  return cudaGetLastError();
}

cudaError_t router_backward(const RouterBwdArgs& a, cudaStream_t s) {
  if (a.B <= 0 || a.S <= 0) return cudaSuccess;
  if (a.rh % 32 || a.rh / 32 > kMaxRhPerLane || a.width % 4 || a.ld_xkv % 4 || (a.r_inter && a.rh % 128))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  router_bwd_kernel<<<sms * 4, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t memory_adjoint(const MemAdjArgs& a, cudaStream_t s) {
  if (a.B <= 0 || a.S <= 0) return cudaSuccess;
  if (a.width % 4 || a.ldu % 4) return cudaErrorInvalidValue;
  const int nball = (a.S + a.blk - 1) / a.blk;
  const unsigned gx = (unsigned)((a.width / 4 + 63) / 64);
  cudaError_t e;
  if (a.nblk > 0) {
    if ((e = cudaMemsetAsync(a.gsum, 0, (size_t)a.B * a.nblk * a.width * sizeof(float), s)) != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    recall_grad_kernel<<<sms * 4, 256, 0, s>>>(a.dy, a.width, a.lam, a.cnt, a.nrec, a.recoff, a.list, a.pairoff,
                                                a.pairbj, a.B * a.nblk, a.S, a.nblk, a.gsum);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  ema_adj_block_kernel<<<dim3(gx, nball, a.B), 64, 0, s>>>(a.dy, a.width, a.lam, a.S, nball, a.blk, a.alpha, a.rsum);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ema_adj_carry_kernel<<<dim3((a.width + 127) / 128, a.B), 128, 0, s>>>(a.rsum, a.width, a.S, nball, a.blk, a.alpha,
                                                                        a.cs);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  ema_adj_apply_kernel<<<dim3(gx, nball, a.B), 64, 0, s>>>(a.dy, a.width, a.lam, a.S, nball, a.nblk, a.blk, a.alpha,
                                                           a.cs, a.gsum, (bf16*)a.u, a.ldu);
  return cudaGetLastError();
}

}  // namespace mka
