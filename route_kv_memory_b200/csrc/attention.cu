// Causal GQA attention over the fused K/V for float32 workloads (notes §3 of the
// MKA paper: one standard causal attention after the route-fuse), with the
// online max-shift of notes §4: a running row maximum mu; each new key rescales
// the earlier partial sums by exp(mu_prev - mu_new).  CUDA-core FFMA keeps the
// float32 accuracy; the bf16 path is tc_attention.cu.
#include "common.cuh"
#include "kernels.h"

namespace mka {

// Plain float32 path: one warp per (query row, head); lanes own d_head / 32 channels.
template <int DH>
__global__ void attn_fwd_f32_kernel(AttnArgs a) {
  constexpr int PER = DH / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (item >= (long long)a.B * a.S * a.Hq) return;
  const int h = (int)(item % a.Hq);
  const int t = (int)((item / a.Hq) % a.S);
  const int bi = (int)(item / ((long long)a.Hq * a.S));
  const int g = h / (a.Hq / a.Hkv);
  const float* q = (const float*)a.q + (size_t)bi * a.q_bstride + (size_t)t * a.q_ld + (size_t)h * DH;
  const float* K = (const float*)a.k + (size_t)bi * a.kv_bstride + (size_t)g * DH;
  const float* V = (const float*)a.v + (size_t)bi * a.kv_bstride + (size_t)g * DH;
  float qr[PER], acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    qr[i] = q[lane + 32 * i];
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j <= t; ++j) {
    const float* kr = K + (size_t)j * a.kv_ld;
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) s = fmaf(qr[i], kr[lane + 32 * i], s);
    s = warp_sum(s) * a.scale;
    float mn = fmaxf(m, s);
    float corr = expf(m - mn);
    float p = expf(s - mn);
    l = l * corr + p;
    const float* vr = V + (size_t)j * a.kv_ld;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = fmaf(acc[i], corr, p * vr[lane + 32 * i]);
    m = mn;
  }
  float* o = (float*)a.o + (size_t)bi * a.o_bstride + (size_t)t * a.o_ld + (size_t)h * DH;
  float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < PER; ++i) o[lane + 32 * i] = acc[i] * inv;
}

cudaError_t attention_prefill(const AttnArgs& a, int bf16_, cudaStream_t s) {
  if (a.B <= 0 || a.S <= 0) return cudaSuccess;
  if (bf16_) return cudaErrorInvalidValue;  // bf16 runs on tcgen05: attention_prefill_tc
  long long items = (long long)a.B * a.S * a.Hq;
  unsigned blocks = (unsigned)((items + 7) / 8);
  if (a.dh == 128) attn_fwd_f32_kernel<128><<<blocks, 256, 0, s>>>(a);
  else attn_fwd_f32_kernel<64><<<blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mka
