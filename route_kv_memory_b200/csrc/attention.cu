// Causal GQA attention over the fused K/V (notes §3 of the MKA paper: one
// standard causal attention after the route-fuse), with the online max-shift of
// notes §4: a running row maximum mu; on each key tile the earlier partial sums
// are rescaled by exp(mu_prev - mu_new).
#include "common.cuh"
#include "kernels.h"

namespace mka {

namespace fa {
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }
__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *(uint32_t*)&v;
}

constexpr int BQ = 128, BKV = 64, NW = 8, NT = NW * 32;

// Row r of a [rows][DH] bf16 tile: chunk c (16 B) stored at c ^ (r & 7).
template <int DH> __device__ __forceinline__ int swz(int r, int c) { return r * DH + ((c ^ (r & 7)) << 3); }

template <int DH>
__global__ void __launch_bounds__(NT) attn_fwd_bf16_kernel(AttnArgs a) {
  constexpr int CH = DH / 8;  // 16-B chunks per row
  extern __shared__ __align__(128) uint8_t smem_raw[];
  bf16* sQ = (bf16*)smem_raw;            // [BQ][DH]
  bf16* sK = sQ + BQ * DH;               // [2][BKV][DH]
  bf16* sV = sK + 2 * BKV * DH;          // [2][BKV][DH]
  const int nqt = (a.S + BQ - 1) / BQ;
  const int qt = nqt - 1 - (int)blockIdx.x;  // longest rows first
  const int h = blockIdx.y, bi = blockIdx.z;
  const int g = h / (a.Hq / a.Hkv);
  const int q0 = qt * BQ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bf16* Q = (const bf16*)a.q + (size_t)bi * a.q_bstride + (size_t)h * DH;
  const bf16* Kp = (const bf16*)a.k + (size_t)bi * a.kv_bstride + (size_t)g * DH;
  const bf16* Vp = (const bf16*)a.v + (size_t)bi * a.kv_bstride + (size_t)g * DH;

  for (int i = tid; i < BQ * CH; i += NT) {
    int r = i / CH, c = i % CH, t = q0 + r;
    bool ok = t < a.S;
    cp_async16(smem_u32(sQ + swz<DH>(r, c)), ok ? (const void*)(Q + (size_t)t * a.q_ld + c * 8) : (const void*)Q, ok ? 16 : 0);
  }
  const int kv_end = min(a.S, q0 + BQ);
  const int nkv = (kv_end + BKV - 1) / BKV;
  auto load_kv = [&](int stage, int kt) {
    bf16* k = sK + stage * BKV * DH;
    bf16* v = sV + stage * BKV * DH;
    for (int i = tid; i < BKV * CH; i += NT) {
      int r = i / CH, c = i % CH, j = kt * BKV + r;
      bool ok = j < kv_end;
      cp_async16(smem_u32(k + swz<DH>(r, c)), ok ? (const void*)(Kp + (size_t)j * a.kv_ld + c * 8) : (const void*)Kp, ok ? 16 : 0);
      cp_async16(smem_u32(v + swz<DH>(r, c)), ok ? (const void*)(Vp + (size_t)j * a.kv_ld + c * 8) : (const void*)Vp, ok ? 16 : 0);
    }
  };
  load_kv(0, 0);
  cp_commit();

  const float sl2 = a.scale * 1.4426950408889634f;  // scale * log2(e)
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  float o[DH / 8][4];
#pragma unroll
  for (int i = 0; i < DH / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  uint32_t qf[DH / 16][4];
  const int row0 = q0 + warp * 16 + (lane >> 2);  // rows row0 and row0 + 8

  for (int kt = 0; kt < nkv; ++kt) {
    if (kt + 1 < nkv) load_kv((kt + 1) & 1, kt + 1);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        int r = warp * 16 + (lane & 15), c = kk * 2 + (lane >> 4);
        ldsm_x4(qf[kk], smem_u32(sQ + swz<DH>(r, c)));
      }
    }
    const bf16* k = sK + (kt & 1) * BKV * DH;
    const bf16* v = sV + (kt & 1) * BKV * DH;
    float s[BKV / 8][4];
#pragma unroll
    for (int i = 0; i < BKV / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < DH / 16; ++kk) {
#pragma unroll
      for (int nj = 0; nj < BKV / 16; ++nj) {
        uint32_t b[4];
        int r = nj * 16 + ((lane >> 4) << 3) + (lane & 7), c = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(b, smem_u32(k + swz<DH>(r, c)));
        mma_bf16(s[2 * nj], qf[kk], b[0], b[1]);
        mma_bf16(s[2 * nj + 1], qf[kk], b[2], b[3]);
      }
    }
    const int k0 = kt * BKV;
    const bool diag = k0 + BKV - 1 > q0 + warp * 16;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int ni = 0; ni < BKV / 8; ++ni) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v2 = s[ni][e] * sl2;
        if (diag) {
          int j = k0 + ni * 8 + (lane & 3) * 2 + (e & 1);
          int i = row0 + ((e >> 1) << 3);
          if (j > i) v2 = -INFINITY;
        }
        s[ni][e] = v2;
        mx[e >> 1] = fmaxf(mx[e >> 1], v2);
      }
    }
    float corr[2], mref[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      float mn = fmaxf(m_r[r], mx[r]);
      mref[r] = mn == -INFINITY ? 0.f : mn;
      corr[r] = exp2f(m_r[r] - mref[r]);
      m_r[r] = mn;
      l_r[r] *= corr[r];
    }
#pragma unroll
    for (int i = 0; i < DH / 8; ++i) {
      o[i][0] *= corr[0];
      o[i][1] *= corr[0];
      o[i][2] *= corr[1];
      o[i][3] *= corr[1];
    }
    uint32_t pf[BKV / 16][4];
#pragma unroll
    for (int ni = 0; ni < BKV / 8; ++ni) {
      float p0 = exp2f(s[ni][0] - mref[0]), p1 = exp2f(s[ni][1] - mref[0]);
      float p2 = exp2f(s[ni][2] - mref[1]), p3 = exp2f(s[ni][3] - mref[1]);
      l_r[0] += p0 + p1;
      l_r[1] += p2 + p3;
      int kk = ni >> 1;
      if ((ni & 1) == 0) {
        pf[kk][0] = pack_bf16(p0, p1);
        pf[kk][1] = pack_bf16(p2, p3);
      } else {
        pf[kk][2] = pack_bf16(p0, p1);
        pf[kk][3] = pack_bf16(p2, p3);
      }
    }
#pragma unroll
    for (int kk = 0; kk < BKV / 16; ++kk) {
#pragma unroll
      for (int dj = 0; dj < DH / 16; ++dj) {
        uint32_t b[4];
        int r = kk * 16 + (((lane >> 3) & 1) << 3) + (lane & 7), c = dj * 2 + (lane >> 4);
        ldsm_x4_t(b, smem_u32(v + swz<DH>(r, c)));
        mma_bf16(o[2 * dj], pf[kk], b[0], b[1]);
        mma_bf16(o[2 * dj + 1], pf[kk], b[2], b[3]);
      }
    }
    __syncthreads();
  }
  cp_wait<0>();
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
  }
  bf16* O = (bf16*)a.o + (size_t)bi * a.o_bstride + (size_t)h * DH;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    int t = row0 + r * 8;
    if (t >= a.S) continue;
    float inv = 1.f / l_r[r];
#pragma unroll
    for (int i = 0; i < DH / 8; ++i) {
      int c = i * 8 + (lane & 3) * 2;
      *(__nv_bfloat162*)(O + (size_t)t * a.o_ld + c) = __floats2bfloat162_rn(o[i][2 * r] * inv, o[i][2 * r + 1] * inv);
    }
  }
}
}  // namespace fa

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
  if (bf16_) {
    dim3 grid((a.S + fa::BQ - 1) / fa::BQ, a.Hq, a.B);
    if (a.dh == 128) {
      size_t sm = (size_t)(fa::BQ + 4 * fa::BKV) * 128 * 2;
      cudaError_t e = set_max_smem(fa::attn_fwd_bf16_kernel<128>, sm, s);
      if (e != cudaSuccess) return e;
      fa::attn_fwd_bf16_kernel<128><<<grid, fa::NT, sm, s>>>(a);
    } else {
      size_t sm = (size_t)(fa::BQ + 4 * fa::BKV) * 64 * 2;
      cudaError_t e = set_max_smem(fa::attn_fwd_bf16_kernel<64>, sm, s);
      if (e != cudaSuccess) return e;
      fa::attn_fwd_bf16_kernel<64><<<grid, fa::NT, sm, s>>>(a);
    }
  } else {
    long long items = (long long)a.B * a.S * a.Hq;
    unsigned blocks = (unsigned)((items + 7) / 8);
    if (a.dh == 128) attn_fwd_f32_kernel<128><<<blocks, 256, 0, s>>>(a);
    else attn_fwd_f32_kernel<64><<<blocks, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mka
