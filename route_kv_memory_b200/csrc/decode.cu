// One FastMKA decode step (MKA paper, paper-notes page §1-§3: the cache holds
// the fused routed K/V, so a step appends one fused row and runs one attention
// path over the cache).  Four launches:
//   1. gemv      y = x_new [W_q | W_k | W_v | W_q W_r1 | P]          (HBM: weights)
//   2. token     router, L3 recall, fuse, K/V append, EMA / block update (one CTA per sequence)
//   3. split-KV  attention partials over cache[0..pos]                 (HBM: cache)
//   4. merge     max-shift combination of the partials
#include "common.cuh"
#include "kernels.h"

namespace mka {

// ---------------------------------------------------------------- 1. GEMV
constexpr int kMaxDecodeBatch = 8;

template <typename T>
__global__ void __launch_bounds__(256) gemv_kernel(const T* __restrict__ W, int N, int d, const T* __restrict__ x, int B,
                                                   float* __restrict__ y) {
  extern __shared__ float sx[];  // [B][d]
  for (int i = threadIdx.x; i < B * d; i += blockDim.x) sx[i] = to_f<T>(x[i]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 8 + warp;
  if (n >= N) return;
  constexpr int V = 16 / sizeof(T);  // elements per 16-B load
  const T* w = W + (size_t)n * d;
  float acc[kMaxDecodeBatch];
#pragma unroll
  for (int b = 0; b < kMaxDecodeBatch; ++b) acc[b] = 0.f;
  const int nchunks = d / V;
#pragma unroll 4
  for (int c = lane; c < nchunks; c += 32) {
    uint4 u = __ldg((const uint4*)(w + c * V));
    float wf[V];
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162* h = (const __nv_bfloat162*)&u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        wf[2 * i] = f.x;
        wf[2 * i + 1] = f.y;
      }
    } else {
      const float* f = (const float*)&u;
#pragma unroll
      for (int i = 0; i < 4; ++i) wf[i] = f[i];
    }
#pragma unroll
    for (int b = 0; b < kMaxDecodeBatch; ++b) {
      if (b < B) {
        const float* xb = sx + b * d + c * V;
#pragma unroll
        for (int i = 0; i < V; ++i) acc[b] = fmaf(wf[i], xb[i], acc[b]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < kMaxDecodeBatch; ++b) {
    if (b < B) {
      float v = warp_sum(acc[b]);
      if (lane == 0) y[(size_t)b * N + n] = v;
    }
  }
}

// ---------------------------------------------------------------- 2. per-token state update
template <typename T>
__global__ void __launch_bounds__(1024) token_kernel(DecodeArgs a) {
  __shared__ float s_red[32][4];
  __shared__ float s_lam[3];
  __shared__ int s_idx[64];
  __shared__ int s_cnt, s_pos, s_skip;
  __shared__ unsigned s_code;
  __shared__ int s_base[34], s_run[34];
  __shared__ unsigned s_scode;
  const int bi = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const float* y = a.y + (size_t)bi * a.Ntot;
  const int width = 2 * a.dkv;
  const float* q = y;
  const float* xkv = y + a.dq;
  const float* h = xkv + width;
  const float* p = h + a.rh * a.rh_segs;
  const T* xn = (const T*)a.x_new + (size_t)bi * a.d;
  if (tid == 0) {
    int pos = a.pos[bi];
    s_pos = pos;
    s_skip = 0;
    if (pos < 0 || pos >= a.Lmax) {
      s_skip = 1;
      set_status(a.status, kStatusCapacity);
    }
  }
  __syncthreads();
  if (s_skip) return;
  const int pos = s_pos;

  // router (notes §2): z = GELU(h) W_r2, lambda = softmax(z)
  float z0 = 0.f, z1 = 0.f, z2 = 0.f;
  for (int j = tid; j < a.rh; j += blockDim.x) {
    float hv = h[j];
    if (a.rh_segs == 2) hv += h[a.rh + j];
    float gv = gelu_erf(hv);
    z0 = fmaf(gv, a.w_r2[j * 3], z0);
    z1 = fmaf(gv, a.w_r2[j * 3 + 1], z1);
    z2 = fmaf(gv, a.w_r2[j * 3 + 2], z2);
  }
  z0 = warp_sum(z0);
  z1 = warp_sum(z1);
  z2 = warp_sum(z2);
  if (lane == 0) {
    s_red[warp][0] = z0;
    s_red[warp][1] = z1;
    s_red[warp][2] = z2;
  }
  // token code of x_new (exact sign decisions, see memory.cu)
  if (warp == 0) {
    float pv = lane < a.nb ? p[lane] : 0.f;
    float rms = sqrtf(warp_sum(pv * pv) / (float)a.nb);
    float e = (float)a.d * 0x1p-20f * rms;
    bool bit = pv > 0.f;
    unsigned doubt = __ballot_sync(0xffffffffu, lane < a.nb && fabsf(pv) <= e);
    while (doubt) {
      int k = __ffs(doubt) - 1;
      doubt &= doubt - 1;
      double acc = 0.0;
      for (int i = lane; i < a.d; i += 32) acc = fma(to_d<T>(xn[i]), a.pT64[(size_t)k * a.d + i], acc);
      acc = warp_sum_d(acc);
      if (lane == k) bit = acc > 0.0;
    }
    unsigned code = __ballot_sync(0xffffffffu, bit && lane < a.nb);
    if (lane == 0) s_code = code;
  }
  __syncthreads();
  if (tid == 0) {
    float t0 = 0.f, t1 = 0.f, t2 = 0.f;
    for (int w = 0; w < nw; ++w) {
      t0 += s_red[w][0];
      t1 += s_red[w][1];
      t2 += s_red[w][2];
    }
    float m = fmaxf(t0, fmaxf(t1, t2));
    float e0 = expf(t0 - m), e1 = expf(t1 - m), e2 = expf(t2 - m);
    float inv = 1.f / (e0 + e1 + e2);
    s_lam[0] = e0 * inv;
    s_lam[1] = e1 * inv;
    s_lam[2] = e2 * inv;
  }
  // L3 recall over the finished blocks (notes §1): counting select, warp 0
  const int n_elig = min(pos / a.blk, a.maxblk);
  const uint32_t* bc = a.scode + (size_t)bi * a.maxblk;
  if (warp == 0) {
    const uint32_t code = s_code;
    for (int i = lane; i < 34; i += 32) {
      s_base[i] = 0;
      s_run[i] = 0;
    }
    __syncwarp();
    for (int j0 = 0; j0 < n_elig; j0 += 32) {
      int j = j0 + lane;
      if (j < n_elig) atomicAdd(&s_base[__popc(code ^ bc[j])], 1);
    }
    __syncwarp();
    if (lane == 0) {
      int acc = 0;
      for (int dd = 0; dd < 34; ++dd) {
        int hh = s_base[dd];
        s_base[dd] = acc;
        acc += hh;
      }
      s_cnt = min(a.R, n_elig);
    }
    __syncwarp();
    const unsigned lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < n_elig; j0 += 32) {
      int j = j0 + lane;
      bool valid = j < n_elig;
      int dist = valid ? __popc(code ^ bc[j]) : 64 + lane;
      unsigned grp = __match_any_sync(0xffffffffu, dist);
      int rank = __popc(grp & lt);
      int ps = valid ? s_base[dist] + s_run[dist] + rank : a.R;
      __syncwarp();
      if (valid && ps < a.R) s_idx[ps] = j;
      if (valid && rank == 0) s_run[dist] += __popc(grp);
      __syncwarp();
    }
  }
  __syncthreads();
  // fuse (notes §3) and append the fused K/V row; advance the EMA and the block sums
  {
    const float l0 = s_lam[0], l1 = s_lam[1], l2 = s_lam[2];
    const int cnt = s_cnt;
    const float s3 = cnt ? 1.f / ((float)cnt * (float)a.blk) : 0.f;
    const float* summ = a.summ + (size_t)bi * a.maxblk * width;
    float* ema = a.ema + (size_t)bi * width;
    float* bsum = a.blk_sum + (size_t)bi * width;
    for (int c = tid; c < width; c += blockDim.x) {
      float xv = xkv[c];
      float m2 = ema[c];
      float m3 = 0.f;
      for (int r = 0; r < cnt; ++r) m3 += summ[(size_t)s_idx[r] * width + c];
      float o = fmaf(l0, xv, fmaf(l1, m2, l2 * s3 * m3));
      T* dst = (T*)(c < a.dkv ? a.kcache : a.vcache) + ((size_t)bi * a.Lmax + pos) * a.dkv + (c < a.dkv ? c : c - a.dkv);
      *dst = from_f<T>(o);
      ema[c] = fmaf(a.alpha, m2, (1.f - a.alpha) * xv);
      bsum[c] += xv;
    }
    for (int i = tid; i < a.d; i += blockDim.x) a.blk_x[(size_t)bi * a.d + i] += to_d<T>(xn[i]);
    // query for the attention, rounded to the layer dtype as the prefill path stores it
    for (int c = tid; c < a.dq; c += blockDim.x) a.qf[(size_t)bi * a.dq + c] = to_f<T>(from_f<T>(q[c]));
  }
  __syncthreads();
  // finish a block: summary = its projected-row sum; code = signs of its exact float64
  // d_model-space sum projected in float64 (the same decision as the prefill path)
  if ((pos + 1) % a.blk == 0 && pos / a.blk < a.maxblk) {
    const int j = pos / a.blk;
    float* bsum = a.blk_sum + (size_t)bi * width;
    float* summ = a.summ + ((size_t)bi * a.maxblk + j) * width;
    if (tid == 0) s_scode = 0u;
    __syncthreads();
    const double* bx = a.blk_x + (size_t)bi * a.d;
    for (int k = warp; k < a.nb; k += nw) {
      double v = 0.0;
      for (int i = lane; i < a.d; i += 32) v = fma(bx[i], a.pT64[(size_t)k * a.d + i], v);
      v = warp_sum_d(v);
      if (lane == 0 && v > 0.0) atomicOr(&s_scode, 1u << k);
    }
    for (int c = tid; c < width; c += blockDim.x) {
      summ[c] = bsum[c];
      bsum[c] = 0.f;
    }
    __syncthreads();
    for (int i = tid; i < a.d; i += blockDim.x) a.blk_x[(size_t)bi * a.d + i] = 0.0;
    if (tid == 0) a.scode[(size_t)bi * a.maxblk + j] = s_scode;
  }
  if (tid == 0) a.pos[bi] = pos + 1;
}

// ---------------------------------------------------------------- 3. split-KV attention, bf16 tensor cores
namespace dk {
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
constexpr int TP = 32;  // positions per warp tile
constexpr int NWD = 4;  // warps per CTA
template <int DH> __device__ __forceinline__ int swz(int r, int c) { return r * DH + ((c ^ (r & 7)) << 3); }

// Grid (nsplit, Hkv, B).  The G = Hq/Hkv query heads of a KV group are the rows
// of one 16-row MMA tile (rows >= G are zero).  Each warp owns a 32-position
// tile per step; the CTA streams its split through a 2-stage cp.async ring.
template <int DH>
__global__ void __launch_bounds__(NWD * 32) decode_attn_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  constexpr int CH = DH / 8;
  constexpr int TILE = TP * DH;  // elements of one K (or V) warp tile
  bf16* sK = (bf16*)smem_raw;                // [2][NWD][TP][DH]
  bf16* sV = sK + 2 * NWD * TILE;            // [2][NWD][TP][DH]
  __shared__ float s_m[NWD][16], s_l[NWD][16];
  const int split = blockIdx.x, g = blockIdx.y, bi = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;
  const int L = a.pos[bi];  // cache length after the append
  const int step = NWD * TP;
  int chunk = (L + a.nsplit - 1) / a.nsplit;
  chunk = (chunk + step - 1) / step * step;
  const int p0 = split * chunk, p1 = min(L, p0 + chunk);
  const bf16* Kp = (const bf16*)a.kcache + (size_t)bi * a.Lmax * a.dkv + (size_t)g * DH;
  const bf16* Vp = (const bf16*)a.vcache + (size_t)bi * a.Lmax * a.dkv + (size_t)g * DH;

  // query fragments (rows = heads g*G .. g*G+G-1)
  uint32_t qf[DH / 16][4];
  {
    const float* qb = a.qf + (size_t)bi * a.dq + (size_t)g * G * DH;
    int r0 = lane >> 2, r1 = r0 + 8;
#pragma unroll
    for (int kk = 0; kk < DH / 16; ++kk) {
      int c = kk * 16 + (lane & 3) * 2;
      float v00 = r0 < G ? qb[r0 * DH + c] : 0.f, v01 = r0 < G ? qb[r0 * DH + c + 1] : 0.f;
      float v10 = r1 < G ? qb[r1 * DH + c] : 0.f, v11 = r1 < G ? qb[r1 * DH + c + 1] : 0.f;
      float w00 = r0 < G ? qb[r0 * DH + c + 8] : 0.f, w01 = r0 < G ? qb[r0 * DH + c + 9] : 0.f;
      float w10 = r1 < G ? qb[r1 * DH + c + 8] : 0.f, w11 = r1 < G ? qb[r1 * DH + c + 9] : 0.f;
      qf[kk][0] = pack_bf16(v00, v01);
      qf[kk][1] = pack_bf16(v10, v11);
      qf[kk][2] = pack_bf16(w00, w01);
      qf[kk][3] = pack_bf16(w10, w11);
    }
  }
  auto load = [&](int stage, int base) {
    for (int i = tid; i < NWD * TP * CH; i += NWD * 32) {
      int w = i / (TP * CH), rem = i % (TP * CH), r = rem / CH, c = rem % CH;
      int j = base + w * TP + r;
      bool ok = j < p1;
      bf16* k = sK + (stage * NWD + w) * TILE;
      bf16* v = sV + (stage * NWD + w) * TILE;
      cp_async16(smem_u32(k + swz<DH>(r, c)), ok ? (const void*)(Kp + (size_t)j * a.dkv + c * 8) : (const void*)Kp, ok ? 16 : 0);
      cp_async16(smem_u32(v + swz<DH>(r, c)), ok ? (const void*)(Vp + (size_t)j * a.dkv + c * 8) : (const void*)Vp, ok ? 16 : 0);
    }
  };
  const float sl2 = a.scale * 1.4426950408889634f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  float o[DH / 8][4];
#pragma unroll
  for (int i = 0; i < DH / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  const int nsteps = p1 > p0 ? (p1 - p0 + step - 1) / step : 0;
  if (nsteps > 0) load(0, p0);
  cp_commit();
  for (int st = 0; st < nsteps; ++st) {
    if (st + 1 < nsteps) load((st + 1) & 1, p0 + (st + 1) * step);
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    const int base = p0 + st * step + warp * TP;
    if (base < p1) {
      const bf16* k = sK + ((st & 1) * NWD + warp) * TILE;
      const bf16* v = sV + ((st & 1) * NWD + warp) * TILE;
      float s[TP / 8][4];
#pragma unroll
      for (int i = 0; i < TP / 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
#pragma unroll
        for (int nj = 0; nj < TP / 16; ++nj) {
          uint32_t b[4];
          int r = nj * 16 + ((lane >> 4) << 3) + (lane & 7), c = kk * 2 + ((lane >> 3) & 1);
          ldsm_x4(b, smem_u32(k + swz<DH>(r, c)));
          mma_bf16(s[2 * nj], qf[kk], b[0], b[1]);
          mma_bf16(s[2 * nj + 1], qf[kk], b[2], b[3]);
        }
      }
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int ni = 0; ni < TP / 8; ++ni)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int j = base + ni * 8 + (lane & 3) * 2 + (e & 1);
          float v2 = j < p1 ? s[ni][e] * sl2 : -INFINITY;
          s[ni][e] = v2;
          mx[e >> 1] = fmaxf(mx[e >> 1], v2);
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
      uint32_t pf[TP / 16][4];
#pragma unroll
      for (int ni = 0; ni < TP / 8; ++ni) {
        float q0 = exp2f(s[ni][0] - mref[0]), q1 = exp2f(s[ni][1] - mref[0]);
        float q2 = exp2f(s[ni][2] - mref[1]), q3 = exp2f(s[ni][3] - mref[1]);
        l_r[0] += q0 + q1;
        l_r[1] += q2 + q3;
        int kk = ni >> 1;
        if ((ni & 1) == 0) {
          pf[kk][0] = pack_bf16(q0, q1);
          pf[kk][1] = pack_bf16(q2, q3);
        } else {
          pf[kk][2] = pack_bf16(q0, q1);
          pf[kk][3] = pack_bf16(q2, q3);
        }
      }
#pragma unroll
      for (int kk = 0; kk < TP / 16; ++kk)
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
  // merge the warps: rows r = lane/4 (+8); quad lanes hold disjoint columns
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
  }
  if ((lane & 3) == 0) {
    s_m[warp][lane >> 2] = m_r[0];
    s_m[warp][(lane >> 2) + 8] = m_r[1];
    s_l[warp][lane >> 2] = l_r[0];
    s_l[warp][(lane >> 2) + 8] = l_r[1];
  }
  __syncthreads();
  float* so = (float*)smem_raw;  // reuse the ring: [16][DH] merged output (after all loads finished)
  for (int i = tid; i < 16 * DH; i += NWD * 32) so[i] = 0.f;
  __syncthreads();
  float M[2], Lsum[2], wgt[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    int row = (lane >> 2) + 8 * r;
    float mm = -INFINITY;
    for (int w = 0; w < NWD; ++w) mm = fmaxf(mm, s_m[w][row]);
    M[r] = mm;
    float ls = 0.f;
    for (int w = 0; w < NWD; ++w) ls += s_m[w][row] == -INFINITY ? 0.f : s_l[w][row] * exp2f(s_m[w][row] - mm);
    Lsum[r] = ls;
    wgt[r] = m_r[r] == -INFINITY ? 0.f : exp2f(m_r[r] - mm);
  }
  for (int w = 0; w < NWD; ++w) {
    if (warp == w) {
#pragma unroll
      for (int i = 0; i < DH / 8; ++i) {
        int c = i * 8 + (lane & 3) * 2;
        int r0 = lane >> 2;
        so[r0 * DH + c] += o[i][0] * wgt[0];
        so[r0 * DH + c + 1] += o[i][1] * wgt[0];
        so[(r0 + 8) * DH + c] += o[i][2] * wgt[1];
        so[(r0 + 8) * DH + c + 1] += o[i][3] * wgt[1];
      }
    }
    __syncthreads();
  }
  // partial record per (b, head, split): [m (log2 units), l, o[DH] (unnormalised)]
  const int rec = DH + 2;
  for (int i = tid; i < G * DH; i += NWD * 32) {
    int r = i / DH, c = i % DH;
    int hq = g * G + r;
    a.part[(((size_t)bi * a.Hq + hq) * a.nsplit + split) * rec + 2 + c] = so[r * DH + c];
  }
  if (warp == 0 && (lane & 3) == 0) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      int row = (lane >> 2) + 8 * r;
      if (row < G) {
        float* pr = a.part + (((size_t)bi * a.Hq + g * G + row) * a.nsplit + split) * rec;
        pr[0] = M[r];
        pr[1] = Lsum[r];
      }
    }
  }
}
}  // namespace dk

// float32 split-KV attention (CUDA cores): grid (nsplit, Hq, B), one warp per position stride.
template <int DH>
__global__ void decode_attn_f32_kernel(DecodeArgs a) {
  constexpr int PER = DH / 32;
  __shared__ float s_m[8], s_l[8];
  __shared__ float s_o[8][DH];
  const int split = blockIdx.x, hq = blockIdx.y, bi = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int g = hq / (a.Hq / a.Hkv);
  const int L = a.pos[bi];
  const int chunk = (L + a.nsplit - 1) / a.nsplit;
  const int p0 = split * chunk, p1 = min(L, p0 + chunk);
  const float* qb = a.qf + (size_t)bi * a.dq + (size_t)hq * DH;
  float qr[PER], acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    qr[i] = qb[lane + 32 * i];
    acc[i] = 0.f;
  }
  const float* K = (const float*)a.kcache + (size_t)bi * a.Lmax * a.dkv + (size_t)g * DH;
  const float* V = (const float*)a.vcache + (size_t)bi * a.Lmax * a.dkv + (size_t)g * DH;
  float m = -INFINITY, l = 0.f;
  for (int j = p0 + warp; j < p1; j += nw) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) s = fmaf(qr[i], K[(size_t)j * a.dkv + lane + 32 * i], s);
    s = warp_sum(s) * a.scale * 1.4426950408889634f;
    float mn = fmaxf(m, s);
    float corr = exp2f(m - mn), pw = exp2f(s - mn);
    l = l * corr + pw;
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = fmaf(acc[i], corr, pw * V[(size_t)j * a.dkv + lane + 32 * i]);
    m = mn;
  }
  if (lane == 0) {
    s_m[warp] = m;
    s_l[warp] = l;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) s_o[warp][lane + 32 * i] = acc[i];
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, s_m[w]);
    float Ls = 0.f;
    float out[PER] = {};
    for (int w = 0; w < nw; ++w) {
      float wg = s_m[w] == -INFINITY ? 0.f : exp2f(s_m[w] - M);
      Ls += s_l[w] * wg;
#pragma unroll
      for (int i = 0; i < PER; ++i) out[i] += s_o[w][lane + 32 * i] * wg;
    }
    const int rec = DH + 2;
    float* pr = a.part + (((size_t)bi * a.Hq + hq) * a.nsplit + split) * rec;
    if (lane == 0) {
      pr[0] = M;
      pr[1] = Ls;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) pr[2 + lane + 32 * i] = out[i];
  }
}

// ---------------------------------------------------------------- 4. merge
template <typename T>
__global__ void decode_merge_kernel(DecodeArgs a) {
  const int hq = blockIdx.x, bi = blockIdx.y;
  const int rec = a.dh + 2;
  const float* pr = a.part + ((size_t)bi * a.Hq + hq) * a.nsplit * rec;
  float M = -INFINITY;
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, pr[(size_t)s * rec]);
  float Ls = 0.f;
  for (int s = 0; s < a.nsplit; ++s) {
    float m = pr[(size_t)s * rec];
    if (m != -INFINITY) Ls += pr[(size_t)s * rec + 1] * exp2f(m - M);
  }
  for (int c = threadIdx.x; c < a.dh; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < a.nsplit; ++s) {
      float m = pr[(size_t)s * rec];
      if (m != -INFINITY) acc += pr[(size_t)s * rec + 2 + c] * exp2f(m - M);
    }
    ((T*)a.out)[(size_t)bi * a.dq + (size_t)hq * a.dh + c] = from_f<T>(acc / Ls);
  }
}

cudaError_t decode_step(const DecodeArgs& a, cudaStream_t s) {
  if (a.B <= 0) return cudaSuccess;
  if (a.B > kMaxDecodeBatch) return cudaErrorInvalidValue;
  size_t smx = (size_t)a.B * a.d * sizeof(float);
  cudaError_t e;
#define MARK(i) \
  if (a.prof) cudaEventRecord(a.prof[i], s);
  MARK(0);
  if (a.x_bf16) {
    e = set_max_smem(gemv_kernel<bf16>, smx, s);
    if (e != cudaSuccess) return e;
    gemv_kernel<bf16><<<(a.Ntot + 7) / 8, 256, smx, s>>>((const bf16*)a.wcatT, a.Ntot, a.d, (const bf16*)a.x_new, a.B, a.y);
    MARK(1);
    token_kernel<bf16><<<a.B, 1024, 0, s>>>(a);
    MARK(2);
    size_t sm = (size_t)2 * 2 * dk::NWD * dk::TP * a.dh * sizeof(bf16);
    dim3 grid(a.nsplit, a.Hkv, a.B);
    if (a.dh == 128) {
      e = set_max_smem(dk::decode_attn_kernel<128>, sm, s);
      if (e != cudaSuccess) return e;
      dk::decode_attn_kernel<128><<<grid, dk::NWD * 32, sm, s>>>(a);
    } else {
      e = set_max_smem(dk::decode_attn_kernel<64>, sm, s);
      if (e != cudaSuccess) return e;
      dk::decode_attn_kernel<64><<<grid, dk::NWD * 32, sm, s>>>(a);
    }
    MARK(3);
    decode_merge_kernel<bf16><<<dim3(a.Hq, a.B), 128, 0, s>>>(a);
    MARK(4);
  } else {
    e = set_max_smem(gemv_kernel<float>, smx, s);
    if (e != cudaSuccess) return e;
    gemv_kernel<float><<<(a.Ntot + 7) / 8, 256, smx, s>>>((const float*)a.wcatT, a.Ntot, a.d, (const float*)a.x_new, a.B, a.y);
    MARK(1);
    token_kernel<float><<<a.B, 1024, 0, s>>>(a);
    MARK(2);
    dim3 grid(a.nsplit, a.Hq, a.B);
    if (a.dh == 128) decode_attn_f32_kernel<128><<<grid, 256, 0, s>>>(a);
    else decode_attn_f32_kernel<64><<<grid, 256, 0, s>>>(a);
    MARK(3);
    decode_merge_kernel<float><<<dim3(a.Hq, a.B), 128, 0, s>>>(a);
    MARK(4);
  }
#undef MARK
  return cudaGetLastError();
}

}  // namespace mka
