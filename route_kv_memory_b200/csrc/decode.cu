// One FastMKA decode step (MKA paper, paper-notes page §1-§3: the cache holds
// the fused routed K/V, so a step appends one fused row and runs one attention
// path over the cache).  bf16 layers run it as one cooperative launch (the fused
// step below); float32 layers as four launches:
//   1. gemv      y = x_new [W_q | W_k | W_v | W_q W_r1 | P]          (HBM: weights)
//   2. token     router, L3 recall, fuse, K/V append, EMA / block update (one CTA per sequence)
//   3. split-KV  attention partials over cache[0..pos]                 (HBM: cache)
//   4. merge     max-shift combination of the partials
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mka {

// ---------------------------------------------------------------- split-KV partial records
// One record per (sequence, query head, split): o[DH] (unnormalised), then m (log2 units) and
// l, padded to a multiple of four floats so that every record's o starts 16-byte aligned.
__host__ __device__ constexpr int part_rec(int dh) { return dh + 4; }

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
__device__ void token_update(const DecodeArgs& a, const int bi) {
  __shared__ float s_red[32][4];
  __shared__ float s_lam[3];
  __shared__ int s_idx[64];
  __shared__ int s_cnt, s_pos, s_skip;
  __shared__ unsigned s_code;
  __shared__ int s_base[34], s_run[34];
  __shared__ unsigned s_scode;
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

  // router (notes §2): z = GELU(h) W_r2, lambda = route_gate(z) (softmax for the published layer)
  float z0 = 0.f, z1 = 0.f, z2 = 0.f;
  for (int j = tid; j < a.rh; j += blockDim.x) {
    float hv;
    if (a.r_inter) hv = h[(j >> 7) * 256 + (j & 127)] + h[(j >> 7) * 256 + 128 + (j & 127)];
    else hv = a.rh_segs == 2 ? h[j] + h[a.rh + j] : h[j];
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
    route_gate(t0, t1, t2, a.route_mode, a.tiers, s_lam);
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

template <typename T>
__global__ void __launch_bounds__(1024) token_kernel(DecodeArgs a) {
  token_update<T>(a, blockIdx.x);
}

// ---------------------------------------------------------------- 3. split-KV attention, bf16 tensor cores
namespace dk {
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
// L2 cache policies: the K/V cache streams through once per step (evict first); the packed weights
// are read every step (evict last), so they stay in L2 while long caches stream past them.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void cp_async16_hint(uint32_t dst, const void* src, int src_bytes, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src), "r"(src_bytes),
               "l"(pol));
}
__device__ __forceinline__ uint4 ldg_nc_hint(const uint4* p, uint64_t pol) {
  uint4 v;
  asm("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(src));
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
constexpr int TP = 16;  // positions per warp tile
constexpr int NWD = 4;  // warps per CTA
template <int DH> __device__ __forceinline__ int swz(int r, int c) { return r * DH + ((c ^ (r & 7)) << 3); }

// One split of one KV group: positions [split * chunk, ...) of cache[0, L).  The
// G = Hq/Hkv query heads of the group are the rows of one 16-row MMA tile (rows
// >= G are zero); q is read from qsrc (row stride qstride) and rounded to bf16.
// Each warp owns a 32-position tile per step; the CTA (NWD warps) streams its
// split through a 2-stage cp.async ring in smem_raw (2 * 2 * NWD * TP * DH bf16).
template <int DH>
__device__ void attn_unit(const DecodeArgs& a, const int split, const int g, const int bi, const int L,
                          const float* qsrc, const int qstride, uint8_t* smem_raw) {
  constexpr int CH = DH / 8;
  constexpr int TILE = TP * DH;  // elements of one K (or V) warp tile
  bf16* sK = (bf16*)smem_raw;                // [2][NWD][TP][DH]
  bf16* sV = sK + 2 * NWD * TILE;            // [2][NWD][TP][DH]
  __shared__ float s_m[NWD][16], s_l[NWD][16];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;
  const int step = NWD * TP;
  int chunk = (L + a.nsplit - 1) / a.nsplit;
  chunk = (chunk + step - 1) / step * step;
  const int p0 = split * chunk, p1 = min(L, p0 + chunk);
  const bf16* Kp = (const bf16*)a.kcache + (size_t)bi * a.Lmax * a.dkv + (size_t)g * DH;
  const bf16* Vp = (const bf16*)a.vcache + (size_t)bi * a.Lmax * a.dkv + (size_t)g * DH;

  // query fragments (rows = heads g*G .. g*G+G-1)
  uint32_t qf[DH / 16][4];
  {
    const float* qb = qsrc + (size_t)bi * qstride + (size_t)g * G * DH;
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
  const uint64_t pol_kv = l2_evict_first();
  auto load = [&](int stage, int base) {
    for (int i = tid; i < NWD * TP * CH; i += NWD * 32) {
      int w = i / (TP * CH), rem = i % (TP * CH), r = rem / CH, c = rem % CH;
      int j = base + w * TP + r;
      bool ok = j < p1;
      bf16* k = sK + (stage * NWD + w) * TILE;
      bf16* v = sV + (stage * NWD + w) * TILE;
      cp_async16_hint(smem_u32(k + swz<DH>(r, c)), ok ? (const void*)(Kp + (size_t)j * a.dkv + c * 8) : (const void*)Kp,
                      ok ? 16 : 0, pol_kv);
      cp_async16_hint(smem_u32(v + swz<DH>(r, c)), ok ? (const void*)(Vp + (size_t)j * a.dkv + c * 8) : (const void*)Vp,
                      ok ? 16 : 0, pol_kv);
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
  // Each warp parks its weighted rows in the (now idle) ring, then one pass sums the
  // warps in a fixed order: deterministic, one barrier.
  float* so = (float*)smem_raw;  // [NWD][16][DH]
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
  {
    float* mine = so + (size_t)warp * 16 * DH;
#pragma unroll
    for (int i = 0; i < DH / 8; ++i) {
      int c = i * 8 + (lane & 3) * 2;
      int r0 = lane >> 2;
      mine[r0 * DH + c] = o[i][0] * wgt[0];
      mine[r0 * DH + c + 1] = o[i][1] * wgt[0];
      mine[(r0 + 8) * DH + c] = o[i][2] * wgt[1];
      mine[(r0 + 8) * DH + c + 1] = o[i][3] * wgt[1];
    }
  }
  __syncthreads();
  // partial record per (b, head, split): [o[DH] (unnormalised), m (log2 units), l]
  constexpr int rec = part_rec(DH);
  for (int i = tid; i < G * DH; i += NWD * 32) {
    int r = i / DH, c = i % DH;
    int hq = g * G + r;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < NWD; ++w) v += so[((size_t)w * 16 + r) * DH + c];
    a.part[(((size_t)bi * a.Hq + hq) * a.nsplit + split) * rec + c] = v;
  }
  if (warp == 0 && (lane & 3) == 0) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      int row = (lane >> 2) + 8 * r;
      if (row < G) {
        float* pr = a.part + (((size_t)bi * a.Hq + g * G + row) * a.nsplit + split) * rec;
        pr[DH] = M[r];
        pr[DH + 1] = Lsum[r];
      }
    }
  }
  __syncthreads();  // the next unit of this CTA reuses the shared memory
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
    constexpr int rec = part_rec(DH);
    float* pr = a.part + (((size_t)bi * a.Hq + hq) * a.nsplit + split) * rec;
    if (lane == 0) {
      pr[DH] = M;
      pr[DH + 1] = Ls;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) pr[lane + 32 * i] = out[i];
  }
}

// ---------------------------------------------------------------- 4. merge
template <typename T>
__global__ void decode_merge_kernel(DecodeArgs a) {
  const int hq = blockIdx.x, bi = blockIdx.y;
  const int rec = part_rec(a.dh), dh = a.dh;
  const float* pr = a.part + ((size_t)bi * a.Hq + hq) * a.nsplit * rec;
  float M = -INFINITY;
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, pr[(size_t)s * rec + dh]);
  float Ls = 0.f;
  for (int s = 0; s < a.nsplit; ++s) {
    float m = pr[(size_t)s * rec + dh];
    if (m != -INFINITY) Ls += pr[(size_t)s * rec + dh + 1] * exp2f(m - M);
  }
  for (int c = threadIdx.x; c < a.dh; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < a.nsplit; ++s) {
      float m = pr[(size_t)s * rec + dh];
      if (m != -INFINITY) acc += pr[(size_t)s * rec + c] * exp2f(m - M);
    }
    ((T*)a.out)[(size_t)bi * a.dq + (size_t)hq * a.dh + c] = from_f<T>(acc / Ls);
  }
}

// ---------------------------------------------------------------- token update, parallel form
// Per-token decisions, recomputed by every CTA of the fused launch (deterministic, cheap):
// lambda (router), the code of x_new (exact sign decisions), and the recalled blocks.
// Batch-1 GEMV of the fused step: every warp of the grid (TW of them) takes the same number of
// whole rows, q0 = Ntot / TW; the rem leftover rows at the end are split into halves of d / 2,
// dealt one per warp round-robin over the CTAs, so every SM streams about the same bytes (a warp
// with one more whole row than the others held its CTA's SM ~30% longer).  First halves go to y,
// second halves to y2.  Only when the leftover rows lie past the query and K/V rows (the router
// and hash rows, which only the token update reads and which it sums from both), when there are
// enough warps, and when d / 2 is a whole number of 16-byte vectors per lane.  The returned first
// split row is Ntot when rows are not split.
__device__ __forceinline__ int gemv_split_row(const DecodeArgs& a, int TW) {
  const int q0 = a.Ntot / TW, rem = a.Ntot - q0 * TW;
  const bool on = a.B == 1 && a.y2 && rem > 0 && 2 * rem <= TW && q0 * TW >= a.dq + 2 * a.dkv && a.d % 512 == 0;
  return on ? q0 * TW : a.Ntot;
}

struct TokenDecision {
  float lam[3];
  int cnt;
  int idx[64];
};

// Values of one sequence's token update that do not depend on the step's projection row, loaded
// by a token CTA into shared memory before phase A (batch 1): the block codes and this CTA's
// slices of the EMA state, the block sums, the d_model-space block sum and x_new.
struct TokenPrefetch {
  const uint32_t* bc;  // [maxblk] block codes
  const float* ema;    // [c1 - c0]
  const float* bsum;   // [c1 - c0]
  const double* bx;    // [i1 - i0]
  const bf16* xn;      // [i1 - i0]
};

template <typename T>
__device__ void token_decide(const DecodeArgs& a, const int bi, const int pos, TokenDecision* td,
                             const TokenPrefetch* pf, const int split_row) {
  __shared__ float s_red[32][3];
  __shared__ unsigned s_code;
  __shared__ int s_base[34], s_run[34];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  const float* y = a.y + (size_t)bi * a.Ntot;
  const float* y2 = a.y2 + (size_t)bi * a.Ntot;
  const int hrow = a.dq + 2 * a.dkv, prow = hrow + a.rh * a.rh_segs;
  // row r of the projection: y[r], plus its second half for the rows the GEMV split
  auto yr = [&](int r) { return r >= split_row ? y[r] + y2[r - split_row] : y[r]; };
  const T* xn = (const T*)a.x_new + (size_t)bi * a.d;
  float z0 = 0.f, z1 = 0.f, z2 = 0.f;
  for (int j = tid; j < a.rh; j += blockDim.x) {
    float hv;
    if (a.r_inter) hv = yr(hrow + (j >> 7) * 256 + (j & 127)) + yr(hrow + (j >> 7) * 256 + 128 + (j & 127));
    else hv = a.rh_segs == 2 ? yr(hrow + j) + yr(hrow + a.rh + j) : yr(hrow + j);
    const float gv = gelu_erf(hv);
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
  if (warp == 0) {  // code of x_new, same decision rule as the prefill path
    const float pv = lane < a.nb ? yr(prow + lane) : 0.f;
    const float rms = sqrtf(warp_sum(pv * pv) / (float)a.nb);
    const float e = (float)a.d * 0x1p-21f * rms;
    bool bit = pv > 0.f;
    unsigned doubt = __ballot_sync(0xffffffffu, lane < a.nb && fabsf(pv) <= e);
    while (doubt) {
      const int k = __ffs(doubt) - 1;
      doubt &= doubt - 1;
      double acc = 0.0;
      for (int i = lane; i < a.d; i += 32) acc = fma(to_d<T>(xn[i]), a.pT64[(size_t)k * a.d + i], acc);
      acc = warp_sum_d(acc);
      if (lane == k) bit = acc > 0.0;
    }
    const unsigned code = __ballot_sync(0xffffffffu, bit && lane < a.nb);
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
    route_gate(t0, t1, t2, a.route_mode, a.tiers, td->lam);
  }
  // recall among the finished blocks: counting select by (distance, index)
  const int n_elig = min(pos / a.blk, a.maxblk);
  const uint32_t* bc = pf ? pf->bc : a.scode + (size_t)bi * a.maxblk;
  if (warp == 0) {
    const uint32_t code = s_code;
    for (int i = lane; i < 34; i += 32) {
      s_base[i] = 0;
      s_run[i] = 0;
    }
    __syncwarp();
    for (int j0 = 0; j0 < n_elig; j0 += 32) {
      const int j = j0 + lane;
      if (j < n_elig) atomicAdd(&s_base[__popc(code ^ bc[j])], 1);
    }
    __syncwarp();
    if (lane == 0) {
      int acc = 0;
      for (int dd = 0; dd < 34; ++dd) {
        const int hh = s_base[dd];
        s_base[dd] = acc;
        acc += hh;
      }
      td->cnt = min(a.R, n_elig);
    }
    __syncwarp();
    const unsigned lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < n_elig; j0 += 32) {
      const int j = j0 + lane;
      const bool valid = j < n_elig;
      const int dist = valid ? __popc(code ^ bc[j]) : 64 + lane;
      const unsigned grp = __match_any_sync(0xffffffffu, dist);
      const int rank = __popc(grp & lt);
      const int ps = valid ? s_base[dist] + s_run[dist] + rank : a.R;
      __syncwarp();
      if (valid && ps < a.R) td->idx[ps] = j;
      if (valid && rank == 0) s_run[dist] += __popc(grp);
      __syncwarp();
    }
  }
  __syncthreads();
}

// This CTA's share of the token's state update: fused K/V columns [c0, c1) appended at
// `pos`, their EMA values and block sums, and d_model-space block sums [i0, i1).  A token
// at the start of a block (pos % b == 0) starts the block sums from zero.
template <typename T>
__device__ void token_slice(const DecodeArgs& a, const int bi, const int pos, const TokenDecision* td, const int c0,
                            const int c1, const int i0, const int i1, const TokenPrefetch* pf = nullptr) {
  const int width = 2 * a.dkv;
  const float* xkv = a.y + (size_t)bi * a.Ntot + a.dq;
  const T* xn = (const T*)a.x_new + (size_t)bi * a.d;
  const bool fresh = (pos % a.blk) == 0;
  const float l0 = td->lam[0], l1 = td->lam[1], l2 = td->lam[2];
  const int cnt = td->cnt;
  const float s3 = cnt ? 1.f / ((float)cnt * (float)a.blk) : 0.f;
  const float* summ = a.summ + (size_t)bi * a.maxblk * width;
  float* ema = a.ema + (size_t)bi * width;
  float* bsum = a.blk_sum + (size_t)bi * width;
  for (int c = c0 + threadIdx.x; c < c1; c += blockDim.x) {
    const float xv = xkv[c];
    const float m2 = pf ? pf->ema[c - c0] : ema[c];
    // the recalled summaries' loads are independent: issued eight at a time
    float m3 = 0.f;
    for (int r0 = 0; r0 < cnt; r0 += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = r0 + u < cnt ? summ[(size_t)td->idx[r0 + u] * width + c] : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) m3 += v[u];
    }
    const float o = fmaf(l0, xv, fmaf(l1, m2, l2 * s3 * m3));
    T* dst = (T*)(c < a.dkv ? a.kcache : a.vcache) + ((size_t)bi * a.Lmax + pos) * a.dkv + (c < a.dkv ? c : c - a.dkv);
    *dst = from_f<T>(o);
    ema[c] = fmaf(a.alpha, m2, (1.f - a.alpha) * xv);
    bsum[c] = (fresh ? 0.f : (pf ? pf->bsum[c - c0] : bsum[c])) + xv;
  }
  double* bx = a.blk_x + (size_t)bi * a.d;
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x)
    bx[i] = (fresh ? 0.0 : (pf ? pf->bx[i - i0] : bx[i])) + to_d<T>(pf ? (T)pf->xn[i - i0] : xn[i]);
}

// ---------------------------------------------------------------- fused decode step (bf16)
// One cooperative launch, two CTAs per SM, NWD warps each:
//   A  the projection row y = x_new [W_q | W_k | W_v | W_q W_r1 | P] for every sequence.
//      Batch 1: every warp streams two packed weight rows at a time through registers, while
//      the token CTAs copy their state slices into shared memory (cp.async); larger batches
//      stream each CTA's rows through a 2-stage shared-memory ring of TMA bulk copies
//   -- grid barrier --
//   B  the first ntok CTAs: the token update of each sequence (router, L3 recall, fuse, append
//      the fused K/V row at position pos, EMA / block update, pos + 1), split over their column
//      slices; every CTA (from CTA ntok on): split-KV attention of the new queries over the old
//      cache rows [0, pos).  Each attention unit and each token CTA then adds one to a
//      completion count in the state (per (sequence, KV group) and per sequence)
//   C  per (sequence, query head), on the CTAs that have one, once this step's counts are in:
//      merge the split partials and the new row's own term (its score against the appended K
//      row, weight on the appended V row); a block closed by this token gets its summary and
//      code.  The other CTAs leave without waiting.
// The grid barrier and the counts live in the decode state and only grow; every wait is bounded
// by a time limit that records MKA_ERR_DEVICE_TIMEOUT.  All CTAs are co-resident (cooperative
// launch), so no wait can deadlock on scheduling.  A CTA whose wait ran out leaves the step.
// the token CTAs' prefetch area (batch 1): block codes, EMA and block-sum slices, d_model slices
constexpr int kPfCodes = 2048, kPfCols = 256, kPfD = 128;
constexpr size_t kPfBytes = (size_t)kPfCodes * 4 + 2 * kPfCols * 4 + kPfD * (8 + 2);
constexpr int kFusedRing = 2 * 2 * dk::NWD * dk::TP * 128 * 2;  // 64 KB: GEMV chunks, then K/V tiles
static_assert(kFusedRing >= dk::NWD * 16 * 128 * 4, "attention merge scratch must fit the ring");

// Grid barrier on a 64-bit arrival count that only grows: a CTA's own arrival number tells it
// which barrier it is in (every launch passes whole barriers of nblocks arrivals), so the barrier
// is released by the last arrival itself, with no reset and no second word.  A step whose wait
// ran out leaves the count mid-barrier; a prefill into the state (or mka_state_init) zeroes it.
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ bool grid_sync(unsigned long long* count, unsigned nblocks, int* status, unsigned long long* index = nullptr) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    s_ok = 1;
    __threadfence();
    const unsigned long long arrival = atomicAdd(count, 1ull);
    const unsigned long long target = (arrival / nblocks + 1) * nblocks;
    if (index) *index = arrival / nblocks;  // barriers since the count was zeroed
    if (ld_acquire_u64(count) < target) {
      const unsigned long long t0 = sm100::globaltimer();
      const unsigned long long lim = wait_limit(status, kWaitGrid, sm100::kWaitLimitNs);
      while (ld_acquire_u64(count) < target) {
        if (sm100::globaltimer() - t0 > lim) {
          set_status(status, kStatusTimeout);
          s_ok = 0;
          break;
        }
        __nanosleep(32);
      }
    }
    __threadfence();
  }
  __syncthreads();
  return s_ok != 0;
}

// Thread 0 waits until *count reaches target (acquire), then the CTA goes on; false (status set) if
// the wait ran out.
__device__ bool wait_count(const unsigned long long* count, unsigned long long target, int* status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    s_ok = 1;
    if (ld_acquire_u64(count) < target) {
      const unsigned long long t0 = sm100::globaltimer();
      const unsigned long long lim = wait_limit(status, kWaitGrid, sm100::kWaitLimitNs);
      while (ld_acquire_u64(count) < target) {
        if (sm100::globaltimer() - t0 > lim) {
          set_status(status, kStatusTimeout);
          s_ok = 0;
          break;
        }
        __nanosleep(32);
      }
    }
  }
  __syncthreads();
  return s_ok != 0;
}
// One arrival on *count once all of the CTA's writes so far are visible (the barrier orders them
// before thread 0's fence, as in grid_sync).
__device__ __forceinline__ void count_done(unsigned long long* count) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(count, 1ull);
  }
}

__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   sm100::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
               : "memory");
}

// Block-wide sum / max of one value per thread (blockDim.x <= 1024).
__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, u) : v + u;
  }
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = red[0];
  for (int w = 1; w < nw; ++w) t = is_max ? fmaxf(t, red[w]) : t + red[w];
  return t;
}

constexpr int kMaxSplits = 512;

// Block-wide (sum, max) of a pair of values in one pass (blockDim.x <= 1024).
__device__ __forceinline__ float2 block_reduce_sum_max(float s, float m, float2* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  }
  __syncthreads();
  if (lane == 0) red[warp] = make_float2(s, m);
  __syncthreads();
  float2 t = red[0];
  for (int w = 1; w < nw; ++w) t = make_float2(t.x + red[w].x, fmaxf(t.y, red[w].y));
  return t;
}

constexpr int kMergeBatch = 16;  // splits whose o a warp holds in registers at a time

// Combines the split partials (unnormalised o, m in log2 units, l) of (sequence bi, query head
// hq) and, when the step appended a row at pos_old, that row's own term.  Every load that needs
// no reduction goes out first (the new row's terms, each split's m and l, a warp's first
// kMergeBatch splits' o); the splits are shared out over the warps (16-byte loads of o), then
// summed over the warps in a fixed order: deterministic.
template <int DH>
// The split partials are final when this runs; the new row's own term (its K and V rows, written
// by the token-update CTAs) is read only after *tok_count reaches tok_target, so the partials'
// loads fly while the token update finishes.  False if that wait ran out.
__device__ bool merge_unit(const DecodeArgs& a, const int bi, const int hq, const int pos_old,
                           const unsigned long long* tok_count, unsigned long long tok_target) {
  __shared__ float s_w[kMaxSplits];
  __shared__ float red[32];
  __shared__ float2 red2[32];
  __shared__ float4 s_acc[dk::NWD][DH / 4];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int rec = part_rec(DH);
  const int g = hq / (a.Hq / a.Hkv);
  const float* pr = a.part + ((size_t)bi * a.Hq + hq) * a.nsplit * rec;
  const bool has_new = pos_old < a.Lmax;
  const bf16* kn = (const bf16*)a.kcache + ((size_t)bi * a.Lmax + pos_old) * a.dkv + (size_t)g * DH;
  const bf16* vn = (const bf16*)a.vcache + ((size_t)bi * a.Lmax + pos_old) * a.dkv + (size_t)g * DH;
  const float* q = a.y + (size_t)bi * a.Ntot + (size_t)hq * DH;
  float mloc = -INFINITY, lfirst = 0.f;
  for (int sp = tid; sp < a.nsplit; sp += blockDim.x) {
    const float m = __ldcg(pr + (size_t)sp * rec + DH);
    if (sp == tid) lfirst = __ldcg(pr + (size_t)sp * rec + DH + 1);
    s_w[sp] = m;
    mloc = fmaxf(mloc, m);
  }
  float4 ov[kMergeBatch];
  const bool olane = lane < DH / 4;
#pragma unroll
  for (int i = 0; i < kMergeBatch; ++i) {
    const int sp = warp + i * dk::NWD;
    ov[i] = olane && sp < a.nsplit ? __ldcg((const float4*)(pr + (size_t)sp * rec) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (!wait_count(tok_count, tok_target, a.status)) return false;
  float s = 0.f;
  if (has_new)
    for (int c = tid; c < DH; c += blockDim.x)
      s = fmaf(__bfloat162float(__float2bfloat16_rn(__ldcg(q + c))), __bfloat162float(__ldcg(kn + c)), s);
  float vnew[4] = {0.f, 0.f, 0.f, 0.f};  // this thread's columns of the appended V row
  if (has_new && tid < DH / 4)
#pragma unroll
    for (int e = 0; e < 4; ++e) vnew[e] = __bfloat162float(__ldcg(vn + 4 * tid + e));
  const float2 sm = block_reduce_sum_max(s, mloc, red2);
  const float snew = sm.x * a.scale * 1.4426950408889634f;
  const float M = has_new ? fmaxf(sm.y, snew) : sm.y;
  float lloc = 0.f;
  for (int sp = tid; sp < a.nsplit; sp += blockDim.x) {
    const float m = s_w[sp];
    const float w = m == -INFINITY ? 0.f : exp2f(m - M);
    s_w[sp] = w;
    lloc += w * (sp == tid ? lfirst : __ldcg(pr + (size_t)sp * rec + DH + 1));
  }
  const float wn = has_new ? exp2f(snew - M) : 0.f;
  const float Ls = block_reduce(lloc, false, red) + wn;  // also orders the s_w writes before the reads below
  const float inv = 1.f / Ls;
  if (olane) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kMergeBatch; ++i) {
      const int sp = warp + i * dk::NWD;
      const float w = sp < a.nsplit ? s_w[sp] : 0.f;
      acc = make_float4(fmaf(ov[i].x, w, acc.x), fmaf(ov[i].y, w, acc.y), fmaf(ov[i].z, w, acc.z), fmaf(ov[i].w, w, acc.w));
    }
    for (int sp = warp + kMergeBatch * dk::NWD; sp < a.nsplit; sp += dk::NWD) {  // more splits than a batch
      const float4 v = __ldcg((const float4*)(pr + (size_t)sp * rec) + lane);
      const float w = s_w[sp];
      acc = make_float4(fmaf(v.x, w, acc.x), fmaf(v.y, w, acc.y), fmaf(v.z, w, acc.z), fmaf(v.w, w, acc.w));
    }
    s_acc[warp][lane] = acc;
  }
  __syncthreads();
  if (tid < DH / 4) {
    float4 t = s_acc[0][tid];
#pragma unroll
    for (int w = 1; w < dk::NWD; ++w) {
      const float4 u = s_acc[w][tid];
      t = make_float4(t.x + u.x, t.y + u.y, t.z + u.z, t.w + u.w);
    }
    float o[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 4 * tid + e;
      if (has_new) o[e] = fmaf(wn, vnew[e], o[e]);
      ((bf16*)a.out)[(size_t)bi * a.dq + (size_t)hq * DH + c] = __float2bfloat16_rn(o[e] * inv);
    }
  }
  __syncthreads();
  return true;
}

template <int DH>
__device__ __forceinline__ void decode_fused_body(const DecodeArgs& a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  bf16* sx = (bf16*)(smem + kFusedRing);
  uint64_t* gbar = (uint64_t*)(smem + kFusedRing + (((size_t)a.B * a.d * 2 + 15) & ~(size_t)15));
  __shared__ int s_pos[kMaxDecodeBatch];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NW = dk::NWD;
  const unsigned nblk = gridDim.x;
  // positions before this step changes them (visible to the CTA after the first grid barrier)
  if (tid < a.B) s_pos[tid] = a.pos[tid];
  // batch 1 with d_model a multiple of 256 up to 4096: phase A streams the weight rows through
  // registers (no shared-memory ring, no set-up barrier)
  const bool reg_gemv = a.B == 1 && (a.d & 255) == 0 && a.d <= 4096;
  // rows from split_row on go to the GEMV as halves (batch 1, see gemv_split_row)
  const int split_row = reg_gemv ? gemv_split_row(a, (int)nblk * NW) : a.Ntot;
  if (!reg_gemv) {
    if (tid == 0) {
      sm100::mbar_init(&gbar[0], 1);
      sm100::mbar_init(&gbar[1], 1);
      sm100::fence_barrier_init();
    }
    for (int i = tid; i < a.B * a.d / 8; i += blockDim.x) ((uint4*)sx)[i] = ((const uint4*)a.x_new)[i];
    __syncthreads();
  }

  // Batch 1: a token CTA copies what its token update reads from the state (not from this step's
  // projection row) into shared memory while phase A runs (cp.async: the thread does not wait)
  const int ntok = min((int)nblk, 32);
  const int width = 2 * a.dkv;
  const int cpc = (width + ntok - 1) / ntok;  // fused columns per token CTA
  const int dpc = (a.d + ntok - 1) / ntok;    // d_model elements per token CTA
  const bool tok_pf = reg_gemv && (int)blockIdx.x < ntok && a.maxblk <= kPfCodes && cpc <= kPfCols && dpc <= kPfD &&
                      (dpc & 1) == 0;
  TokenPrefetch pf{};
  if (tok_pf) {
    uint8_t* pfa = smem + kFusedRing + (((size_t)a.B * a.d * 2 + 15) & ~(size_t)15) + 64;
    uint32_t* pbc = (uint32_t*)pfa;
    float* pema = (float*)(pbc + kPfCodes);
    float* pbs = pema + kPfCols;
    double* pbx = (double*)(pbs + kPfCols);
    bf16* pxn = (bf16*)(pbx + kPfD);
    const int c0 = min(width, (int)blockIdx.x * cpc), c1 = min(width, c0 + cpc);
    const int i0 = min(a.d, (int)blockIdx.x * dpc), i1 = min(a.d, i0 + dpc);
    for (int k = tid; k < a.maxblk; k += blockDim.x) dk::cp_async4(dk::smem_u32(pbc + k), a.scode + k);
    for (int k = tid; k < c1 - c0; k += blockDim.x) {
      dk::cp_async4(dk::smem_u32(pema + k), a.ema + c0 + k);
      dk::cp_async4(dk::smem_u32(pbs + k), a.blk_sum + c0 + k);
    }
    for (int k = tid; k < i1 - i0; k += blockDim.x) dk::cp_async8(dk::smem_u32(pbx + k), a.blk_x + i0 + k);
    for (int k = 2 * tid; k < i1 - i0; k += 2 * blockDim.x)
      dk::cp_async4(dk::smem_u32(pxn + k), (const bf16*)a.x_new + i0 + k);
    dk::cp_commit();
    pf = TokenPrefetch{pbc, pema, pbs, pbx, pxn};
  }

  // ---- A: projection row, this CTA's share of the packed weight rows
  if (reg_gemv) {
    // Every warp of the grid takes the rows r = gw, gw + TW, ... two at a time; a lane holds the
    // 16-byte vectors lane + 32 k (k < d / 256) of both rows, all of a row's loads issued before
    // its dot products, so each SM keeps ~100 KB of weights in flight.
    const int TW = (int)nblk * NW, gw = (int)blockIdx.x * NW + warp;
    const int kv = a.d / 256;
    const uint4* W = (const uint4*)a.wcatT;
    const size_t rowv = (size_t)a.d / 8;
    const uint4* xv = (const uint4*)a.x_new;  // read through L1: every warp reads the same 16 B pieces
    const uint64_t pol_w = dk::l2_evict_last();
    for (int r = gw; r < split_row; r += 2 * TW) {
      const int r2 = r + TW;
      const bool two = r2 < split_row;
      uint4 w1[16], w2[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (k < kv) {
          w1[k] = dk::ldg_nc_hint(W + (size_t)r * rowv + lane + 32 * k, pol_w);
          if (two) w2[k] = dk::ldg_nc_hint(W + (size_t)r2 * rowv + lane + 32 * k, pol_w);
        }
      }
      float a1[2] = {0.f, 0.f}, a2[2] = {0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if (k < kv) {
          const uint4 xu = __ldg(xv + lane + 32 * k);
          const __nv_bfloat162* xh = (const __nv_bfloat162*)&xu;
          const __nv_bfloat162* h1 = (const __nv_bfloat162*)&w1[k];
          const __nv_bfloat162* h2 = (const __nv_bfloat162*)&w2[k];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xf = __bfloat1622float2(xh[e]);
            const float2 f1 = __bfloat1622float2(h1[e]);
            a1[k & 1] = fmaf(f1.x, xf.x, a1[k & 1]);
            a1[k & 1] = fmaf(f1.y, xf.y, a1[k & 1]);
            if (two) {
              const float2 f2 = __bfloat1622float2(h2[e]);
              a2[k & 1] = fmaf(f2.x, xf.x, a2[k & 1]);
              a2[k & 1] = fmaf(f2.y, xf.y, a2[k & 1]);
            }
          }
        }
      }
      const float v1 = warp_sum(a1[0] + a1[1]);
      const float v2 = two ? warp_sum(a2[0] + a2[1]) : 0.f;
      if (lane == 0) {
        a.y[r] = v1;
        if (two) a.y[r2] = v2;
      }
    }
    // half-row hi of the split rows: warp (CTA c, warp wi) takes hi = wi * nblk + c
    const int hi = warp * (int)nblk + (int)blockIdx.x;
    if (hi < 2 * (a.Ntot - split_row)) {
      const int row = split_row + (hi >> 1), half = hi & 1;
      const int hv = a.d / 512;            // 16-byte vectors per lane in half a row
      const size_t off = (size_t)half * (rowv / 2);
      uint4 w1[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (k < hv) w1[k] = dk::ldg_nc_hint(W + (size_t)row * rowv + off + lane + 32 * k, pol_w);
      float a1[2] = {0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k < hv) {
          const uint4 xu = __ldg(xv + off + lane + 32 * k);
          const __nv_bfloat162* xh = (const __nv_bfloat162*)&xu;
          const __nv_bfloat162* h1 = (const __nv_bfloat162*)&w1[k];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 xf = __bfloat1622float2(xh[e]);
            const float2 f1 = __bfloat1622float2(h1[e]);
            a1[k & 1] = fmaf(f1.x, xf.x, a1[k & 1]);
            a1[k & 1] = fmaf(f1.y, xf.y, a1[k & 1]);
          }
        }
      }
      const float v1 = warp_sum(a1[0] + a1[1]);
      if (lane == 0) {
        if (half) a.y2[row - split_row] = v1;
        else a.y[row] = v1;
      }
    }
  } else {
    const int rpc = (a.Ntot + (int)nblk - 1) / (int)nblk;
    const int r0 = blockIdx.x * rpc, r1 = min(a.Ntot, r0 + rpc);
    const size_t row_bytes = (size_t)a.d * 2;
    const int CR = (int)((kFusedRing / 2) / row_bytes);  // rows per ring stage
    const int nrows = max(0, r1 - r0);
    const int nch = (nrows + CR - 1) / CR;
    const bf16* W = (const bf16*)a.wcatT;
    auto issue = [&](int c) {
      if (tid == 0) {
        const int ra = r0 + c * CR, rb = min(r1, ra + CR);
        uint8_t* dst = ring + (size_t)(c & 1) * CR * row_bytes;
        sm100::mbar_expect_tx(&gbar[c & 1], (uint32_t)((rb - ra) * row_bytes));
        for (int r = ra; r < rb; ++r)
          bulk_copy(dst + (size_t)(r - ra) * row_bytes, W + (size_t)r * a.d, (uint32_t)row_bytes, &gbar[c & 1]);
      }
    };
    __shared__ int abort_flag;
    if (tid == 0) abort_flag = 0;
    __syncthreads();
    if (nch > 0) issue(0);
    for (int c = 0; c < nch; ++c) {
      if (c + 1 < nch) issue(c + 1);
      const bool ok = sm100::mbar_wait(&gbar[c & 1], (c >> 1) & 1, (volatile int*)&abort_flag, a.status);
      // one decision for the whole CTA (a wait that ran out raised abort_flag for the others);
      // before leaving, let the copies in flight (chunks c and c + 1) land, within a fixed bound
      if (__syncthreads_or(!ok)) {
        if (tid == 0) {
          const unsigned long long t0 = sm100::globaltimer();
          for (int cc = c; cc < min(c + 2, nch); ++cc)
            while (!sm100::mbar_try_wait(&gbar[cc & 1], (cc >> 1) & 1) && sm100::globaltimer() - t0 < 100000000ull) {
            }
        }
        __syncthreads();
        return;
      }
      const int ra = r0 + c * CR, rb = min(r1, ra + CR);
      const bf16* wst = (const bf16*)(ring + (size_t)(c & 1) * CR * row_bytes);
      for (int r = ra + warp; r < rb; r += NW) {
        const bf16* wr = wst + (size_t)(r - ra) * a.d;
        float acc[kMaxDecodeBatch];
#pragma unroll
        for (int b = 0; b < kMaxDecodeBatch; ++b) acc[b] = 0.f;
        for (int i = lane * 8; i < a.d; i += 256) {
          const uint4 wu = *(const uint4*)(wr + i);
          const __nv_bfloat162* wh = (const __nv_bfloat162*)&wu;
          float wf[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(wh[e]);
            wf[2 * e] = f.x;
            wf[2 * e + 1] = f.y;
          }
#pragma unroll
          for (int b = 0; b < kMaxDecodeBatch; ++b) {
            if (b < a.B) {
              const uint4 xu = *(const uint4*)(sx + (size_t)b * a.d + i);
              const __nv_bfloat162* xh = (const __nv_bfloat162*)&xu;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(xh[e]);
                acc[b] = fmaf(wf[2 * e], f.x, acc[b]);
                acc[b] = fmaf(wf[2 * e + 1], f.y, acc[b]);
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < kMaxDecodeBatch; ++b) {
          if (b < a.B) {
            const float v = warp_sum(acc[b]);
            if (lane == 0) a.y[(size_t)b * a.Ntot + r] = v;
          }
        }
      }
      __syncthreads();  // stage (c & 1) is free for chunk c + 2
    }
  }
  if (tok_pf) dk::cp_wait<0>();  // the prefetched values, visible to the CTA after the barrier
  __shared__ unsigned long long s_step;  // index of this step since the counts were zeroed
  if (!grid_sync(a.sync, nblk, a.status, &s_step)) return;
  const unsigned long long step = s_step;
  unsigned long long* att_done = a.sync + 1;            // [B][Hkv] units of split attention finished
  unsigned long long* tok_done = a.sync + 1 + a.B * a.Hkv;  // [B] token-update CTAs finished

  // ---- B: split-KV attention over the old rows (units handed out from CTA ntok on), and the
  // token update, split over the first ntok CTAs
  {
    const int units = a.B * a.Hkv * a.nsplit;
    for (int u = ((int)blockIdx.x - ntok + (int)nblk) % (int)nblk; u < units; u += nblk) {
      const int split = u % a.nsplit, g = (u / a.nsplit) % a.Hkv, bi = u / (a.nsplit * a.Hkv);
      dk::attn_unit<DH>(a, split, g, bi, min(s_pos[bi], a.Lmax), a.y, a.Ntot, ring);
      count_done(&att_done[bi * a.Hkv + g]);
    }
    if ((int)blockIdx.x < ntok) {
      __shared__ TokenDecision td;
      for (int bi = 0; bi < a.B; ++bi) {
        const int pos = s_pos[bi];
        if (pos < 0 || pos >= a.Lmax) {
          if (blockIdx.x == 0 && threadIdx.x == 0) set_status(a.status, kStatusCapacity);
          count_done(&tok_done[bi]);
          continue;
        }
        const int c0 = min(width, (int)blockIdx.x * cpc), c1 = min(width, c0 + cpc);
        const int i0 = min(a.d, (int)blockIdx.x * dpc), i1 = min(a.d, i0 + dpc);
        token_decide<bf16>(a, bi, pos, &td, tok_pf ? &pf : nullptr, split_row);
        token_slice<bf16>(a, bi, pos, &td, c0, c1, i0, i1, tok_pf ? &pf : nullptr);
        count_done(&tok_done[bi]);
      }
      if (blockIdx.x == 0 && threadIdx.x < a.B && s_pos[threadIdx.x] < a.Lmax)
        a.pos[threadIdx.x] = s_pos[threadIdx.x] + 1;
    }
  }

  // ---- C: merge, and finish a block completed by this token: its projected sum becomes
  // the summary, its code the signs of the exact float64 d_model-space sum projected on P.  No grid
  // barrier: a CTA with work here waits only for the counts it needs (this step's split units of
  // the head's KV group, and the sequence's token-update CTAs); the others leave.
  const int ntok_run = ntok;
  for (int u = blockIdx.x; u < a.B * a.Hq; u += nblk) {
    const int bi = u / a.Hq, hq = u % a.Hq, g = hq / (a.Hq / a.Hkv);
    if (!wait_count(&att_done[bi * a.Hkv + g], (step + 1) * (unsigned long long)a.nsplit, a.status) ||
        !merge_unit<DH>(a, bi, hq, s_pos[bi], &tok_done[bi], (step + 1) * (unsigned long long)ntok_run))
      return;
  }
  {
    const int width = 2 * a.dkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int bi = 0; bi < a.B; ++bi) {
      const int pos = s_pos[bi];
      if (pos < 0 || pos >= a.Lmax || (pos + 1) % a.blk != 0 || pos / a.blk >= a.maxblk) continue;
      const int j = pos / a.blk;
      const float* bsum = a.blk_sum + (size_t)bi * width;
      float* summ = a.summ + ((size_t)bi * a.maxblk + j) * width;
      // bit k on CTA (nblk - 1 - k), one warp per bit
      const int k = (int)nblk - 1 - (int)blockIdx.x;
      // the block's sums are final once every token-update CTA of this step has finished
      const bool copies = (int)blockIdx.x * (int)blockDim.x < width;
      if ((copies || (k >= 0 && k < a.nb)) &&
          !wait_count(&tok_done[bi], (step + 1) * (unsigned long long)ntok_run, a.status))
        return;
      for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < width; c += nblk * blockDim.x) summ[c] = bsum[c];
      if (k >= 0 && k < a.nb && warp == 0) {
        const double* bx = a.blk_x + (size_t)bi * a.d;
        double v = 0.0;
        for (int i = lane; i < a.d; i += 32) v = fma(bx[i], a.pT64[(size_t)k * a.d + i], v);
        v = warp_sum_d(v);
        if (lane == 0 && v > 0.0) atomicOr(a.scode + (size_t)bi * a.maxblk + j, 1u << k);
      }
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(dk::NWD * 32, 2) decode_fused_kernel(DecodeArgs a) {
  decode_fused_body<DH>(a);
}

size_t decode_fused_smem(int B, int d) {
  return kFusedRing + (((size_t)B * d * 2 + 15) & ~(size_t)15) + 64 + (B == 1 ? kPfBytes : 0);
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
    const size_t sm = decode_fused_smem(a.B, a.d);
    if (sm > 227 * 1024) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = a.dh == 128 ? set_max_smem(decode_fused_kernel<128>, sm, s) : set_max_smem(decode_fused_kernel<64>, sm, s);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    int occ = 1;
    if (a.dh == 128) cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_fused_kernel<128>, dk::NWD * 32, sm);
    else cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_fused_kernel<64>, dk::NWD * 32, sm);
    if (occ < 1) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3((occ >= 2 ? 2 : 1) * sms);  // co-resident CTAs (two per SM when they fit)
    cfg.blockDim = dim3(dk::NWD * 32);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (a.dh == 128) e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<128>, a);
    else e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<64>, a);
    if (e != cudaSuccess) return e;
    MARK(1);
    MARK(2);
    MARK(3);
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
