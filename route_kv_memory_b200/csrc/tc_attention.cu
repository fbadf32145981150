// Causal GQA attention on tcgen05 tensor cores (MKA paper notes §3: one causal
// attention over the fused K/V; §4: online max-shift, partial sums rescaled by
// exp(mu_old - mu_new) when the running maximum grows).
//
// Persistent CTAs walk work items (sequence b, query head h, 128-row query tile i)
// longest first.  Per item the CTA streams the 128-key tiles j <= i of KV group
// g(h) = h / (Hq / Hkv):
//   warp 0      TMA: the Q tile once, then K_j and V_j into a 2-stage ring
//   warp 1      MMA: S_j = Q K_j^T into one of two TMEM score buffers, then
//               O += P_j V_j with P_j read from TMEM (A operand) and V_j from
//               shared memory as an MN-major B operand
//   warps 2-5   softmax, one query row per thread: scale, causal mask, running
//               maximum, P = exp2(s - m) packed to bf16 into TMEM over S_j; O is
//               rescaled (TMEM load, scale, store) only when the running maximum
//               of some row in the warp grew by more than 2^8, so the stale
//               maximum bounds P by 256; at the end O / l goes to global memory.
// TMEM: O in columns [0, 128), S/P buffers at [128, 256) and [256, 384).
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.cuh"

namespace mka {

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows);

namespace tca {

using namespace sm100;

constexpr int BQ = 128, BKV = 128;
constexpr int NTHREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 0, S_COL0 = 128;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

template <int DH>
struct Cfg {
  static constexpr int Q_BYTES = BQ * DH * 2;
  static constexpr int K_BYTES = BKV * DH * 2;
  static constexpr int V_BYTES = BKV * DH * 2;
  static constexpr int KV_BYTES = K_BYTES + V_BYTES;
  static constexpr int HALF = 128 * 64 * 2;  // one 128-row x 64-column swizzled box
  static constexpr int SMEM = Q_BYTES + 2 * KV_BYTES + 1024 + 256;
};

struct Work {
  int b, h, qt;
};
__device__ __forceinline__ Work work_item(int w, int B, int Hq, int nqt) {
  Work r;
  const int per = B * Hq;
  r.qt = nqt - 1 - w / per;  // longest rows first
  const int rem = w % per;
  r.h = rem % Hq;
  r.b = rem / Hq;
  return r;
}

// MN-major (V) descriptor: 8-key groups of 128-B rows 1024 B apart (stride byte
// offset), 64-column halves of the head dimension 16 KB apart (leading byte offset).
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(const void* tile) {
  const uint64_t addr = smem_u32(tile);
  uint64_t d = (addr >> 4) & 0x3FFFull;
  d |= (uint64_t)(16384 >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

template <int DH>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnArgs a, int* status) {
  using C = Cfg<DH>;
  constexpr int NH = DH / 64;  // 64-column boxes per row
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV);
  constexpr uint32_t IDESC_O = idesc_bf16_f32_bmn(BQ, DH);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::Q_BYTES;  // stage st: K at st*KV_BYTES, V at st*KV_BYTES + K_BYTES
  uint64_t* bars = (uint64_t*)(smem + C::Q_BYTES + 2 * C::KV_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;   // [2]
  uint64_t* kv_empty = bars + 4;  // [2]
  uint64_t* s_full = bars + 6;    // [2]
  uint64_t* p_full = bars + 8;    // [2]
  uint64_t* pv_done = bars + 10;
  uint64_t* o_full = bars + 11;
  uint64_t* o_empty = bars + 12;
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = (uint32_t*)(bars + 14);
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 4);
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const int nqt = (a.S + BQ - 1) / BQ;
  const int nwork = a.B * a.Hq * nqt;
  const int G = a.Hq / a.Hkv;
  const long long q_rows_per_b = a.q_bstride / a.q_ld;    // rows of the 2-D q view per sequence
  const long long kv_rows_per_b = a.kv_bstride / a.kv_ld;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int wi = 0, kvit = 0;
      for (int w = blockIdx.x; w < nwork; w += gridDim.x, ++wi) {
        const Work it = work_item(w, a.B, a.Hq, nqt);
        const int g = it.h / G;
        if (!mbar_wait(q_empty, (wi & 1) ^ 1, abort, status)) break;
        mbar_expect_tx(q_full, C::Q_BYTES);
        const int qy = (int)(it.b * q_rows_per_b) + it.qt * BQ;
        for (int hb = 0; hb < NH; ++hb) tma_load_2d(sQ + hb * C::HALF, &tmQ, q_full, it.h * DH + hb * 64, qy);
        const int nkv = it.qt + 1;
        bool ok = true;
        for (int j = 0; j < nkv; ++j, ++kvit) {
          const int st = kvit & 1;
          if (!mbar_wait(&kv_empty[st], ((kvit >> 1) & 1) ^ 1, abort, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&kv_full[st], C::KV_BYTES);
          uint8_t* kdst = sKV + st * C::KV_BYTES;
          const int ky = (int)(it.b * kv_rows_per_b) + j * BKV;
          for (int hb = 0; hb < NH; ++hb) {
            tma_load_2d(kdst + hb * C::HALF, &tmK, &kv_full[st], g * DH + hb * 64, ky);
            tma_load_2d(kdst + C::K_BYTES + hb * C::HALF, &tmV, &kv_full[st], g * DH + hb * 64, ky);
          }
        }
        if (!ok) break;
      }
      if (*abort) {  // let issued copies land (bounded) before unwinding
        const unsigned long long t0 = globaltimer();
        while (globaltimer() - t0 < 50000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int wi = 0, kvit = 0;
      for (int w = blockIdx.x; w < nwork; w += gridDim.x, ++wi) {
        const Work it = work_item(w, a.B, a.Hq, nqt);
        const int nkv = it.qt + 1;
        if (!mbar_wait(q_full, wi & 1, abort, status)) break;
        tc_fence_after();
        const uint64_t qd = sdesc_kmajor_sw128(sQ);
        bool ok = true;
        // S_0
        auto issue_s = [&](int kv_index) -> bool {
          const int st = kv_index & 1;
          if (!mbar_wait(&kv_full[st], (kv_index >> 1) & 1, abort, status)) return false;
          tc_fence_after();
          const uint64_t kd = sdesc_kmajor_sw128(sKV + st * C::KV_BYTES);
          const uint32_t d_tmem = tbase + S_COL0 + (kv_index & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint64_t off = (uint64_t)((kk >> 2) * (C::HALF >> 4) + (kk & 3) * 2);
            umma_bf16_ss(d_tmem, qd + off, kd + off, IDESC_S, kk != 0);
          }
          umma_commit(&s_full[kv_index & 1]);
          return true;
        };
        if (!issue_s(kvit)) break;
        for (int j = 0; j < nkv; ++j) {
          const int cur = kvit + j;
          if (j + 1 < nkv) {
            if (!issue_s(cur + 1)) {
              ok = false;
              break;
            }
          }
          if (j + 1 == nkv) umma_commit(q_empty);  // last use of Q by this item
          if (!mbar_wait(&p_full[cur & 1], (cur >> 1) & 1, abort, status)) {
            ok = false;
            break;
          }
          if (j == 0 && !mbar_wait(o_empty, (wi & 1) ^ 1, abort, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int st = cur & 1;
          const uint64_t vd = sdesc_mnmajor_sw128(sKV + st * C::KV_BYTES + C::K_BYTES);
          const uint32_t p_tmem = tbase + S_COL0 + (cur & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)
            umma_bf16_ts(tbase + O_COL, p_tmem + kk * 8, vd + (uint64_t)(kk * (2048 >> 4)), IDESC_O, (j | kk) != 0);
          umma_commit(pv_done);
          umma_commit(&kv_empty[st]);
        }
        if (!ok) break;
        kvit += nkv;
        umma_commit(o_full);
      }
      if (*abort) {
        umma_commit(drain);
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 100000000ull) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;                 // TMEM lane quadrant
    const int r = q4 * 32 + lane;            // row within the query tile
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;
    int wi = 0, sit = 0;
    for (int w = blockIdx.x; w < nwork; w += gridDim.x, ++wi) {
      const Work it = work_item(w, a.B, a.Hq, nqt);
      const int nkv = it.qt + 1;
      const int row = it.qt * BQ + r;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv; ++j, ++sit) {
        const int buf = sit & 1;
        if (!mbar_wait(&s_full[buf], (sit >> 1) & 1, abort, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t s_tmem = tbase + lane_off + S_COL0 + buf * 128;
        uint32_t sv[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_tmem + c * 32, *(uint32_t(*)[32])(sv + c * 32));
        tmem_ld_wait();
        const bool diag = (j == nkv - 1);
        const int key0 = j * BKV;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          float v = __uint_as_float(sv[c]) * sl2;
          if (diag && key0 + c > row) v = -INFINITY;
          sv[c] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
        // lazy rescale: move the reference maximum only when it is exceeded by > 2^8
        const bool need = mx > m_ref + RESCALE_THRESHOLD;
        float corr = 1.f;
        if (need) {
          corr = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
          m_ref = mx;
          l *= corr;
        }
        const unsigned vote = __ballot_sync(0xffffffffu, need && j > 0);
        if (vote) {  // rescale O rows of this warp once PV_{j-1} has landed
          if (!mbar_wait(pv_done, (sit - 1) & 1, abort, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < DH; c += 32) {
            uint32_t ov[32];
            tmem_ld32(tbase + lane_off + O_COL + c, ov);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
            uint32_t lo[16], hi[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              lo[e] = ov[e];
              hi[e] = ov[16 + e];
            }
            tmem_st16(tbase + lane_off + O_COL + c, lo);
            tmem_st16(tbase + lane_off + O_COL + c + 16, hi);
          }
        }
        // P = exp2(s - m_ref), packed bf16 pairs, written over the first 64 columns of S
        const float mr = m_ref;
        float lsum = 0.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = exp2f(__uint_as_float(sv[c4 * 32 + 2 * e]) - mr);
            const float p1 = exp2f(__uint_as_float(sv[c4 * 32 + 2 * e + 1]) - mr);
            lsum += p0 + p1;
            __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
            pk[e] = *(uint32_t*)&hb;
          }
          tmem_st16(s_tmem + c4 * 16, pk);
        }
        l += lsum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[buf]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> global
      if (!mbar_wait(o_full, wi & 1, abort, status)) break;
      tc_fence_after();
      const float inv = 1.f / l;
      bf16* orow = (bf16*)a.o + (size_t)it.b * a.o_bstride + (size_t)row * a.o_ld + (size_t)it.h * DH;
#pragma unroll
      for (int c = 0; c < DH; c += 32) {
        uint32_t ov[32];
        tmem_ld32(tbase + lane_off + O_COL + c, ov);
        tmem_ld_wait();
        if (row < a.S) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            uint32_t* wv = (uint32_t*)&u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(ov[v * 8 + 2 * e]) * inv,
                                                        __uint_as_float(ov[v * 8 + 2 * e + 1]) * inv);
              wv[e] = *(uint32_t*)&hb;
            }
            *(uint4*)(orow + c + v * 8) = u;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
}

}  // namespace tca

cudaError_t attention_prefill_tc(const AttnArgs& a, int* status, cudaStream_t s) {
  if (a.B <= 0 || a.S <= 0) return cudaSuccess;
  if ((a.dh != 64 && a.dh != 128) || (a.q_ld % 8) || (a.kv_ld % 8) || (a.o_ld % 8) || (a.q_bstride % a.q_ld) ||
      (a.kv_bstride % a.kv_ld))
    return cudaErrorInvalidValue;
  const long long q_rows = (long long)a.B * (a.q_bstride / a.q_ld);
  const long long kv_rows = (long long)a.B * (a.kv_bstride / a.kv_ld);
  if (q_rows >= (1LL << 31) || kv_rows >= (1LL << 31)) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  cudaError_t e = make_tmap_bf16(&tq, a.q, (int)q_rows, a.Hq * a.dh, a.q_ld, tca::BQ);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tk, a.k, (int)kv_rows, a.Hkv * a.dh, a.kv_ld, tca::BKV);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tv, a.v, (int)kv_rows, a.Hkv * a.dh, a.kv_ld, tca::BKV);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int nwork = a.B * a.Hq * ((a.S + tca::BQ - 1) / tca::BQ);
  const int grid = nwork < sms ? nwork : sms;
  if (a.dh == 128) {
    e = set_max_smem(tca::attn_tc_kernel<128>, tca::Cfg<128>::SMEM, s);
    if (e != cudaSuccess) return e;
    tca::attn_tc_kernel<128><<<grid, tca::NTHREADS, tca::Cfg<128>::SMEM, s>>>(tq, tk, tv, a, status);
  } else {
    e = set_max_smem(tca::attn_tc_kernel<64>, tca::Cfg<64>::SMEM, s);
    if (e != cudaSuccess) return e;
    tca::attn_tc_kernel<64><<<grid, tca::NTHREADS, tca::Cfg<64>::SMEM, s>>>(tq, tk, tv, a, status);
  }
  return cudaGetLastError();
}

}  // namespace mka
