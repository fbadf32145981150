// Backward of the causal GQA attention on tcgen05 tensor cores (the layer's attention, MKA paper
// notes §3; its online max-shift, §4, leaves each row's normaliser lse = m + log2(l), which the
// forward keeps).  With P = 2^(s * scale * log2e - lse) recomputed from the scores and
// D = rowsum(dO * O):
//   dS = P * (dO V^T - D),  dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO,
// dK and dV summed over the G = Hq / Hkv query heads of a KV group.  Two kernels, no atomics:
//
//   attn_bwd_dq_kernel    per (sequence, query head, 128-row query tile), streaming the key
//                         tiles j <= its own (K in a 3-stage ring, V in a 2-stage one):
//                         S = Q K_j^T and dP = dO V_j^T into TMEM, the compute warps turn them
//                         into scale * dS (bf16, packed over dP), then dQ += dS K_j with dS read
//                         from TMEM and K_j as an MN-major operand.
//   attn_bwd_dkdv_kernel  per (sequence, KV group, 128-key tile), K and V staying in shared
//                         memory while the query tiles t >= its own of all G heads stream through
//                         two 2-stage rings (Q with its lse and D rows; dO): S^T = K Q^T and
//                         dP^T = V dO^T into TMEM, the compute warps write P^T and dS^T (bf16)
//                         over dP^T, then dK += dS^T Q and dV += P^T dO accumulate in TMEM (dK
//                         takes its factor scale when it is written out).
// Warp 0 loads (TMA), warp 1 issues the MMAs, warps 2-9 compute: two warps per TMEM lane quadrant,
// each taking 64 of a row's 128 columns; a warp packs its bf16 results into the first 32 columns of
// its own 64-column range (so neither half overwrites what the other still reads), and the MMAs
// read K-step kk (16 columns) at packed column kk * 8 + (kk >= 4 ? 32 : 0).
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.cuh"

namespace mka {

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows);

namespace tcb {

using namespace sm100;

constexpr int BT = 128;  // rows of every tile (query and key)
constexpr int NTHREADS = 320;
constexpr int NCOMPUTE = 8;  // compute warps

// TMEM column (32-bit) of K-step kk of a packed bf16 A operand written by the two column halves.
__device__ __forceinline__ uint32_t packed_col(int kk) { return (uint32_t)(kk * 8 + (kk >= 4 ? 32 : 0)); }
constexpr uint32_t TMEM_COLS = 512;

template <int DH>
struct Cfg {
  static constexpr int NH = DH / 64;             // 64-column boxes per row
  static constexpr int TILE = BT * DH * 2;       // one 128-row bf16 tile
  static constexpr int HALF = BT * 64 * 2;       // one 128-row x 64-column swizzled box
  static constexpr int VEC = BT * 4;             // 128 floats (lse or D of a query tile)
  static constexpr int QSTAGE = TILE + 1024;     // dK/dV Q ring stage: Q, lse, D (1024-aligned)
  static constexpr int KST = 3, VST = 2;           // dQ kernel: K ring stages, V ring stages
  static constexpr int SMEM_DQ = (2 + KST + VST) * TILE + 1024 + 256;
  static constexpr int SMEM_DKDV = 2 * TILE + 2 * QSTAGE + 2 * TILE + 1024 + 256;
};

__device__ __forceinline__ int snake(int r, int grid, int cta, int nwork) {
  const int w = r * grid + ((r & 1) ? grid - 1 - cta : cta);
  return w < nwork ? w : -1;
}

// Offset of K-step kk (16 elements of the K dimension) in a K-major 128B-swizzled tile descriptor.
__device__ __forceinline__ uint64_t kstep(int kk, int half_bytes) {
  return (uint64_t)((kk >> 2) * (half_bytes >> 4) + (kk & 3) * 2);
}

// scale * dS (or P) for 32 columns, packed as bf16 pairs.
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *(uint32_t*)&h;
}

// ============================================================================ dQ
template <int DH>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       AttnBwdArgs a, int* status) {
  using C = Cfg<DH>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BT, BT);
  constexpr uint32_t IDESC_D = idesc_bf16_f32_bmn(BT, DH);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sdO = smem + C::TILE;
  // K and V rings of their own: K_j is read by S(j) and dQ(j), V_j only by dP(j), which ends a
  // whole step earlier, so K takes one stage more
  uint8_t* sK = smem + 2 * C::TILE;                // stage st at st * TILE
  uint8_t* sV = smem + (2 + C::KST) * C::TILE;
  uint64_t* bars = (uint64_t*)(smem + (2 + C::KST + C::VST) * C::TILE);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;                 // [KST]
  uint64_t* k_empty = k_full + C::KST;         // [KST]
  uint64_t* v_full = k_empty + C::KST;         // [VST]
  uint64_t* v_empty = v_full + C::VST;         // [VST]
  uint64_t* s_full = v_empty + C::VST;
  uint64_t* p_full = s_full + 1;
  uint64_t* dq_full = s_full + 2;
  uint64_t* dq_empty = s_full + 3;
  uint64_t* drain = s_full + 4;
  uint64_t* s_free = s_full + 5;   // the compute warps hold S in registers: its columns are free
  uint64_t* dp_full = s_full + 6;  // dP has landed
  uint32_t* tmem_slot = (uint32_t*)(s_full + 7);
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::KST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::VST; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, NCOMPUTE);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, NCOMPUTE);
    mbar_init(s_free, NCOMPUTE);
    mbar_init(dp_full, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  constexpr uint32_t S_COL = 0, P_COL = 128, Q_COL = 256;  // S (then scale*dS), dP, dQ

  const int nqt = (a.S + BT - 1) / BT;
  const int nwork = a.B * a.Hq * nqt;
  const int G = a.Hq / a.Hkv;
  // item w: query tile qt (longest first), head h, sequence b
  auto item = [&](int w, int& b, int& h, int& qt) {
    const int per = a.B * a.Hq;
    qt = nqt - 1 - w / per;
    const int rem = w % per;
    h = rem % a.Hq;
    b = rem / a.Hq;
  };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmdO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int kvit = 0;
      bool ok = true;
      for (int rr = 0; ok; ++rr) {
        const int w = snake(rr, gridDim.x, blockIdx.x, nwork);
        if (w < 0) break;
        int b, h, qt;
        item(w, b, h, qt);
        if (!mbar_wait(q_empty, (rr & 1) ^ 1, abort, status)) break;
        mbar_expect_tx(q_full, 2 * C::TILE);
        for (int hb = 0; hb < C::NH; ++hb) {
          tma_load_2d(sQ + hb * C::HALF, &tmQ, q_full, h * DH + hb * 64, b * a.S + qt * BT);
          tma_load_2d(sdO + hb * C::HALF, &tmdO, q_full, h * DH + hb * 64, b * a.S + qt * BT);
        }
        for (int j = 0; j <= qt; ++j, ++kvit) {
          const int ks = kvit % C::KST, vs = kvit % C::VST;
          if (!mbar_wait(&k_empty[ks], ((kvit / C::KST) & 1) ^ 1, abort, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&k_full[ks], C::TILE);
          for (int hb = 0; hb < C::NH; ++hb)
            tma_load_2d(sK + ks * C::TILE + hb * C::HALF, &tmK, &k_full[ks], (h / G) * DH + hb * 64, b * a.S + j * BT);
          if (!mbar_wait(&v_empty[vs], ((kvit / C::VST) & 1) ^ 1, abort, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&v_full[vs], C::TILE);
          for (int hb = 0; hb < C::NH; ++hb)
            tma_load_2d(sV + vs * C::TILE + hb * C::HALF, &tmV, &v_full[vs], (h / G) * DH + hb * 64, b * a.S + j * BT);
        }
      }
    }
  } else if (warp == 1) {  // the whole warp runs the MMA role; one elected lane issues
    const uint64_t qd = sdesc_kmajor_sw128(sQ), dod = sdesc_kmajor_sw128(sdO);
    int kvit = 0, pc = 0, sf = 0;
    bool ok = true, first = true;
    // S = Q K^T for the key tile in K ring slot `st`
    auto issue_s = [&](int st) {
      const uint64_t kd = sdesc_kmajor_sw128(sK + st * C::TILE);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk)
        umma_bf16_ss_w(tbase + S_COL, qd + kstep(kk, C::HALF), kd + kstep(kk, C::HALF), IDESC_S, kk != 0);
      umma_commit_w(s_full);
    };
    // dP = dO V^T, V in V ring slot `st` (freed when dP lands)
    auto issue_dp = [&](int st) {
      const uint64_t vd = sdesc_kmajor_sw128(sV + st * C::TILE);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk)
        umma_bf16_ss_w(tbase + P_COL, dod + kstep(kk, C::HALF), vd + kstep(kk, C::HALF), IDESC_S, kk != 0);
      umma_commit_w(dp_full);
      umma_commit_w(&v_empty[st]);
    };
    // dQ += scale*dS K_j, dS packed over the dP columns
    auto issue_dq = [&](int st, bool acc) {
      const uint64_t kd = sdesc_mnmajor_sw128(sK + st * C::TILE);
#pragma unroll
      for (int kk = 0; kk < BT / 16; ++kk)
        umma_bf16_ts_w(tbase + Q_COL, tbase + P_COL + packed_col(kk), kd + (uint64_t)(kk * (2048 >> 4)), IDESC_D,
                     (acc || kk) ? 1u : 0u);
    };
    // S(j+1) goes in as soon as the compute warps hold S(j) in registers, so their exponentials
    // of tile j+1 run under dQ(j) and dP(j+1); dP(j+1) follows dQ(j), which reads dS(j) over dP.
    for (int rr = 0; ok; ++rr) {
      const int w = snake(rr, gridDim.x, blockIdx.x, nwork);
      if (w < 0) break;
      int b, h, qt;
      item(w, b, h, qt);
      const int n = qt + 1;
      if (!mbar_wait_warp(q_full, rr & 1, abort, status)) break;
      if (!mbar_wait_warp(&k_full[kvit % C::KST], (kvit / C::KST) & 1, abort, status)) break;
      if (!first) {
        if (!mbar_wait_warp(s_free, sf & 1, abort, status)) break;
        ++sf;
      }
      first = false;
      tc_fence_after();
      issue_s(kvit % C::KST);
      if (!mbar_wait_warp(&v_full[kvit % C::VST], (kvit / C::VST) & 1, abort, status)) break;
      tc_fence_after();
      issue_dp(kvit % C::VST);
      if (n == 1) umma_commit_w(q_empty);
      for (int j = 0; j < n; ++j) {
        const int cur = kvit + j, nxt = cur + 1;
        if (j + 1 < n) {
          if (!mbar_wait_warp(&k_full[nxt % C::KST], (nxt / C::KST) & 1, abort, status)) { ok = false; break; }
          if (!mbar_wait_warp(s_free, sf & 1, abort, status)) { ok = false; break; }
          ++sf;
          tc_fence_after();
          issue_s(nxt % C::KST);
        }
        if (!mbar_wait_warp(p_full, pc & 1, abort, status)) { ok = false; break; }
        ++pc;
        if (j == 0 && !mbar_wait_warp(dq_empty, (rr & 1) ^ 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        issue_dq(cur % C::KST, j > 0);
        umma_commit_w(&k_empty[cur % C::KST]);
        if (j + 1 < n) {
          if (!mbar_wait_warp(&v_full[nxt % C::VST], (nxt / C::VST) & 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          issue_dp(nxt % C::VST);
          if (j + 2 == n) umma_commit_w(q_empty);  // Q and dO's last use
        }
      }
      if (!ok) break;
      umma_commit_w(dq_full);
      kvit += n;
    }
    if (__any_sync(0xffffffffu, *abort)) {
      umma_commit_w(drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 100000000ull) {
      }
    }
  } else {
    const int q4 = warp & 3, half = (warp - 2) >> 2;  // lane quadrant; columns [64 half, 64 half + 64)
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_tmem = tbase + lane_off + S_COL, p_tmem = tbase + lane_off + P_COL;
    const uint32_t q_tmem = tbase + lane_off + Q_COL + half * (DH / 2);
    const float sl2 = a.scale * 1.4426950408889634f, l2scale = log2f(a.scale);
    int sit = 0;
    for (int rr = 0;; ++rr) {
      const int w = snake(rr, gridDim.x, blockIdx.x, nwork);
      if (w < 0) break;
      int b, h, qt;
      item(w, b, h, qt);
      const int n = qt + 1, row = qt * BT + r;
      const bool valid = row < a.S;
      const size_t li = ((size_t)b * a.Hq + h) * a.lse_ld + (valid ? row : 0);
      // scale * P = 2^(s sl2 - lse + log2 scale): dQ's factor scale rides in the exponent
      const float lse2 = (valid ? a.lse[li] : 0.f) - l2scale, drow = valid ? a.dsum[li] : 0.f;
      const float2 sl2v = make_float2(sl2, sl2), nlse2v = make_float2(-lse2, -lse2);
      const float2 ndrowv = make_float2(-drow, -drow);
      bool ok = true;
      for (int j = 0; j < n; ++j, ++sit) {
        if (!mbar_wait_warp(s_full, sit & 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        const int lim = valid ? row - j * BT : -1;  // keys c > lim are masked (all, for a padding row)
        const bool diag = __any_sync(0xffffffffu, j == n - 1 || !valid);  // warp-uniform
        // phase 1: this half's 64 scores into registers (S's columns are then free for S(j+1)),
        // P = 2^(s sl2 - lse) in float32
        uint32_t sv[2][32];
        tmem_ld32(s_tmem + 64 * half, sv[0]);
        tmem_ld32(s_tmem + 64 * half + 32, sv[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * half + cc;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 x2 = __ffma2_rn(make_float2(__uint_as_float(sv[cc][2 * e]), __uint_as_float(sv[cc][2 * e + 1])),
                                         sl2v, nlse2v);
            float p0 = ex2(x2.x), p1 = ex2(x2.y);
            if (diag) {
              const int k0 = c * 32 + 2 * e;
              p0 = k0 <= lim ? p0 : 0.f;
              p1 = k0 + 1 <= lim ? p1 : 0.f;
            }
            sv[cc][2 * e] = __float_as_uint(p0);
            sv[cc][2 * e + 1] = __float_as_uint(p1);
          }
        }
        // phase 2: scale dS = (scale P) (dP - D), packed over the first 32 of this half's dP columns
        if (!mbar_wait_warp(dp_full, sit & 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        uint32_t pv[2][32];
        tmem_ld32(p_tmem + 64 * half, pv[0]);
        tmem_ld32(p_tmem + 64 * half + 32, pv[1]);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 d2 = __fadd2_rn(make_float2(__uint_as_float(pv[cc][2 * e]), __uint_as_float(pv[cc][2 * e + 1])),
                                         ndrowv);
            const float2 r2 = __fmul2_rn(make_float2(__uint_as_float(sv[cc][2 * e]), __uint_as_float(sv[cc][2 * e + 1])), d2);
            pk[e] = pack2(r2.x, r2.y);
          }
          tmem_st16(p_tmem + 64 * half + cc * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      if (!mbar_wait_warp(dq_full, rr & 1, abort, status)) break;
      tc_fence_after();
      float* dst = a.dq + ((size_t)b * a.S + (valid ? row : 0)) * (size_t)(a.Hq * DH) + (size_t)h * DH +
                   half * (DH / 2);
#pragma unroll
      for (int c = 0; c < DH / 2; c += 32) {
        uint32_t v[32];
        tmem_ld32(q_tmem + c, v);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t u[8] = {v[8 * e], v[8 * e + 1], v[8 * e + 2], v[8 * e + 3],
                                   v[8 * e + 4], v[8 * e + 5], v[8 * e + 6], v[8 * e + 7]};
            st_global_v8(dst + c + 8 * e, u);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
    if (lane == 0) linger_after_abort(abort);  // copies issued before a role gave up land first
  }
}

// ============================================================================ dK, dV
template <int DH>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                         const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         AttnBwdArgs a, int* status) {
  using C = Cfg<DH>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BT, BT);
  constexpr uint32_t IDESC_D = idesc_bf16_f32_bmn(BT, DH);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::TILE;
  // Q (with its lse and D rows) and dO in rings of their own: dK(s), the last reader of Q(s), is
  // issued before dV(s), so Q(s + 2), all that S^T(s + 2) needs, loads while dV(s) runs
  uint8_t* sQ = smem + 2 * C::TILE;                  // stage st at st * QSTAGE: Q, lse[128], D[128]
  uint8_t* sdO = sQ + 2 * C::QSTAGE;                 // stage st at st * TILE
  uint64_t* bars = (uint64_t*)(sdO + 2 * C::TILE);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;    // [2]
  uint64_t* q_empty = bars + 4;   // [2]
  uint64_t* do_full = bars + 6;   // [2]
  uint64_t* do_empty = bars + 8;  // [2]
  uint64_t* s_full = bars + 10;
  uint64_t* p_full = bars + 11;
  uint64_t* acc_full = bars + 12;
  uint64_t* acc_empty = bars + 13;
  uint64_t* drain = bars + 14;
  uint64_t* s_free = bars + 15;   // the compute warps hold S^T in registers: its columns are free
  uint64_t* dp_full = bars + 16;  // dP^T has landed
  uint32_t* tmem_slot = (uint32_t*)(bars + 17);
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&do_full[i], 1);
      mbar_init(&do_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, NCOMPUTE);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, NCOMPUTE);
    mbar_init(s_free, NCOMPUTE);
    mbar_init(dp_full, 1);
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  constexpr uint32_t S_COL = 0, P_COL = 128, V_COL = 256, K_COL = 256 + DH;  // S^T/P^T, dP^T/dS^T, dV, dK

  const int nqt = (a.S + BT - 1) / BT;
  const int nwork = a.B * a.Hkv * nqt;
  const int G = a.Hq / a.Hkv;
  // item w: key tile kt (longest first: the most query tiles), KV group g, sequence b; its steps
  // run the G heads (outer) over the query tiles kt..nqt-1 (inner)
  auto item = [&](int w, int& b, int& g, int& kt) {
    const int per = a.B * a.Hkv;
    kt = w / per;
    const int rem = w % per;
    g = rem % a.Hkv;
    b = rem / a.Hkv;
  };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmdO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int qdit = 0;
      bool ok = true;
      for (int rr = 0; ok; ++rr) {
        const int w = snake(rr, gridDim.x, blockIdx.x, nwork);
        if (w < 0) break;
        int b, g, kt;
        item(w, b, g, kt);
        if (!mbar_wait(kv_empty, (rr & 1) ^ 1, abort, status)) break;
        mbar_expect_tx(kv_full, 2 * C::TILE);
        for (int hb = 0; hb < C::NH; ++hb) {
          tma_load_2d(sK + hb * C::HALF, &tmK, kv_full, g * DH + hb * 64, b * a.S + kt * BT);
          tma_load_2d(sV + hb * C::HALF, &tmV, kv_full, g * DH + hb * 64, b * a.S + kt * BT);
        }
        const int nq = nqt - kt;
        for (int s = 0; s < G * nq; ++s, ++qdit) {
          const int h = g * G + s / nq, qt = kt + s % nq, st = qdit & 1, ph = ((qdit >> 1) & 1) ^ 1;
          if (!mbar_wait(&q_empty[st], ph, abort, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&q_full[st], C::TILE + 2 * C::VEC);
          uint8_t* dst = sQ + st * C::QSTAGE;
          for (int hb = 0; hb < C::NH; ++hb)
            tma_load_2d(dst + hb * C::HALF, &tmQ, &q_full[st], h * DH + hb * 64, b * a.S + qt * BT);
          const size_t li = ((size_t)b * a.Hq + h) * a.lse_ld + (size_t)qt * BT;
          bulk_load(dst + C::TILE, a.lse + li, C::VEC, &q_full[st]);
          bulk_load(dst + C::TILE + C::VEC, a.dsum + li, C::VEC, &q_full[st]);
          if (!mbar_wait(&do_empty[st], ph, abort, status)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&do_full[st], C::TILE);
          for (int hb = 0; hb < C::NH; ++hb)
            tma_load_2d(sdO + st * C::TILE + hb * C::HALF, &tmdO, &do_full[st], h * DH + hb * 64, b * a.S + qt * BT);
        }
      }
    }
  } else if (warp == 1) {  // the whole warp runs the MMA role; one elected lane issues
    const uint64_t kd = sdesc_kmajor_sw128(sK), vd = sdesc_kmajor_sw128(sV);
    int qdit = 0, pc = 0, sf = 0;
    bool ok = true, first = true;
    // S^T = K Q^T for the query stage `st`
    auto issue_s = [&](int st) {
      const uint64_t qd = sdesc_kmajor_sw128(sQ + st * C::QSTAGE);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk)
        umma_bf16_ss_w(tbase + S_COL, kd + kstep(kk, C::HALF), qd + kstep(kk, C::HALF), IDESC_S, kk != 0);
      umma_commit_w(s_full);
    };
    // dP^T = V dO^T
    auto issue_dp = [&](int st) {
      const uint64_t dod = sdesc_kmajor_sw128(sdO + st * C::TILE);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk)
        umma_bf16_ss_w(tbase + P_COL, vd + kstep(kk, C::HALF), dod + kstep(kk, C::HALF), IDESC_S, kk != 0);
      umma_commit_w(dp_full);
    };
    // dK += dS^T Q, then dV += P^T dO, each freeing its ring slot; the compute warps pack
    // P^T and dS^T over the dP^T columns: K-step kk (16 queries) of P^T at
    // 64 (kk / 4) + 32 ((kk / 2) % 2) + 8 (kk % 2), of dS^T 16 further
    auto issue_acc = [&](int st, bool acc) {
      const uint64_t dq = sdesc_mnmajor_sw128(sQ + st * C::QSTAGE);
      const uint64_t dd = sdesc_mnmajor_sw128(sdO + st * C::TILE);
#pragma unroll
      for (int kk = 0; kk < BT / 16; ++kk) {
        const uint32_t pcol = P_COL + 64 * (kk >> 2) + 32 * ((kk >> 1) & 1) + 8 * (kk & 1);
        umma_bf16_ts_w(tbase + K_COL, tbase + pcol + 16, dq + (uint64_t)(kk * (2048 >> 4)), IDESC_D,
                     (acc || kk) ? 1u : 0u);
      }
      umma_commit_w(&q_empty[st]);
#pragma unroll
      for (int kk = 0; kk < BT / 16; ++kk) {
        const uint32_t pcol = P_COL + 64 * (kk >> 2) + 32 * ((kk >> 1) & 1) + 8 * (kk & 1);
        umma_bf16_ts_w(tbase + V_COL, tbase + pcol, dd + (uint64_t)(kk * (2048 >> 4)), IDESC_D, (acc || kk) ? 1u : 0u);
      }
      umma_commit_w(&do_empty[st]);
    };
    // S^T(s+1) goes in as soon as the compute warps hold S^T(s) in registers, so their
    // exponentials of step s+1 run under dV / dK(s) and dP^T(s+1); dP^T(s+1) follows dV / dK(s),
    // which read P^T(s) and dS^T(s) over the dP^T columns.
    for (int rr = 0; ok; ++rr) {
      const int w = snake(rr, gridDim.x, blockIdx.x, nwork);
      if (w < 0) break;
      int b, g, kt;
      item(w, b, g, kt);
      const int n = G * (nqt - kt);
      if (!mbar_wait_warp(kv_full, rr & 1, abort, status)) break;
      if (!mbar_wait_warp(&q_full[qdit & 1], (qdit >> 1) & 1, abort, status)) break;
      if (!first) {
        if (!mbar_wait_warp(s_free, sf & 1, abort, status)) break;
        ++sf;
      }
      first = false;
      tc_fence_after();
      issue_s(qdit & 1);
      if (!mbar_wait_warp(&do_full[qdit & 1], (qdit >> 1) & 1, abort, status)) break;
      tc_fence_after();
      issue_dp(qdit & 1);
      for (int s = 0; s < n; ++s) {
        const int cur = qdit + s, st = cur & 1, nst = (cur + 1) & 1, nph = ((cur + 1) >> 1) & 1;
        if (s + 1 < n) {
          if (!mbar_wait_warp(&q_full[nst], nph, abort, status)) { ok = false; break; }
          if (!mbar_wait_warp(s_free, sf & 1, abort, status)) { ok = false; break; }
          ++sf;
          tc_fence_after();
          issue_s(nst);
        }
        if (!mbar_wait_warp(p_full, pc & 1, abort, status)) { ok = false; break; }
        ++pc;
        if (s == 0 && !mbar_wait_warp(acc_empty, (rr & 1) ^ 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        issue_acc(st, s > 0);
        if (s + 1 < n) {
          if (!mbar_wait_warp(&do_full[nst], nph, abort, status)) { ok = false; break; }
          tc_fence_after();
          issue_dp(nst);
        }
      }
      if (!ok) break;
      umma_commit_w(kv_empty);
      umma_commit_w(acc_full);
      qdit += n;
    }
    if (__any_sync(0xffffffffu, *abort)) {
      umma_commit_w(drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 100000000ull) {
      }
    }
  } else {
    const int q4 = warp & 3, half = (warp - 2) >> 2;  // lane quadrant; query columns [64 half, 64 half + 64)
    const int r = q4 * 32 + lane;  // key row of the tile
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_tmem = tbase + lane_off + S_COL, p_tmem = tbase + lane_off + P_COL;
    const float sl2 = a.scale * 1.4426950408889634f;
    int sit = 0;
    for (int rr = 0;; ++rr) {
      const int w = snake(rr, gridDim.x, blockIdx.x, nwork);
      if (w < 0) break;
      int b, g, kt;
      item(w, b, g, kt);
      const int nq = nqt - kt, n = G * nq, key = kt * BT + r;
      bool ok = true;
      for (int s = 0; s < n; ++s, ++sit) {
        const int qt = kt + s % nq, st = sit & 1;
        // the stage's lse and D rows: landed with its Q (the stage is not refilled before this
        // step's dK MMAs, which wait for this warp)
        if (!mbar_wait_warp(&q_full[st], (sit >> 1) & 1, abort, status)) { ok = false; break; }
        if (!mbar_wait_warp(s_full, sit & 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        const float* lse2 = (const float*)(sQ + st * C::QSTAGE + C::TILE);
        const float* dsum = lse2 + BT;
        // query column c is used iff it is a real row at or after this key: q0 + c < S, q0 + c >= key
        const int q0 = qt * BT, cmax = a.S - q0, cmin = key - q0;
        const bool masked = __any_sync(0xffffffffu, cmin > 64 * half || cmax < 64 * half + 64);  // warp-uniform
        const float2 sl2v = make_float2(sl2, sl2);
        // phase 1: this half's 64 scores into registers (S^T's columns are then free for the next
        // step), P^T = 2^(s sl2 - lse) in float32
        uint32_t sv[2][32];
        tmem_ld32(s_tmem + 64 * half, sv[0]);
        tmem_ld32(s_tmem + 64 * half + 32, sv[1]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * half + cc;
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {  // lse of four query columns per shared-memory load
            const float4 l4 = *(const float4*)(lse2 + c * 32 + 4 * e4);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int e = 2 * e4 + k, c0 = c * 32 + 2 * e;
              const float2 nl = k ? make_float2(-l4.z, -l4.w) : make_float2(-l4.x, -l4.y);
              const float2 x2 = __ffma2_rn(make_float2(__uint_as_float(sv[cc][2 * e]), __uint_as_float(sv[cc][2 * e + 1])),
                                           sl2v, nl);
              float p0 = ex2(x2.x), p1 = ex2(x2.y);
              if (masked) {
                p0 = (c0 < cmax && c0 >= cmin) ? p0 : 0.f;
                p1 = (c0 + 1 < cmax && c0 + 1 >= cmin) ? p1 : 0.f;
              }
              sv[cc][2 * e] = __float_as_uint(p0);
              sv[cc][2 * e + 1] = __float_as_uint(p1);
            }
          }
        }
        // phase 2: dS^T = P^T (dP^T - D) (dK takes its factor scale in the epilogue); P^T and dS^T
        // packed over this half's dP^T columns,
        // chunk cc at [32 cc, 32 cc + 16) and [32 cc + 16, 32 cc + 32) of the half
        if (!mbar_wait_warp(dp_full, sit & 1, abort, status)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {  // chunk by chunk: a chunk's outputs go only over its own inputs
          const int c = 2 * half + cc;
          uint32_t pv[32];
          tmem_ld32(p_tmem + 64 * half + 32 * cc, pv);
          tmem_ld_wait();
          uint32_t pp[16], pd[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 d4 = *(const float4*)(dsum + c * 32 + 4 * e4);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int e = 2 * e4 + k;
              const float2 nd = k ? make_float2(-d4.z, -d4.w) : make_float2(-d4.x, -d4.y);
              const float2 p2 = make_float2(__uint_as_float(sv[cc][2 * e]), __uint_as_float(sv[cc][2 * e + 1]));
              pp[e] = pack2(p2.x, p2.y);
              const float2 d2 = __fadd2_rn(make_float2(__uint_as_float(pv[2 * e]), __uint_as_float(pv[2 * e + 1])), nd);
              const float2 r2 = __fmul2_rn(p2, d2);
              pd[e] = pack2(r2.x, r2.y);
            }
          }
          tmem_st16(p_tmem + 64 * half + 32 * cc, pp);
          tmem_st16(p_tmem + 64 * half + 32 * cc + 16, pd);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      if (!mbar_wait_warp(acc_full, rr & 1, abort, status)) break;
      tc_fence_after();
      const bool valid = key < a.S;
      const int wkv = 2 * a.Hkv * DH;
      float* dst = a.dkv + ((size_t)b * a.S + (valid ? key : 0)) * (size_t)wkv + (size_t)g * DH;
      {  // the first warpgroup writes dK (columns [0, dkv)) = scale * sum dS^T Q, the second dV ([dkv, 2 dkv))
        const uint32_t src = tbase + lane_off + (half ? V_COL : K_COL);
        float* d = dst + (half ? a.Hkv * DH : 0);
        const float f = half ? 1.f : a.scale;
#pragma unroll
        for (int c = 0; c < DH; c += 32) {
          uint32_t v[32];
          tmem_ld32(src + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
          if (valid) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t u[8] = {v[8 * e], v[8 * e + 1], v[8 * e + 2], v[8 * e + 3],
                                     v[8 * e + 4], v[8 * e + 5], v[8 * e + 6], v[8 * e + 7]};
              st_global_v8(d + c + 8 * e, u);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
    if (lane == 0) linger_after_abort(abort);  // copies issued before a role gave up land first
  }
}

}  // namespace tcb

template <int DH>
static cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                              const CUtensorMap& tv, const AttnBwdArgs& a, int* status, int sms, cudaStream_t s) {
  using C = tcb::Cfg<DH>;
  const int nqt = (a.S + tcb::BT - 1) / tcb::BT;
  cudaError_t e = set_max_smem(tcb::attn_bwd_dkdv_kernel<DH>, C::SMEM_DKDV, s);
  if (e != cudaSuccess) return e;
  const int nkv = a.B * a.Hkv * nqt, nq = a.B * a.Hq * nqt;
  tcb::attn_bwd_dkdv_kernel<DH><<<nkv < sms ? nkv : sms, tcb::NTHREADS, C::SMEM_DKDV, s>>>(tq, tdo, tk, tv, a, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = set_max_smem(tcb::attn_bwd_dq_kernel<DH>, C::SMEM_DQ, s)) != cudaSuccess) return e;
  tcb::attn_bwd_dq_kernel<DH><<<nq < sms ? nq : sms, tcb::NTHREADS, C::SMEM_DQ, s>>>(tq, tdo, tk, tv, a, status);
  return cudaGetLastError();
}

cudaError_t attention_backward_tc(const AttnBwdArgs& a, int* status, cudaStream_t s) {
  if (a.B <= 0 || a.S <= 0) return cudaSuccess;
  if ((a.dh != 64 && a.dh != 128) || a.Hq % a.Hkv || a.lse_ld < (a.S + tcb::BT - 1) / tcb::BT * tcb::BT ||
      ((uintptr_t)a.dq & 31) || ((uintptr_t)a.dkv & 31) || ((uintptr_t)a.lse & 15) || ((uintptr_t)a.dsum & 15) ||
      (long long)a.B * a.S >= (1LL << 31))
    return cudaErrorInvalidValue;
  CUtensorMap tq, tdo, tk, tv;
  const int rows = a.B * a.S;
  cudaError_t e = make_tmap_bf16(&tq, a.q, rows, a.Hq * a.dh, a.Hq * a.dh, tcb::BT);
  if (e == cudaSuccess) e = make_tmap_bf16(&tdo, a.dout, rows, a.Hq * a.dh, a.Hq * a.dh, tcb::BT);
  if (e == cudaSuccess) e = make_tmap_bf16(&tk, a.k, rows, a.Hkv * a.dh, a.Hkv * a.dh, tcb::BT);
  if (e == cudaSuccess) e = make_tmap_bf16(&tv, a.v, rows, a.Hkv * a.dh, a.Hkv * a.dh, tcb::BT);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return a.dh == 128 ? launch_bwd<128>(tq, tdo, tk, tv, a, status, sms, s)
                     : launch_bwd<64>(tq, tdo, tk, tv, a, status, sms, s);
}

}  // namespace mka
