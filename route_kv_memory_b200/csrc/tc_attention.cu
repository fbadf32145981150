// Causal GQA attention on tcgen05 tensor cores (MKA paper notes §3: one causal
// attention over the fused K/V; §4: online max-shift, partial sums rescaled by
// exp(mu_old - mu_new) when the running maximum grows).
//
// Persistent CTAs walk work items (sequence b, query head h, pair p of 128-row
// query tiles 2p and 2p+1) longest first, dealt to the CTAs in snake order.  Per item the CTA streams the 128-key
// tiles j <= 2p+1 of KV group g(h) = h / (Hq / Hkv), shared by both query tiles:
//   warp 0      TMA: both Q tiles once, then K_j and V_j into a 2-stage ring
//   warp 1      MMA, ping-pong between the two query tiles t = 0, 1:
//               S_t = Q_t K_j^T into TMEM, O_t += P_t V_j with P_t read from
//               TMEM (A operand) and V_j from shared memory (MN-major B operand);
//               while one softmax warpgroup works on S_0 the tensor pipe runs
//               the other tile's P V and next S
//   warps 2-5   softmax warpgroup of tile 0, warps 6-9 of tile 1, one query row
//               per thread: running maximum over the row, P = 2^(s*scale*log2e - m)
//               packed to bf16 into TMEM over S_t; O_t is rescaled (TMEM load,
//               scale, store) only when a row's maximum grew by more than 2^8, so
//               the stale maximum bounds P by 256; at the end O_t / l goes to
//               global memory.
// TMEM columns: O_0 [0,128), O_1 [128,256), S_0/P_0 [256,384), S_1/P_1 [384,512).
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.cuh"

namespace mka {

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows);

namespace tca {

using namespace sm100;

constexpr int BQ = 128, BKV = 128;
constexpr int NTHREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

template <int DH>
struct Cfg {
  static constexpr int Q_BYTES = BQ * DH * 2;    // one query tile
  static constexpr int K_BYTES = BKV * DH * 2;
  static constexpr int KV_BYTES = 2 * K_BYTES;   // K then V
  static constexpr int HALF = 128 * 64 * 2;      // one 128-row x 64-column swizzled box
  static constexpr int SMEM = 2 * Q_BYTES + 2 * KV_BYTES + 1024 + 256;
  // recalled-block pass: each softmax row's recalled block indices, staged per item
  static constexpr int REC_BYTES = 2 * BQ * 16 * 4;
};
constexpr int MAX_RECALL_RC = 16;  // recall_r the recalled-block pass stages in shared memory

struct Work {
  int b, h, pair;
};
__device__ __forceinline__ Work work_item(int w, int B, int Hq, int npairs) {
  Work r;
  const int per = B * Hq;
  r.pair = npairs - 1 - w / per;  // longest rows first
  const int rem = w % per;
  r.h = rem % Hq;
  r.b = rem / Hq;
  return r;
}

// Work item of round r for this CTA: items are sorted longest first and dealt in a
// snake order (CTA order reversed every other round), which balances the causal
// work across CTAs far better than plain round-robin.  -1 past the end.
__device__ __forceinline__ int snake_item(int r, int grid, int cta, int nwork) {
  const int w = r * grid + ((r & 1) ? grid - 1 - cta : cta);
  return w < nwork ? w : -1;
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

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// RC selects the recalled-block pass of full MKA: tile t of a pair runs only the key tiles
// before its query block's L3 block (n_t = (qt / m) * m for L3 blocks of m key tiles, possibly
// 0), a row keeps a key tile only if that tile's block is among the row's recalled blocks, and
// the epilogue writes lam0 * (causal output already in a.o) + lam1 * v2 + lam2 * this pass.
template <int DH, bool RC>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnArgs a, int* status) {
  using C = Cfg<DH>;
  constexpr int NH = DH / 64;  // 64-column boxes per row
  constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV);
  constexpr uint32_t IDESC_O = idesc_bf16_f32_bmn(BQ, DH);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                      // tile t at t * Q_BYTES
  uint8_t* sKV = smem + 2 * C::Q_BYTES;    // stage st: K at st*KV_BYTES, V at + K_BYTES
  uint64_t* bars = (uint64_t*)(smem + 2 * C::Q_BYTES + 2 * C::KV_BYTES);
  uint64_t* q_full = bars + 0;    // [2] query tiles
  uint64_t* q_empty = bars + 2;   // [2]
  uint64_t* kv_full = bars + 4;   // [2] stages
  uint64_t* kv_empty = bars + 6;  // [2]
  uint64_t* s_full = bars + 8;    // [2] query tiles
  uint64_t* p_full = bars + 10;   // [2]
  uint64_t* pv_done = bars + 12;  // [2]
  uint64_t* o_full = bars + 14;   // [2]
  uint64_t* o_empty = bars + 16;  // [2]
  uint64_t* drain = bars + 18;
  uint32_t* tmem_slot = (uint32_t*)(bars + 19);
  int* srec = (int*)(smem + 2 * C::Q_BYTES + 2 * C::KV_BYTES + 256);  // RC only: [2][BQ][MAX_RECALL_RC]
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // TMEM column of O_t and of S_t / P_t
#define O_COL(t) (128u * (uint32_t)(t))
#define S_COL(t) (256u + 128u * (uint32_t)(t))

  const int nqt = (a.S + BQ - 1) / BQ;
  const int npairs = (nqt + 1) / 2;
  const int nwork = a.B * a.Hq * npairs;
  const int G = a.Hq / a.Hkv;
  const long long q_rows_per_b = a.q_bstride / a.q_ld;
  const long long kv_rows_per_b = a.kv_bstride / a.kv_ld;
  const int mt = RC ? a.blk / BKV : 1;  // key tiles per L3 block
  // key tiles query tile qt runs: causal up to its own tile, or the tiles of strictly past L3 blocks
  auto ntiles = [&](int qt) { return RC ? (qt / mt) * mt : qt + 1; };

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int kvit = 0;
      for (int rr = 0; rr * (int)gridDim.x < nwork; ++rr) {
        const int w = snake_item(rr, gridDim.x, blockIdx.x, nwork);
        if (w < 0) break;
        const int wi = rr;  // items this CTA has started before this one
        const Work it = work_item(w, a.B, a.Hq, npairs);
        const int g = it.h / G;
        bool qok = true;
        for (int t = 0; t < 2; ++t) {  // each tile as soon as the previous item's last S_t has read it
          if (!mbar_wait(&q_empty[t], (wi & 1) ^ 1, abort, status)) {
            qok = false;
            break;
          }
          mbar_expect_tx(&q_full[t], C::Q_BYTES);
          const int qy = (int)(it.b * q_rows_per_b) + (2 * it.pair + t) * BQ;
          for (int hb = 0; hb < NH; ++hb)
            tma_load_2d(sQ + t * C::Q_BYTES + hb * C::HALF, &tmQ, &q_full[t], it.h * DH + hb * 64, qy);
        }
        if (!qok) break;
        const int nkv = ntiles(2 * it.pair + 1);
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
      int kvit = 0, pc[2] = {0, 0};
      bool ok = true;
      const uint64_t qd0 = sdesc_kmajor_sw128(sQ), qd1 = sdesc_kmajor_sw128(sQ + C::Q_BYTES);
      auto issue_s = [&](int t, int st) {
        const uint64_t kd = sdesc_kmajor_sw128(sKV + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint64_t off = (uint64_t)((kk >> 2) * (C::HALF >> 4) + (kk & 3) * 2);
          umma_bf16_ss(tbase + S_COL(t), (t ? qd1 : qd0) + off, kd + off, IDESC_S, kk != 0);
        }
        umma_commit(&s_full[t]);
      };
      auto issue_pv = [&](int t, int st, int j) {
        const uint64_t vd = sdesc_mnmajor_sw128(sKV + st * C::KV_BYTES + C::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          umma_bf16_ts(tbase + O_COL(t), tbase + S_COL(t) + kk * 8, vd + (uint64_t)(kk * (2048 >> 4)), IDESC_O,
                       (j | kk) != 0);
        umma_commit(&pv_done[t]);
      };
      for (int rr = 0; rr * (int)gridDim.x < nwork && ok; ++rr) {
        const int w = snake_item(rr, gridDim.x, blockIdx.x, nwork);
        if (w < 0) break;
        const int wi = rr;  // items this CTA has started before this one
        const Work it = work_item(w, a.B, a.Hq, npairs);
        const int n0 = ntiles(2 * it.pair), n1 = ntiles(2 * it.pair + 1);  // n0 <= n1
        if (!mbar_wait(&q_full[0], wi & 1, abort, status)) break;
        if (n1 > 0 && !mbar_wait(&kv_full[kvit & 1], (kvit >> 1) & 1, abort, status)) break;
        tc_fence_after();
        if (n0 > 0) issue_s(0, kvit & 1);
        if (n0 <= 1) umma_commit(&q_empty[0]);  // Q_0's last use (or none)
        // No key tile: the epilogue adds nothing from TMEM, but o_full still moves one phase per
        // item, and only after the previous item's epilogue released O_t: without that wait two
        // items in a row could commit two phases before the softmax warps wait for the first,
        // which then reads as the wrong parity and never completes.
        if (n0 == 0) {
          if (!mbar_wait(&o_empty[0], (wi & 1) ^ 1, abort, status)) break;
          umma_commit(&o_full[0]);
        }
        if (!mbar_wait(&q_full[1], wi & 1, abort, status)) break;
        tc_fence_after();
        if (n1 > 0) issue_s(1, kvit & 1);
        if (n1 <= 1) umma_commit(&q_empty[1]);
        if (n1 == 0) {
          if (!mbar_wait(&o_empty[1], (wi & 1) ^ 1, abort, status)) break;
          umma_commit(&o_full[1]);
        }
        for (int j = 0; j < n1; ++j) {
          const int cur = kvit + j, st = cur & 1, nst = (cur + 1) & 1;
          bool next_ready = false;
          if (j < n0) {
            if (!mbar_wait(&p_full[0], pc[0] & 1, abort, status)) { ok = false; break; }
            if (j == 0 && !mbar_wait(&o_empty[0], (wi & 1) ^ 1, abort, status)) { ok = false; break; }
            tc_fence_after();
            issue_pv(0, st, j);
            ++pc[0];
            if (j + 1 == n0) umma_commit(&o_full[0]);
            if (j + 1 < n0) {
              if (!mbar_wait(&kv_full[nst], ((cur + 1) >> 1) & 1, abort, status)) { ok = false; break; }
              tc_fence_after();
              next_ready = true;
              issue_s(0, nst);
              if (j + 2 == n0) umma_commit(&q_empty[0]);  // Q_0's last use
            }
          }
          if (!mbar_wait(&p_full[1], pc[1] & 1, abort, status)) { ok = false; break; }
          if (j == 0 && !mbar_wait(&o_empty[1], (wi & 1) ^ 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          issue_pv(1, st, j);
          ++pc[1];
          umma_commit(&kv_empty[st]);
          if (j + 1 < n1) {
            if (!next_ready) {
              if (!mbar_wait(&kv_full[nst], ((cur + 1) >> 1) & 1, abort, status)) { ok = false; break; }
              tc_fence_after();
            }
            issue_s(1, nst);
            if (j + 2 == n1) umma_commit(&q_empty[1]);  // Q_1's last use
          } else {
            umma_commit(&o_full[1]);
          }
        }
        if (!ok) break;
        kvit += n1;
      }
      if (*abort) {
        umma_commit(drain);
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 100000000ull) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue, tile t
    const int t = (warp - 2) >> 2;           // 0 for warps 2-5, 1 for warps 6-9
    const int q4 = warp & 3;                 // TMEM lane quadrant
    const int r = q4 * 32 + lane;            // row within the query tile
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t s_tmem = tbase + lane_off + S_COL(t);
    const uint32_t o_tmem = tbase + lane_off + O_COL(t);
    const float sl2 = a.scale * 1.4426950408889634f;
    int sit = 0;
    for (int rr = 0; rr * (int)gridDim.x < nwork; ++rr) {
      const int w = snake_item(rr, gridDim.x, blockIdx.x, nwork);
      if (w < 0) break;
      const int wi = rr;
      const Work it = work_item(w, a.B, a.Hq, npairs);
      const int qt = 2 * it.pair + t;
      const int nkv = ntiles(qt);
      const int row = qt * BQ + r;
      // recalled-block pass: this row's recalled L3 blocks
      int my_cnt = 0;
      if (RC) {  // stage this row's recalled blocks in shared memory (keeps them out of registers)
        const size_t tok = (size_t)it.b * a.S + row;
        my_cnt = row < a.S ? a.rcnt[tok] : 0;
        for (int q = 0; q < my_cnt; ++q) srec[(t * BQ + r) * MAX_RECALL_RC + q] = a.ridx[tok * a.R + q];
        if (row < a.S) {  // the epilogue's inputs (causal output, L2 value) into L2 while the tiles run
          const char* o1 = (const char*)((const bf16*)a.o + (size_t)it.b * a.o_bstride + (size_t)row * a.o_ld +
                                         (size_t)it.h * DH);
          const char* v2 = (const char*)(a.v2 + tok * (size_t)(a.Hkv * DH) + (size_t)(it.h / G) * DH);
#pragma unroll
          for (int k = 0; k < DH * 2; k += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(o1 + k));
#pragma unroll
          for (int k = 0; k < DH * 4; k += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(v2 + k));
        }
      }
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv; ++j, ++sit) {
        if (!mbar_wait(&s_full[t], sit & 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        const bool diag = !RC && (j == nkv - 1);
        bool keep = true;  // RC: this key tile belongs to one of the row's recalled blocks
        if (RC) {
          keep = false;
          const int* rec = srec + (t * BQ + r) * MAX_RECALL_RC;
          for (int q = 0; q < my_cnt; ++q) keep |= (rec[q] == j / mt);
        }
        const int lim = row - j * BKV;  // keys c > lim are in the future of this row
        // pass 1: row maximum of the raw scores (four TMEM loads behind one wait; 3-input
        // max); only the diagonal tile needs the causal mask (a warp-uniform branch)
        float mx = -INFINITY;
        {
          uint32_t v[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(s_tmem + c * 32, v[c]);
          tmem_ld_wait();
          if (diag) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e <= lim) mx = fmaxf(mx, __uint_as_float(v[c][e]));
          } else {
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                m4[0] = max3(m4[0], __uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1]));
                m4[1] = max3(m4[1], __uint_as_float(v[c][e + 2]), __uint_as_float(v[c][e + 3]));
                m4[2] = max3(m4[2], __uint_as_float(v[c][e + 4]), __uint_as_float(v[c][e + 5]));
                m4[3] = max3(m4[3], __uint_as_float(v[c][e + 6]), __uint_as_float(v[c][e + 7]));
              }
            mx = fmaxf(max3(m4[0], m4[1], m4[2]), m4[3]);
          }
        }
        mx *= sl2;
        if (RC && !keep) mx = -INFINITY;
        // lazy rescale: move the reference maximum only when it is exceeded by more than 2^8
        const bool need = mx > m_ref + RESCALE_THRESHOLD;
        float corr = 1.f;
        bool rescale = false;  // O and l hold earlier tiles only once a key has been kept
        if (need) {
          rescale = m_ref != -INFINITY;
          corr = rescale ? ex2(m_ref - mx) : 0.f;
          m_ref = mx;
          l *= corr;
        }
        // pass 2: P = 2^(s*sl2 - m_ref) as bf16 pairs over the first 64 columns of S; the
        // TMEM load of chunk c+1 is in flight while chunk c is exponentiated
        const float nm = -m_ref;
        const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(nm, nm);
        float2 lsum2 = make_float2(0.f, 0.f);
        uint32_t vb[2][32];
        tmem_ld32(s_tmem, vb[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld_wait();
          if (c + 1 < 4) tmem_ld32(s_tmem + (c + 1) * 32, vb[(c + 1) & 1]);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            // packed FP32x2: one FFMA2 scales and shifts both scores, one FADD2 accumulates
            const float2 x2 = __ffma2_rn(make_float2(__uint_as_float(vb[c & 1][2 * e]), __uint_as_float(vb[c & 1][2 * e + 1])),
                                         sl2v, nmv);
            float p0 = ex2(x2.x), p1 = ex2(x2.y);
            if (diag) {
              if (c * 32 + 2 * e > lim) p0 = 0.f;
              if (c * 32 + 2 * e + 1 > lim) p1 = 0.f;
            }
            if (RC && !keep) {
              p0 = 0.f;
              p1 = 0.f;
            }
            lsum2 = __fadd2_rn(lsum2, make_float2(p0, p1));
            __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
            pk[e] = *(uint32_t*)&hb;
          }
          tmem_st16(s_tmem + c * 16, pk);
        }
        const float lsum = lsum2.x + lsum2.y;
        l += lsum;
        // rescale the O rows (rare with the lazy threshold).  S_j landing means PV_{j-1},
        // issued before QK_j, has completed, so the wait below returns at once.  PV_j is
        // issued only after p_full, so it accumulates onto the rescaled rows.
        if (__ballot_sync(0xffffffffu, rescale)) {
          if (!mbar_wait(&pv_done[t], (sit - 1) & 1, abort, status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < DH; c += 32) {
            uint32_t ov[32];
            tmem_ld32(o_tmem + c, ov);
            tmem_ld_wait();
            const float2 c2 = make_float2(corr, corr);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])), c2);
              ov[e] = __float_as_uint(o2.x);
              ov[e + 1] = __float_as_uint(o2.y);
            }
            tmem_st16(o_tmem + c, *reinterpret_cast<const uint32_t(*)[16]>(&ov[0]));
            tmem_st16(o_tmem + c + 16, *reinterpret_cast<const uint32_t(*)[16]>(&ov[16]));
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // epilogue: O_t / l -> bf16 -> global
      if (!mbar_wait(&o_full[t], wi & 1, abort, status)) break;
      tc_fence_after();
      // RC: a row with no kept key (l == 0) adds nothing, and TMEM may then hold a stale tile
      const bool has_o = !RC || l > 0.f;
      const float inv = has_o ? 1.f / l : 0.f;
      bf16* orow = (bf16*)a.o + (size_t)it.b * a.o_bstride + (size_t)row * a.o_ld + (size_t)it.h * DH;
      float lam0 = 1.f, lam1 = 0.f, lam2 = 0.f;
      const float* v2row = nullptr;
      if (RC && row < a.S) {
        const size_t tok = (size_t)it.b * a.S + row;
        lam0 = a.lam[tok * 3];
        lam1 = a.lam[tok * 3 + 1];
        lam2 = a.lam[tok * 3 + 2];
        v2row = a.v2 + tok * (size_t)(a.Hkv * DH) + (size_t)(it.h / G) * DH;
      }
#pragma unroll
      for (int c = 0; c < DH; c += 32) {
        uint32_t ov[32];
        tmem_ld32(o_tmem + c, ov);
        tmem_ld_wait();
        if (row < a.S) {
          if (RC) {
            // lam0 * causal output + lam1 * L2 value + lam2 * recalled-block output, 16 columns at a
            // time with that half's loads issued together (the stores would otherwise order them)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int c0 = c + hh * 16;
              uint4 o1[2];
              float4 v2c[4];
#pragma unroll
              for (int v = 0; v < 2; ++v) o1[v] = *(const uint4*)(orow + c0 + v * 8);
#pragma unroll
              for (int v = 0; v < 4; ++v) v2c[v] = *(const float4*)(v2row + c0 + v * 4);
#pragma unroll
              for (int v = 0; v < 2; ++v) {
                uint4 u;
                uint32_t* wv = (uint32_t*)&u;
                const uint32_t* o1w = (const uint32_t*)&o1[v];
                const float v2e[8] = {v2c[2 * v].x, v2c[2 * v].y, v2c[2 * v].z, v2c[2 * v].w,
                                      v2c[2 * v + 1].x, v2c[2 * v + 1].y, v2c[2 * v + 1].z, v2c[2 * v + 1].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int k = hh * 16 + v * 8 + 2 * e;
                  const float2 f1 = __bfloat1622float2(*(const __nv_bfloat162*)&o1w[e]);
                  const float x0 = has_o ? __uint_as_float(ov[k]) * inv : 0.f;
                  const float x1 = has_o ? __uint_as_float(ov[k + 1]) * inv : 0.f;
                  __nv_bfloat162 hb = __floats2bfloat162_rn(fmaf(lam0, f1.x, fmaf(lam1, v2e[2 * e], lam2 * x0)),
                                                            fmaf(lam0, f1.y, fmaf(lam1, v2e[2 * e + 1], lam2 * x1)));
                  wv[e] = *(uint32_t*)&hb;
                }
                *(uint4*)(orow + c0 + v * 8) = u;
              }
            }
          } else {
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[t]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
#undef O_COL
#undef S_COL
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
  const int nqt = (a.S + tca::BQ - 1) / tca::BQ;
  const int nwork = a.B * a.Hq * ((nqt + 1) / 2);
  const int grid = nwork < sms ? nwork : sms;
  if (a.ridx && (!a.rcnt || !a.lam || !a.v2 || a.R < 1 || a.R > tca::MAX_RECALL_RC || a.blk < tca::BKV ||
                 a.blk % tca::BKV))
    return cudaErrorInvalidValue;
  if (a.dh == 128) {
    if (a.ridx) {
      constexpr int sm = tca::Cfg<128>::SMEM + tca::Cfg<128>::REC_BYTES;
      e = set_max_smem(tca::attn_tc_kernel<128, true>, sm, s);
      if (e != cudaSuccess) return e;
      tca::attn_tc_kernel<128, true><<<grid, tca::NTHREADS, sm, s>>>(tq, tk, tv, a, status);
    } else {
      e = set_max_smem(tca::attn_tc_kernel<128, false>, tca::Cfg<128>::SMEM, s);
      if (e != cudaSuccess) return e;
      tca::attn_tc_kernel<128, false><<<grid, tca::NTHREADS, tca::Cfg<128>::SMEM, s>>>(tq, tk, tv, a, status);
    }
  } else {
    if (a.ridx) {
      constexpr int sm = tca::Cfg<64>::SMEM + tca::Cfg<64>::REC_BYTES;
      e = set_max_smem(tca::attn_tc_kernel<64, true>, sm, s);
      if (e != cudaSuccess) return e;
      tca::attn_tc_kernel<64, true><<<grid, tca::NTHREADS, sm, s>>>(tq, tk, tv, a, status);
    } else {
      e = set_max_smem(tca::attn_tc_kernel<64, false>, tca::Cfg<64>::SMEM, s);
      if (e != cudaSuccess) return e;
      tca::attn_tc_kernel<64, false><<<grid, tca::NTHREADS, tca::Cfg<64>::SMEM, s>>>(tq, tk, tv, a, status);
    }
  }
  return cudaGetLastError();
}

}  // namespace mka
