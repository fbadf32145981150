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
//
// MODE 1 (block-gathered, for Block-MKA's block-sparse attention and full MKA's recalled-block
// path): an item is a pair of 128-row tiles of (token, head) rows that all read the keys of one
// L3 block (block_sparse.cu lists them).  The loader warp gathers the query rows four at a time
// with TMA (tile::gather4) into the same swizzled tile layout; each row keeps its own softmax
// over the block's key tiles (the causal mask only for the block's own tokens) and leaves O / l
// in bf16 with its log2 normaliser for the merge.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.cuh"

namespace mka {

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows);
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, int d0, int d1, int d2, long long s1, long long s2,
                              int box1);

namespace tca {

using namespace sm100;

constexpr int BQ = 128, BKV = 128;
constexpr int NTHREADS = 320;
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units
constexpr int kNoMask = 0x7fffffff;

template <int DH>
struct Cfg {
  static constexpr int Q_BYTES = BQ * DH * 2;    // one query tile
  static constexpr int K_BYTES = BKV * DH * 2;
  static constexpr int KV_BYTES = 2 * K_BYTES;   // K then V
  static constexpr int HALF = 128 * 64 * 2;      // one 128-row x 64-column swizzled box
  static constexpr int SMEM = 2 * Q_BYTES + 2 * KV_BYTES + 1024 + 256;
  static constexpr int GATHER_BYTES = 2 * BQ * 4;  // MODE 1: the loader's token lists of both tiles
};

struct Work {
  int b, h, pair;
};
// Items run in chunks of `chunk` streams, a stream being one (sequence, KV group): chunk by
// chunk, within a chunk the longest query-tile pairs first, and for one pair the chunk's streams
// with their G query heads next to each other (the heads that share a K/V tile run together).  The
// CTAs at work then share the K/V of a chunk's streams in L2 (one stream is 67 MB at 131072 keys)
// instead of streaming every group's K/V from DRAM each round of items.  Rounds of items must still
// span few pair lengths, which the static snake schedule needs for its balance; chunk = B * Hkv is
// plain longest-first over all heads.
__device__ __forceinline__ Work work_item(int w, int B, int Hq, int Hkv, int npairs, int chunk) {
  Work r;
  const int G = Hq / Hkv, NS = B * Hkv;
  const int k = w / (chunk * G * npairs);  // chunk (the last one may hold fewer streams)
  const int cs = min(chunk, NS - k * chunk);
  const int rem = w - k * chunk * G * npairs;
  r.pair = npairs - 1 - rem / (cs * G);  // longest rows first
  const int r2 = rem % (cs * G);
  const int st = k * chunk + r2 / G;
  r.b = st / Hkv;
  r.h = (st % Hkv) * G + r2 % G;
  return r;
}

// Work item of round r for this CTA: items are sorted longest first and dealt in a
// snake order (CTA order reversed every other round), which balances the causal
// work across CTAs far better than plain round-robin.  -1 past the end.
__device__ __forceinline__ int snake_item(int r, int grid, int cta, int nwork) {
  const int w = r * grid + ((r & 1) ? grid - 1 - cta : cta);
  return w < nwork ? w : -1;
}

// MODE 1 work item: tile pair P (of the row list of block j of sequence b) for KV group g.
// g_pinfo[P] = b * nblk + j, bit 30 set when the pair's second list tile exists; g_ptok[P] holds the
// pair's 2 tpt list entries ((t << 5) | slot, -1 past the end), written when the lists are built.
struct GWork {
  int b, g, j, P, t1;
};
__device__ __forceinline__ GWork gwork_item(int w, const AttnArgs& a) {
  GWork r;
  r.P = w / a.Hkv;
  r.g = w - r.P * a.Hkv;
  const int info = a.g_pinfo[r.P];
  const int bj = info & 0x3fffffff;
  r.t1 = (info >> 30) & 1;
  r.b = bj / a.nblk;
  r.j = bj - r.b * a.nblk;
  return r;
}
// List entry k of local tile t (t = 0: the pair's second list tile, t = 1: its first); -1 if none.
__device__ __forceinline__ int gwork_entry(const AttnArgs& a, int P, int t, int k, int tpt) {
  return a.g_ptok[(size_t)P * 2 * tpt + (1 - t) * tpt + k];
}
// Token (position in the sequence) of an entry, -1 for none; its partial slot in *slot.
__device__ __forceinline__ int entry_token(int v, int S, int* slot) {
  *slot = v >= 0 ? (v & 31) : 0;
  const int t = v >> 5;
  return v >= 0 && t < S ? t : -1;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}


// MODE 0: causal attention; MODE 1: block-gathered rows (see the top of the file).
template <int DH, int MODE>
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
  uint64_t* p_half = bars + 18;   // [2] keys 0-63 of P_t are in TMEM
  uint64_t* drain = bars + 20;
  uint32_t* tmem_slot = (uint32_t*)(bars + 21);
  int* stok = (int*)(smem + 2 * C::Q_BYTES + 2 * C::KV_BYTES + 256);  // MODE 1: loader's tokens, [2][BQ]
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  constexpr bool GA = MODE == 1;
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
      mbar_init(&p_half[i], 4);
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
  const int nbj = a.B * a.nblk;
  const int nwork = GA ? a.Hkv * a.g_pairoff[nbj] : a.B * a.Hq * npairs;
  const int G = a.Hq / a.Hkv;
  const int RPT = gathered_rows_per_token(G);  // MODE 1: tile rows per token (its G heads first)
  const int tpt = BQ / RPT;                    // MODE 1: tokens per query tile
  const long long q_rows_per_b = a.q_bstride / a.q_ld;
  const long long kv_rows_per_b = a.kv_bstride / a.kv_ld;
  const int mt = GA ? a.blk / BKV : 1;  // MODE 1: key tiles per L3 block
  // Key tiles of the two query tiles of an item (n0 <= n1).  Causal: tile qt runs tiles 0..qt.
  // MODE 1: local tile t holds list tile 2p + 1 - t, so tile 1 always exists and tile 0 may be
  // empty (0 key tiles); both read the same mt key tiles of block j.
  auto item_tiles = [&](int w, int& n0, int& n1) {
    if constexpr (GA) {
      n0 = (a.g_pinfo[w / a.Hkv] >> 30) & 1 ? mt : 0;
      n1 = mt;
    } else {
      const Work it = work_item(w, a.B, a.Hq, a.Hkv, npairs, a.chunk);
      n0 = 2 * it.pair + 1;
      n1 = 2 * it.pair + 2;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if constexpr (GA) {
      // The warp looks up the tile's tokens, then every lane gathers four query rows per 64-column
      // half with one TMA (tmQ views q as [B*S*Hq rows][dh]); lane 0 then issues the block's K/V.
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      // An item's block and the tokens of its two tiles are looked up while the previous item's
      // copies are in flight: lane k < tpt holds the token of slot k (8-row slots), and the
      // tokens of all tpt entries go to stok (gather4).
      GWork it;
      int tk[2] = {-1, -1};
      auto lookup = [&](int w) {
        it = gwork_item(w, a);
        for (int t = 0; t < 2; ++t) {
          int slot;
          tk[t] = lane < tpt ? entry_token(gwork_entry(a, it.P, t, lane, tpt), a.S, &slot) : -1;
          if (RPT != 8 && (t == 1 || it.t1))
            for (int k = lane; k < tpt; k += 32)
              stok[t * BQ + k] = k == lane ? tk[t] : entry_token(gwork_entry(a, it.P, t, k, tpt), a.S, &slot);
        }
      };
      int kvit = 0;
      int w = snake_item(0, gridDim.x, blockIdx.x, nwork);
      if (w >= 0) lookup(w);
      for (int rr = 0; rr * (int)gridDim.x < nwork; ++rr) {
        if (w < 0) break;
        const int wi = rr;
        // the block's K/V first: its stages free up earlier than the query tiles
        bool ok = true;
        if (lane == 0) {
          for (int jj = 0; jj < mt; ++jj, ++kvit) {
            const int st = kvit & 1;
            if (!mbar_wait(&kv_empty[st], ((kvit >> 1) & 1) ^ 1, abort, status)) {
              ok = false;
              break;
            }
            mbar_expect_tx(&kv_full[st], C::KV_BYTES);
            uint8_t* kdst = sKV + st * C::KV_BYTES;
            const int ky = (int)(it.b * kv_rows_per_b) + it.j * a.blk + jj * BKV;
            for (int hb = 0; hb < NH; ++hb) {
              tma_load_2d(kdst + hb * C::HALF, &tmK, &kv_full[st], it.g * DH + hb * 64, ky);
              tma_load_2d(kdst + C::K_BYTES + hb * C::HALF, &tmV, &kv_full[st], it.g * DH + hb * 64, ky);
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        bool qok = true;
        for (int t = 0; t < 2; ++t) {
          const bool full = t == 1 || it.t1;
          const int tok = tk[t];
          const bool ok_t = mbar_wait(&q_empty[t], (wi & 1) ^ 1, abort, status);
          if (!__all_sync(0xffffffffu, ok_t)) {
            qok = false;
            break;
          }
          if (full) {
            if (lane == 0) mbar_expect_tx(&q_full[t], C::Q_BYTES);
            __syncwarp();
            uint8_t* dst_t = sQ + t * C::Q_BYTES;
            if (RPT == 8) {
              // one box of the token's 8 heads from g * G (tmQ: [B*S][Hq][dh]) per 64-column half
              if (lane < tpt) {
                const int z = it.b * a.S + (tok >= 0 ? tok : 0);
#pragma unroll
                for (int hb = 0; hb < NH; ++hb)
                  tma_load_3d(dst_t + hb * C::HALF + lane * 1024, &tmQ, &q_full[t], hb * 64, it.g * G, z);
              }
            } else {
              // four rows per lane and half (tmQ: [B*S*Hq][dh], one-row boxes)
              const int row0 = it.b * a.S * a.Hq;  // a valid row for the padding rows
              int rows[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int r = 4 * lane + u, k = r / G;
                const int tr = k < tpt ? stok[t * BQ + k] : -1;
                rows[u] = tr >= 0 ? (it.b * a.S + tr) * a.Hq + it.g * G + (r - k * G) : row0;
              }
#pragma unroll
              for (int hb = 0; hb < NH; ++hb)
                tma_gather4_2d(dst_t + hb * C::HALF + 4 * lane * 128, &tmQ, &q_full[t], hb * 64, rows[0], rows[1],
                               rows[2], rows[3]);
            }
          } else if (lane == 0) {
            mbar_arrive(&q_full[t]);  // empty tile: nothing to load
          }
          __syncwarp();
        }
        if (!qok) break;
        w = snake_item(rr + 1, gridDim.x, blockIdx.x, nwork);
        if (w >= 0) lookup(w);
      }
    } else if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // L2: a query tile is read by this item only, while the K/V of the chunk's streams are read
      // by every item of the chunk: the Q tiles (and the O rows) must not age the K/V out of L2
      const uint64_t pol_once = policy_evict_first(), pol_kv = policy_evict_last();
      int kvit = 0;
      for (int rr = 0; rr * (int)gridDim.x < nwork; ++rr) {
        const int w = snake_item(rr, gridDim.x, blockIdx.x, nwork);
        if (w < 0) break;
        const int wi = rr;  // items this CTA has started before this one
        const Work it = work_item(w, a.B, a.Hq, a.Hkv, npairs, a.chunk);
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
            tma_load_2d_hint(sQ + t * C::Q_BYTES + hb * C::HALF, &tmQ, &q_full[t], it.h * DH + hb * 64, qy, pol_once);
        }
        if (!qok) break;
        const int nkv = 2 * it.pair + 2;
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
            tma_load_2d_hint(kdst + hb * C::HALF, &tmK, &kv_full[st], g * DH + hb * 64, ky, pol_kv);
            tma_load_2d_hint(kdst + C::K_BYTES + hb * C::HALF, &tmV, &kv_full[st], g * DH + hb * 64, ky, pol_kv);
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // (the whole warp runs the role, converged; one elected lane issues)
    int kvit = 0, pc[2] = {0, 0};
    bool ok = true;
    const uint64_t qd0 = sdesc_kmajor_sw128(sQ), qd1 = sdesc_kmajor_sw128(sQ + C::Q_BYTES);
    auto issue_s = [&](int t, int st) {
      const uint64_t kd = sdesc_kmajor_sw128(sKV + st * C::KV_BYTES);
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        const uint64_t off = (uint64_t)((kk >> 2) * (C::HALF >> 4) + (kk & 3) * 2);
        umma_bf16_ss_w(tbase + S_COL(t), (t ? qd1 : qd0) + off, kd + off, IDESC_S, kk != 0);
      }
      umma_commit_w(&s_full[t]);
    };
    // P V in two halves of four K-steps: keys 0-63 as soon as the softmax has packed them, keys
    // 64-127 after p_full
    auto issue_pv_half = [&](int t, int st, int j, int hh) {
      const uint64_t vd = sdesc_mnmajor_sw128(sKV + st * C::KV_BYTES + C::K_BYTES);
#pragma unroll
      for (int k4 = 0; k4 < BKV / 32; ++k4) {
        const int kk = hh * (BKV / 32) + k4;
        umma_bf16_ts_w(tbase + O_COL(t), tbase + S_COL(t) + kk * 8, vd + (uint64_t)(kk * (2048 >> 4)), IDESC_O,
                       (j | kk) != 0);
      }
      if (hh) umma_commit_w(&pv_done[t]);
    };
    int nx0 = 0, nx1 = 0;  // tiles of the next item, looked up while this one runs
    {
      const int w0 = snake_item(0, gridDim.x, blockIdx.x, nwork);
      if (w0 >= 0) item_tiles(w0, nx0, nx1);
    }
    for (int rr = 0; rr * (int)gridDim.x < nwork && ok; ++rr) {
      const int w = snake_item(rr, gridDim.x, blockIdx.x, nwork);
      if (w < 0) break;
      const int wi = rr;  // items this CTA has started before this one
      const int n0 = nx0, n1 = nx1;  // n0 <= n1, n1 >= 1
      if (!mbar_wait_warp(&q_full[0], wi & 1, abort, status)) break;
      if (n1 > 0 && !mbar_wait_warp(&kv_full[kvit & 1], (kvit >> 1) & 1, abort, status)) break;
      tc_fence_after();
      if (n0 > 0) issue_s(0, kvit & 1);
      if (n0 <= 1) umma_commit_w(&q_empty[0]);  // Q_0's last use (or none)
      // No key tile: the epilogue adds nothing from TMEM, but o_full still moves one phase per
      // item, and only after the previous item's epilogue released O_t: without that wait two
      // items in a row could commit two phases before the softmax warps wait for the first,
      // which then reads as the wrong parity and never completes.
      if (n0 == 0) {
        if (!mbar_wait_warp(&o_empty[0], (wi & 1) ^ 1, abort, status)) break;
        umma_commit_w(&o_full[0]);
      }
      if (!mbar_wait_warp(&q_full[1], wi & 1, abort, status)) break;
      tc_fence_after();
      if (n1 > 0) issue_s(1, kvit & 1);
      if (n1 <= 1) umma_commit_w(&q_empty[1]);
      if (n1 == 0) {
        if (!mbar_wait_warp(&o_empty[1], (wi & 1) ^ 1, abort, status)) break;
        umma_commit_w(&o_full[1]);
      }
      {  // the next item's tile counts, looked up while these S MMAs and the softmax run
        const int wn = snake_item(rr + 1, gridDim.x, blockIdx.x, nwork);
        if (wn >= 0) item_tiles(wn, nx0, nx1);
      }
      for (int j = 0; j < n1; ++j) {
        const int cur = kvit + j, st = cur & 1, nst = (cur + 1) & 1;
        bool next_ready = false;
        if (j < n0) {
          if (!mbar_wait_warp(&p_half[0], pc[0] & 1, abort, status)) { ok = false; break; }
          if (j == 0 && !mbar_wait_warp(&o_empty[0], (wi & 1) ^ 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          issue_pv_half(0, st, j, 0);
          if (!mbar_wait_warp(&p_full[0], pc[0] & 1, abort, status)) { ok = false; break; }
          tc_fence_after();
          issue_pv_half(0, st, j, 1);
          ++pc[0];
          if (j + 1 == n0) umma_commit_w(&o_full[0]);
          if (j + 1 < n0) {
            if (!mbar_wait_warp(&kv_full[nst], ((cur + 1) >> 1) & 1, abort, status)) { ok = false; break; }
            tc_fence_after();
            next_ready = true;
            issue_s(0, nst);
            if (j + 2 == n0) umma_commit_w(&q_empty[0]);  // Q_0's last use
          }
        }
        if (!mbar_wait_warp(&p_half[1], pc[1] & 1, abort, status)) { ok = false; break; }
        if (j == 0 && !mbar_wait_warp(&o_empty[1], (wi & 1) ^ 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        issue_pv_half(1, st, j, 0);
        if (!mbar_wait_warp(&p_full[1], pc[1] & 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        issue_pv_half(1, st, j, 1);
        ++pc[1];
        umma_commit_w(&kv_empty[st]);
        if (j + 1 < n1) {
          if (!next_ready) {
            if (!mbar_wait_warp(&kv_full[nst], ((cur + 1) >> 1) & 1, abort, status)) { ok = false; break; }
            tc_fence_after();
          }
          issue_s(1, nst);
          if (j + 2 == n1) umma_commit_w(&q_empty[1]);  // Q_1's last use
        } else {
          umma_commit_w(&o_full[1]);
        }
      }
      if (!ok) break;
      kvit += n1;
    }
    if (__any_sync(0xffffffffu, *abort)) {
      umma_commit_w(drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 100000000ull) {
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
    // causal output rows start on 32-byte boundaries: one 32-byte store per 16 columns
    const bool o32 = !GA && ((uintptr_t)a.o & 31) == 0 && a.o_ld % 16 == 0 && a.o_bstride % 16 == 0;
    const uint64_t pol_out = policy_evict_first();  // output rows: written once, not read here
    int sit = 0;
    for (int rr = 0; rr * (int)gridDim.x < nwork; ++rr) {
      const int w = snake_item(rr, gridDim.x, blockIdx.x, nwork);
      if (w < 0) break;
      const int wi = rr;
      // This row: causal, position `row` of query head h of sequence b; MODE 1, the token of
      // entry e of the item's list (-1 for a padding row), query head h of KV group g.
      int b, h, row, nkv, slot = 0, key0 = 0;
      int row_lim;  // keys after this position are masked (kNoMask: none)
      bool masked;  // warp-uniform: the causal mask applies to some row of the warp
      if constexpr (GA) {
        const GWork it = gwork_item(w, a);
        const int k = r / RPT, hh = r - k * RPT;
        b = it.b;
        h = it.g * G + hh;
        nkv = t == 1 || it.t1 ? mt : 0;
        row = k < tpt && hh < G ? entry_token(gwork_entry(a, it.P, t, k, tpt), a.S, &slot) : -1;
        key0 = it.j * a.blk;  // keys of the block's tiles start here
        row_lim = row >= 0 && row / a.blk == it.j ? row : kNoMask;  // the block's own tokens only
        masked = __any_sync(0xffffffffu, row_lim != kNoMask);
      } else {
        const Work it = work_item(w, a.B, a.Hq, a.Hkv, npairs, a.chunk);
        const int qt = 2 * it.pair + t;
        b = it.b;
        h = it.h;
        nkv = qt + 1;
        row = qt * BQ + r;
        row_lim = row;
        masked = false;
      }
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv; ++j, ++sit) {
        if (!mbar_wait_warp(&s_full[t], sit & 1, abort, status)) { ok = false; break; }
        tc_fence_after();
        const bool diag = GA ? masked : (j == nkv - 1);
        // keys c > lim of this tile are in the future of this row
        const int lim = row_lim == kNoMask ? kNoMask : row_lim - (key0 + j * BKV);
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
        // rescale the O rows (rare with the lazy threshold) before pass 2, since the first half of
        // P_j V_j starts while pass 2 runs.  S_j landing means P_{j-1} V_{j-1}, issued before QK_j,
        // has completed, so the wait below returns at once.
        if (__ballot_sync(0xffffffffu, rescale)) {
          if (!mbar_wait_warp(&pv_done[t], (sit - 1) & 1, abort, status)) { ok = false; break; }
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
        // pass 2: P = 2^(s*sl2 - m_ref) as bf16 pairs over the first 64 columns of S; the
        // TMEM load of chunk c+1 is in flight while chunk c is exponentiated.  Keys 0-63 (chunks 0
        // and 1) are signalled on p_half so that their half of P V can start.
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
            lsum2 = __fadd2_rn(lsum2, make_float2(p0, p1));
            __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
            pk[e] = *(uint32_t*)&hb;
          }
          tmem_st16(s_tmem + c * 16, pk);
          if (c == 1) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_half[t]);
          }
        }
        const float lsum = lsum2.x + lsum2.y;
        l += lsum;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // epilogue: O_t / l -> bf16 -> global
      if (!mbar_wait_warp(&o_full[t], wi & 1, abort, status)) break;
      tc_fence_after();
      const float inv = 1.f / l;
      // causal: row `row` of the output; MODE 1: slot `slot` of the token's partial results
      bf16* orow;
      bool store;
      if constexpr (GA) {
        store = row >= 0;
        const size_t ps = ((size_t)b * a.S + (store ? row : 0)) * a.nslot + slot;
        orow = (bf16*)a.part_o + ps * (size_t)(a.Hq * DH) + (size_t)h * DH;
        if (store) a.part_lse[ps * a.Hq + h] = m_ref + __log2f(l);
      } else {
        store = row < a.S;
        orow = (bf16*)a.o + (size_t)b * a.o_bstride + (size_t)row * a.o_ld + (size_t)h * DH;
        if (a.lse && store) a.lse[((size_t)b * a.Hq + h) * a.lse_ld + row] = m_ref + __log2f(l);
      }
#pragma unroll
      for (int c = 0; c < DH; c += 64) {  // two TMEM loads behind one wait
        uint32_t ov[2][32];
        tmem_ld32(o_tmem + c, ov[0]);
        tmem_ld32(o_tmem + c + 32, ov[1]);
        tmem_ld_wait();
        if (store) {
          // 16 columns (one full 32-byte sector) per store into the workspace's partials; 8 into o
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t wv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              __nv_bfloat162 hb = __floats2bfloat162_rn(__uint_as_float(ov[v >> 1][(v & 1) * 16 + 2 * e]) * inv,
                                                        __uint_as_float(ov[v >> 1][(v & 1) * 16 + 2 * e + 1]) * inv);
              wv[e] = *(uint32_t*)&hb;
            }
            if (GA) {
              st_global_v8(orow + c + v * 16, wv);
            } else if (o32) {
              st_global_v8_hint(orow + c + v * 16, wv, pol_out);
            } else {
              *(uint4*)(orow + c + v * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
              *(uint4*)(orow + c + v * 16 + 8) = make_uint4(wv[4], wv[5], wv[6], wv[7]);
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
    if (lane == 0) linger_after_abort(abort);  // copies issued before a role gave up land first
  }
#undef O_COL
#undef S_COL
}

}  // namespace tca

template <int DH, int MODE>
cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                        int* status, int grid, cudaStream_t s) {
  constexpr int sm = tca::Cfg<DH>::SMEM + (MODE ? tca::Cfg<DH>::GATHER_BYTES : 0);
  cudaError_t e = set_max_smem(tca::attn_tc_kernel<DH, MODE>, sm, s);
  if (e != cudaSuccess) return e;
  tca::attn_tc_kernel<DH, MODE><<<grid, tca::NTHREADS, sm, s>>>(tq, tk, tv, a, status);
  return cudaGetLastError();
}

cudaError_t attention_prefill_tc(const AttnArgs& a, int* status, cudaStream_t s) {
  if (a.B <= 0 || a.S <= 0) return cudaSuccess;
  if ((a.dh != 64 && a.dh != 128) || (a.q_ld % 8) || (a.kv_ld % 8) || (a.o_ld % 8) || (a.q_bstride % a.q_ld) ||
      (a.kv_bstride % a.kv_ld))
    return cudaErrorInvalidValue;
  const long long q_rows = (long long)a.B * (a.q_bstride / a.q_ld);
  const long long kv_rows = (long long)a.B * (a.kv_bstride / a.kv_ld);
  if (q_rows >= (1LL << 31) || kv_rows >= (1LL << 31)) return cudaErrorInvalidValue;
  const bool ga = a.g_pairoff != nullptr;
  // MODE 1 gathers query rows from q viewed as [B*S*Hq][dh], one-row boxes (q must be dense)
  if (ga && (a.q_ld != a.Hq * a.dh || a.q_bstride != (long long)a.S * a.q_ld ||
             (long long)a.B * a.S * a.Hq >= (1LL << 31)))
    return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  if (!ga) e = make_tmap_bf16(&tq, a.q, (int)q_rows, a.Hq * a.dh, a.q_ld, tca::BQ);
  else if (gathered_rows_per_token(a.Hq / a.Hkv) == 8)  // [B*S][Hq][dh], boxes of 8 heads
    e = make_tmap_bf16_3d(&tq, a.q, a.dh, a.Hq, a.B * a.S, a.dh, a.q_ld, 8);
  else  // [B*S*Hq][dh], one-row boxes for tile::gather4
    e = make_tmap_bf16(&tq, a.q, a.B * a.S * a.Hq, a.dh, a.dh, 1);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tk, a.k, (int)kv_rows, a.Hkv * a.dh, a.kv_ld, tca::BKV);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tv, a.v, (int)kv_rows, a.Hkv * a.dh, a.kv_ld, tca::BKV);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (ga && (((uintptr_t)a.part_o & 31) || !a.g_pinfo || !a.g_ptok || !a.part_o || !a.part_lse || a.nblk < 1 || a.nslot < 1 ||
             a.blk < tca::BKV || a.blk % tca::BKV || a.Hq % a.Hkv || a.Hq / a.Hkv > tca::BQ ||
             (long long)a.nblk * a.blk < a.S))
    return cudaErrorInvalidValue;
  // MODE 1: the item count is on the device (block_lists); idle CTAs leave at once
  const int nqt = (a.S + tca::BQ - 1) / tca::BQ;
  const int nwork = a.B * a.Hq * ((nqt + 1) / 2);
  const int grid = ga ? sms : (nwork < sms ? nwork : sms);
  // causal mode: streams per chunk of the work order.  When the K/V of all streams fits in half of
  // L2, one chunk of all streams; otherwise the fewest streams for which one round of `grid` items
  // spans at most an eighth of the pair lengths.  Measured (with Q and O evict-first, K/V
  // evict-last): at 1 x 131072 (8 streams of 67 MB) 1 stream per chunk reads 8.9 GB per launch
  // from DRAM, where a single chunk read 174 GB; at 2 x 32768 (134 MB of K/V) chunks of 2 streams
  // take 14.08 ms against 14.45 ms for a single chunk.
  AttnArgs c = a;
  if (!ga) {
    const int G = a.Hq / a.Hkv, NS = a.B * a.Hkv, npairs = (nqt + 1) / 2;
    int l2 = 0;
    cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    const double kv_bytes = 2.0 * NS * (double)a.S * a.dh * 2;  // K and V, bf16
    const int want = (8 * grid + G * npairs - 1) / (G * npairs);
    c.chunk = kv_bytes <= 0.5 * l2 ? NS : (want < 1 ? 1 : (want > NS ? NS : want));
  }
  if (a.dh == 128)
    return ga ? launch_attn<128, 1>(tq, tk, tv, c, status, grid, s) : launch_attn<128, 0>(tq, tk, tv, c, status, grid, s);
  return ga ? launch_attn<64, 1>(tq, tk, tv, c, status, grid, s) : launch_attn<64, 0>(tq, tk, tv, c, status, grid, s);
}

}  // namespace mka
