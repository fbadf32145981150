// Tensor-core (tcgen05) GEMM for the layer's dense projections:
// C[M, N] = A[M, K] * B[N, K]^T with bf16 operands and a float32 accumulator
// (MKA paper notes §2-§3: q = X W_q, X W_k, X W_v, the folded router layer
// X (W_q W_r1), and the L3 projection X P all share the A operand X, so they run
// as one GEMM over the packed weight matrix).
//
// Persistent kernel, one CTA per SM, 192 threads (the CTA-pair variant below is the one
// launched; this single-CTA form is the fallback where 2-CTA clusters cannot be placed):
//   warp 0      TMA producer: A and B tiles (128x64 and 256x64, 128-B swizzle)
//               into a 4-stage shared-memory ring
//   warp 1      MMA issuer: 4 x tcgen05.mma (128x256x16) per stage into one of
//               two TMEM accumulators (2 x 256 columns); tcgen05.commit frees the
//               stage and, after the last k-block, hands the accumulator over
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time (each thread owns one
//               output row), convert and store per output segment, then
//               release the accumulator.  The epilogue of tile i overlaps the
//               main loop of tile i+1.
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.cuh"

namespace mka {
namespace tcg {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int NTHREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

__device__ __forceinline__ void store1(const Epilogue& ep, int m, int n, float v) {
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    if (s >= ep.nseg) break;
    const OutSeg& g = ep.seg[s];
    if (n >= g.n_begin && n < g.n_end) {
      size_t off = (size_t)m * g.ld + (n - g.n_begin);
      if (g.is_bf16) ((bf16*)g.ptr)[off] = __float2bfloat16_rn(v);
      else ((float*)g.ptr)[off] = v;
      return;
    }
  }
}

// Columns n .. n+31 of row m.
__device__ __forceinline__ void store_chunk(const Epilogue& ep, int m, int n, uint32_t (&r)[32], int N) {
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    if (s >= ep.nseg) break;
    const OutSeg& g = ep.seg[s];
    if (n >= g.n_begin && n + 32 <= g.n_end && n + 32 <= N) {
      const size_t off = (size_t)m * g.ld + (n - g.n_begin);
      if (g.add) {  // a float32 addend row (e.g. another contribution to the same gradient)
        const float4* ad = (const float4*)(g.add + (size_t)m * g.ld_add + (n - g.n_begin));
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 x = ad[v];
          r[4 * v] = __float_as_uint(__uint_as_float(r[4 * v]) + x.x);
          r[4 * v + 1] = __float_as_uint(__uint_as_float(r[4 * v + 1]) + x.y);
          r[4 * v + 2] = __float_as_uint(__uint_as_float(r[4 * v + 2]) + x.z);
          r[4 * v + 3] = __float_as_uint(__uint_as_float(r[4 * v + 3]) + x.w);
        }
      }
      if (g.is_bf16) {
        bf16* p = (bf16*)g.ptr + off;
        if (((uintptr_t)p & 31) == 0) {  // one 32-byte store per 16 columns
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[v * 16 + 2 * e]), __uint_as_float(r[v * 16 + 2 * e + 1]));
              w[e] = *(uint32_t*)&h;
            }
            st_global_v8(p + v * 16, w);
          }
        } else if ((off & 7) == 0) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            uint32_t* w = (uint32_t*)&u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[v * 8 + 2 * e]), __uint_as_float(r[v * 8 + 2 * e + 1]));
              w[e] = *(uint32_t*)&h;
            }
            *(uint4*)(p + v * 8) = u;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) p[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
        }
      } else {
        float* p = (float*)g.ptr + off;
        if (((uintptr_t)p & 31) == 0) {  // one 32-byte store per 8 columns
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t w[8] = {r[8 * v], r[8 * v + 1], r[8 * v + 2], r[8 * v + 3],
                                   r[8 * v + 4], r[8 * v + 5], r[8 * v + 6], r[8 * v + 7]};
            st_global_v8(p + v * 8, w);
          }
        } else if ((off & 3) == 0) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *(float4*)(p + v * 4) = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) p[i] = __uint_as_float(r[i]);
        }
      }
      return;
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (n + i < N) store1(ep, m, n + i, __uint_as_float(r[i]));
}

// One thread's output row of a finished 128 x 256 accumulator tile (TMEM row `trow`):
// either the router's hidden units (hi in columns [0,128), lo in [128,256)) reduced
// through GELU . W_r2 to 3 partials, or the columns stored per output segment.
__device__ __forceinline__ void epilogue_tile(const Epilogue& ep, uint32_t trow, int m, int n0, int M, int N) {
  if (n0 >= ep.r_begin && n0 < ep.r_end) {
    // router tile: hidden units u0 .. u0+127, hi in columns [0,128), lo in [128,256)
    const int rt = (n0 - ep.r_begin) / BN;
    const int u0 = rt * 128;
    float z0 = 0.f, z1 = 0.f, z2 = 0.f;
    for (int c = 0; c < 128; c += 32) {
      uint32_t hi[32], lo[32];
      tmem_ld32(trow + c, hi);
      tmem_ld32(trow + 128 + c, lo);
      tmem_ld_wait();
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        const float h = __uint_as_float(hi[i]) + __uint_as_float(lo[i]);
        const float g = gelu_erf(h);
        const float* w = ep.w_r2 + (size_t)(u0 + c + i) * 3;
        z0 = fmaf(g, w[0], z0);
        z1 = fmaf(g, w[1], z1);
        z2 = fmaf(g, w[2], z2);
      }
    }
    if (m < M) *(float4*)(ep.zpart + ((size_t)rt * M + m) * 4) = make_float4(z0, z1, z2, 0.f);
  } else {
    for (int c = 0; c < BN; c += 32) {
      if (n0 + c >= N) break;
      uint32_t r[32];
      tmem_ld32(trow + c, r);
      tmem_ld_wait();
      if (m < M) store_chunk(ep, m, n0 + c, r, N);
    }
  }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N, int K,
                   Epilogue ep, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
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

  const int nM = (M + BM - 1) / BM, nN = (N + BN - 1) / BN, ntiles = nM * nN;
  const int kblocks = (K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int it = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int m0 = (tile / nN) * BM, n0 = (tile % nN) * BN;
        for (int k = 0; k < kblocks; ++k, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort, status)) goto producer_done;
          uint8_t* st = smem + s * STAGE_BYTES;
          mbar_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(st, &tmA, &full[s], k * BK, m0);
          tma_load_2d(st + A_BYTES, &tmB, &full[s], k * BK, n0);
        }
      }
    producer_done:
      // On an abort, let the copies already issued land before the CTA unwinds:
      // for each stage, wait (100 ms at most) for its most recent load.
      if (*abort) {
        for (int s = 0; s < STAGES; ++s) {
          if (it - 1 < s) continue;
          const int last = s + ((it - 1 - s) / STAGES) * STAGES;
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(&full[s], (last / STAGES) & 1) && globaltimer() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {  // the whole warp runs the MMA role; one elected lane issues
    int it = 0, tl = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
      const int acc = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      if (!mbar_wait_warp(&tempty[acc], aph ^ 1, abort, status)) break;
      tc_fence_after();
      const uint32_t d_tmem = tbase + acc * BN;
      bool ok = true;
      for (int k = 0; k < kblocks; ++k, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait_warp(&full[s], ph, abort, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = smem + s * STAGE_BYTES;
        const uint64_t a_desc = sdesc_kmajor_sw128(st);
        const uint64_t b_desc = sdesc_kmajor_sw128(st + A_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_bf16_ss_w(d_tmem, a_desc + (uint64_t)(kk * 2), b_desc + (uint64_t)(kk * 2), IDESC, (k | kk) != 0);
        umma_commit_w(&empty[s]);
      }
      if (!ok) break;
      umma_commit_w(&tfull[acc]);
    }
    if (__any_sync(0xffffffffu, *abort)) {  // let the MMAs already issued finish before the TMEM is released
      umma_commit_w(drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 100000000ull) {
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    int tl = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tl) {
      const int acc = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      if (!mbar_wait_warp(&tfull[acc], aph, abort, status)) break;
      tc_fence_after();
      const int m0 = (tile / nN) * BM, n0 = (tile % nN) * BN;
      const int m = m0 + q * 32 + lane;
      const uint32_t trow = tbase + ((uint32_t)(q * 32) << 16) + acc * BN;
      epilogue_tile(ep, trow, m, n0, M, N);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
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

// ---------------------------------------------------------------- CTA-pair variant
// Same GEMM on 256 x 256 output tiles computed by a pair of CTAs (a cluster of 2) with
// tcgen05.mma.cta_group::2: each CTA stages its own 128 rows of A and 128 of the tile's 256
// rows of B (32 KB per k-block instead of 48 KB), so the operand stream per SM is two thirds
// of the single-CTA kernel's and six stages fit.  Rank 0 sets the transaction count of both
// CTAs' loads on its full barrier and issues the MMAs; their commits release both CTAs'
// stages and accumulators (multicast); both CTAs' epilogue warps release rank 0's
// accumulator barrier.  Each CTA's TMEM holds its 128 output rows x 256 columns.
constexpr int PAIR_BM = 256, HALF_ROWS = 128, PAIR_STAGES = 6;
constexpr int PAIR_STAGE_BYTES = 2 * HALF_ROWS * BK * 2;  // A rows + B rows of this CTA
constexpr int PAIR_SMEM_BYTES = PAIR_STAGES * PAIR_STAGE_BYTES + 1024 + 256;
constexpr uint32_t PAIR_IDESC = idesc_bf16_f32(PAIR_BM, BN);

// AMN / BMN: the operand is stored MN-major ([K][M] or [K][N], row stride lda / ldb): its 128 rows
// of a stage come as two 64 x 64 boxes (64 MN elements by 64 K rows, 8 KB apart).
template <bool AMN, bool BMN>
__global__ void __launch_bounds__(NTHREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                    int K, Epilogue ep, int* status) {
  constexpr uint32_t IDESC2 = PAIR_IDESC | (AMN ? 1u << 15 : 0u) | (BMN ? 1u << 16 : 0u);
  constexpr int CHUNK = 64 * BK * 2;  // one 64 x 64 MN-major box
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = (uint64_t*)(smem + PAIR_STAGES * PAIR_STAGE_BYTES);  // rank 0's copy is used
  uint64_t* empty = full + PAIR_STAGES;
  uint64_t* tfull = empty + PAIR_STAGES;
  uint64_t* tempty = tfull + 2;  // rank 0's copy is used
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* abort = (volatile int*)(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(&full[s], 1);   // rank 0's expect_tx arrival; both CTAs' bytes
      mbar_init(&empty[s], 1);  // the pair's MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // 4 epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc2(tmem_slot, TMEM_COLS);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised and TMEM allocated before any use
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const int nM = (M + PAIR_BM - 1) / PAIR_BM, nN = (N + BN - 1) / BN, ntiles = nM * nN;
  const int kblocks = (K + BK - 1) / BK;
  const int pair = (int)cluster_id_x(), npairs = (int)cluster_count_x();

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int it = 0;
      for (int tile = pair; tile < ntiles; tile += npairs) {
        const int ma = (tile / nN) * PAIR_BM + (int)rank * HALF_ROWS;  // this CTA's A rows
        const int nb = (tile % nN) * BN + (int)rank * HALF_ROWS;       // this CTA's B rows
        for (int k = 0; k < kblocks; ++k, ++it) {
          const int s = it % PAIR_STAGES;
          const uint32_t ph = (it / PAIR_STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort, status)) goto producer_done;
          uint8_t* st = smem + s * PAIR_STAGE_BYTES;
          if (rank == 0) mbar_expect_tx(&full[s], 2 * PAIR_STAGE_BYTES);
          if constexpr (AMN) {
            tma_load_2d_pair(st, &tmA, &full[s], ma, k * BK);
            tma_load_2d_pair(st + CHUNK, &tmA, &full[s], ma + 64, k * BK);
          } else {
            tma_load_2d_pair(st, &tmA, &full[s], k * BK, ma);
          }
          if constexpr (BMN) {
            tma_load_2d_pair(st + HALF_ROWS * BK * 2, &tmB, &full[s], nb, k * BK);
            tma_load_2d_pair(st + HALF_ROWS * BK * 2 + CHUNK, &tmB, &full[s], nb + 64, k * BK);
          } else {
            tma_load_2d_pair(st + HALF_ROWS * BK * 2, &tmB, &full[s], k * BK, nb);
          }
        }
      }
    producer_done:
      // Wait (bounded) until the pair's MMAs have released every stage this CTA filled: rank 0
      // reads this CTA's shared memory until then.
      for (int s = 0; s < PAIR_STAGES; ++s) {
        if (it - 1 < s) continue;
        const int last = s + ((it - 1 - s) / PAIR_STAGES) * PAIR_STAGES;
        const unsigned long long t0 = globaltimer();
        while (!mbar_try_wait(&empty[s], (last / PAIR_STAGES) & 1) && globaltimer() - t0 < 200000000ull) {
        }
      }
    }
  } else if (warp == 1 && rank == 0) {  // the whole warp runs the MMA role; one elected lane issues
    int it = 0, tl = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++tl) {
      const int acc = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      if (!mbar_wait_warp(&tempty[acc], aph ^ 1, abort, status)) break;
      tc_fence_after();
      const uint32_t d_tmem = tbase + acc * BN;
      bool ok = true;
      for (int k = 0; k < kblocks; ++k, ++it) {
        const int s = it % PAIR_STAGES;
        const uint32_t ph = (it / PAIR_STAGES) & 1;
        if (!mbar_wait_warp(&full[s], ph, abort, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* st = smem + s * PAIR_STAGE_BYTES;
        const uint64_t a_desc = AMN ? sdesc_mnmajor_sw128(st, CHUNK) : sdesc_kmajor_sw128(st);
        const uint64_t b_desc = BMN ? sdesc_mnmajor_sw128(st + HALF_ROWS * BK * 2, CHUNK)
                                    : sdesc_kmajor_sw128(st + HALF_ROWS * BK * 2);
        // K-step kk: 32 bytes along a K-major row, or 16 K rows (2 KB) of an MN-major box
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma2_bf16_ss_w(d_tmem, a_desc + (uint64_t)(AMN ? kk * (2048 >> 4) : kk * 2),
                        b_desc + (uint64_t)(BMN ? kk * (2048 >> 4) : kk * 2), IDESC2, (k | kk) != 0);
        umma2_commit_mc_w(&empty[s], 0x3);
      }
      if (!ok) break;
      umma2_commit_mc_w(&tfull[acc], 0x3);
    }
    if (__any_sync(0xffffffffu, *abort)) {  // let the MMAs already issued finish before the TMEM is released
      umma2_commit_mc_w(drain, 0x1);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 100000000ull) {
      }
    }
  } else if (warp >= 2) {
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    int tl = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++tl) {
      const int acc = tl & 1;
      const uint32_t aph = (tl >> 1) & 1;
      if (!mbar_wait_warp(&tfull[acc], aph, abort, status)) break;
      tc_fence_after();
      const int n0 = (tile % nN) * BN;
      const int m = (tile / nN) * PAIR_BM + (int)rank * HALF_ROWS + q * 32 + lane;
      const uint32_t trow = tbase + ((uint32_t)(q * 32) << 16) + acc * BN;
      epilogue_tile(ep, trow, m, n0, M, N);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_rank0(&tempty[acc]);
    }
  }
  tc_fence_before();
  cluster_sync();  // neither CTA frees TMEM or leaves while the pair's MMAs may still run
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc2(tbase, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

}  // namespace tcg

// bf16 [rows, cols] row-major (row stride ld elements) as a 2-D TMA tensor with a
// box of box_rows x 64 columns and 128-byte swizzle; out-of-range reads give zeros.
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int rows, int cols, int ld, int box_rows) {
  auto fn = tcg::encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 3-D bf16 tensor [d2][d1][d0] (d0 contiguous, strides s1, s2 elements), box {64, box1, 1}, 128B swizzle.
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, int d0, int d1, int d2, long long s1, long long s2,
                              int box1) {
  auto fn = tcg::encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t gdim[3] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2};
  cuuint64_t gstride[2] = {(cuuint64_t)s1 * 2, (cuuint64_t)s2 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <bool AMN, bool BMN>
static cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K, const Epilogue& ep,
                               int* status, int sms, cudaStream_t s) {
  cudaError_t e = set_max_smem(tcg::gemm_tc2_kernel<AMN, BMN>, tcg::PAIR_SMEM_BYTES, s);
  if (e != cudaSuccess) return e;
  const int ntiles = ((M + tcg::PAIR_BM - 1) / tcg::PAIR_BM) * ((N + tcg::BN - 1) / tcg::BN);
  int pairs = sms / 2;
  if (ntiles < pairs) pairs = ntiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(tcg::NTHREADS);
  cfg.dynamicSmemBytes = tcg::PAIR_SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tcg::gemm_tc2_kernel<AMN, BMN>, ta, tb, M, N, K, ep, status);
}

cudaError_t gemm_bf16_tc(const void* A, int lda, int a_mn, const void* B, int ldb, int b_mn, int M, int N, int K,
                         const Epilogue& ep, int* status, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if ((lda % 8) || (ldb % 8) || ((uintptr_t)A & 15) || ((uintptr_t)B & 15) || (!a_mn && K % 8) ||
      (a_mn && M % 8) || (!b_mn && K % 8) || (b_mn && N % 8))
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  // K-major: [M][K] rows, boxes of 64 K by 128 (A) / 128 (B, per CTA of a pair) rows;
  // MN-major: [K][M] rows, boxes of 64 x 64
  cudaError_t e = a_mn ? make_tmap_bf16(&ta, A, K, M, lda, 64) : make_tmap_bf16(&ta, A, M, K, lda, tcg::BM);
  if (e != cudaSuccess) return e;
  e = b_mn ? make_tmap_bf16(&tb, B, K, N, ldb, 64) : make_tmap_bf16(&tb, B, N, K, ldb, tcg::HALF_ROWS);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // CTA pairs: 256 x 256 tiles, two SMs per tile, grid of whole pairs
  if (a_mn && b_mn) e = launch_pair<true, true>(ta, tb, M, N, K, ep, status, sms, s);
  else if (a_mn) e = launch_pair<true, false>(ta, tb, M, N, K, ep, status, sms, s);
  else if (b_mn) e = launch_pair<false, true>(ta, tb, M, N, K, ep, status, sms, s);
  else e = launch_pair<false, false>(ta, tb, M, N, K, ep, status, sms, s);
  if (e == cudaSuccess || a_mn || b_mn) return e;  // the single-CTA fallback takes K-major operands only
  cudaGetLastError();  // a device or partition that cannot place 2-CTA clusters: one CTA per tile
  e = make_tmap_bf16(&tb, B, N, K, ldb, tcg::BN);
  if (e != cudaSuccess) return e;
  e = set_max_smem(tcg::gemm_tc_kernel, tcg::SMEM_BYTES, s);
  if (e != cudaSuccess) return e;
  const int ntiles1 = ((M + tcg::BM - 1) / tcg::BM) * ((N + tcg::BN - 1) / tcg::BN);
  tcg::gemm_tc_kernel<<<ntiles1 < sms ? ntiles1 : sms, tcg::NTHREADS, tcg::SMEM_BYTES, s>>>(ta, tb, M, N, K, ep, status);
  return cudaGetLastError();
}

cudaError_t gemm_tn_bf16_tc(const void* A, int lda, const void* B, int ldb, int M, int N, int K, const Epilogue& ep,
                            int* status, cudaStream_t s) {
  return gemm_bf16_tc(A, lda, 0, B, ldb, 0, M, N, K, ep, status, s);
}

}  // namespace mka
