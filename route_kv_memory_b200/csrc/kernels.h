// Internal launch interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mka {

// Records `msg` as the calling thread's mka_last_error() text; returns `code`.
int set_last_error(int code, const char* msg);

// One column range of a GEMM output and where it is stored.
struct OutSeg {
  int n_begin, n_end;  // [n_begin, n_end) of the GEMM's N
  void* ptr;           // element (m, n) goes to ptr[m * ld + (n - n_begin)]
  int ld;
  int is_bf16;         // 1: bf16 store, 0: float32 store
  const float* add = nullptr;  // when set, add[m * ld_add + (n - n_begin)] is added before the store
  int ld_add = 0;              //   (ld_add % 4 == 0, 16-byte aligned)
};
constexpr int kMaxSegs = 6;
struct Epilogue {
  int nseg;
  OutSeg seg[kMaxSegs];
  // Router columns [r_begin, r_end) of the bf16 projection GEMM (0, 0: none): tiles of 256
  // columns holding the hi then lo halves of 128 hidden units of X (W_q W_r1).  The
  // epilogue writes zpart[(r * M + m) * 4 + k] = sum_u GELU(hi_u + lo_u) W_r2[u][k] for
  // the r-th such tile, instead of storing the hidden layer.
  int r_begin, r_end;
  const float* w_r2;
  float* zpart;
};

// C[M, N] = A[M, K] * B[N, K]^T (both operands K-major), float32 accumulation.
// bf16 operands on tensor cores; `f32` variants use CUDA-core FFMA (no TF32).
// The bf16 path is the persistent tcgen05 kernel of tc_gemm.cu (K, lda, ldb multiples of 8;
// A and B 16-byte aligned); a bounded wait that runs out records MKA_ERR_DEVICE_TIMEOUT in *status.
cudaError_t gemm_tn_bf16_tc(const void* A, int lda, const void* B, int ldb, int M, int N, int K, const Epilogue& ep,
                            int* status, cudaStream_t s);
// The same product with either operand stored MN-major instead (a_mn: A given as [K][M] with row
// stride lda, i.e. C = A^T-of-storage * ...; b_mn: B given as [K][N] with row stride ldb); the
// MN dimension of an MN-major operand a multiple of 8.
cudaError_t gemm_bf16_tc(const void* A, int lda, int a_mn, const void* B, int ldb, int b_mn, int M, int N, int K,
                         const Epilogue& ep, int* status, cudaStream_t s);
cudaError_t gemm_tn_ffma(const void* A, int lda, int a_bf16, const void* B, int ldb, int b_bf16, int M, int N, int K,
                         const Epilogue& ep, cudaStream_t s);

// out[c, r] = in[r, c] for in [rows, cols] (row stride ld_in), out row stride ld_out.
// elem: 2 (bf16), 4 (f32).  to_f64 widens to float64 output instead.
cudaError_t transpose(const void* in, int rows, int cols, int ld_in, void* out, int ld_out, int elem, int to_f64,
                      cudaStream_t s);
// Split float32 w into bf16 hi = rn(w) and lo = rn(w - hi).
cudaError_t split_hi_lo(const float* w, int n, void* hi, void* lo, cudaStream_t s);
// Copy/widen [n] elements of type (bf16|f32) to float32.
cudaError_t widen_f32(const void* in, int n, int in_bf16, float* out, cudaStream_t s);

// ---------------------------------------------------------------- memory / routing kernels
struct HashArgs {
  const float* proj;     // [T, ldp] float32 token projections (column k = bit k)
  int ldp;
  const void* x;         // [T, d] token rows (dtype) for exact refinement
  int x_bf16;
  const double* pT64;    // [nb, d] float64 P^T
  int d, nb, K;          // K: length of the dot products that produced proj
};

// lambda = route_gate(GELU(h1 + h2) . w_r2) per token (mode, tiers: see route_gate in common.cuh).
cudaError_t router_tail(const float* h1, const float* h2, int ldh, int T, int rh, const float* w_r2, int mode,
                        int tiers, float* lam, cudaStream_t s);
// lambda = route_gate(sum_r zpart[r][t][0..2]) for the router partials of the fused GEMM epilogue.
cudaError_t router_softmax(const float* zpart, int nparts, int T, int mode, int tiers, float* lam, cudaStream_t s);
// Writes the bf16 hi/lo split of w [rh, d] float32 into the rows of the packed matrix so that every
// 256-row group holds the hi then the lo rows of 128 consecutive hidden units (rh % 128 == 0).
cudaError_t split_hi_lo_interleaved(const float* w, int rh, int d, void* dst, cudaStream_t s);
cudaError_t token_codes(const HashArgs& a, int T, uint32_t* codes, cudaStream_t s);
// Codes of the full blocks from exact float64 block sums of x in d_model space projected in float64.
// P64: [d][32] float64 (P row-major, padded to 32 columns).  part: summary_codes_scratch() bytes.
// codes[b*code_bstride + j].
size_t summary_codes_scratch(int d, int B, int nblk);
cudaError_t summary_codes(const void* x, int x_bf16, int d, int B, int S, int nblk, int blk, const double* P64,
                          int nb, double* part, uint32_t* codes, int code_bstride, cudaStream_t s);
// out[r][0..31] = in[r][0..cols) widened to float64, zero padded (in: [rows, cols] bf16 or float32).
cudaError_t widen_pad32_f64(const void* in, int rows, int cols, int in_bf16, double* out, cudaStream_t s);
// Per full block j of each sequence: bsum = sum of its rows, bend = EMA end state from a zero carry,
// gend = the zero-carry EMA end state of each of its 8 row groups (all three nullable).
// x: [B*S, ld] (bf16 or float32), first `width` columns.  bsum[b*bsum_bstride + j*width + c],
// bend[(b*nblk + j)*width + c], gend[((b*nblk + j)*8 + g)*width + c].
cudaError_t block_reduce(const void* x, int x_bf16, int ld, int width, int B, int S, int nblk, int blk, float alpha,
                         float* bsum, long long bsum_bstride, float* bend, float* gend, cudaStream_t s);
cudaError_t ema_carry(const float* bend, int width, int B, int nblk, float alpha_pow_b, const float* carry_in,
                      float* carry, cudaStream_t s);
cudaError_t recall_select(const uint32_t* tok_codes, const uint32_t* blk_codes, int blk_codes_bstride, int B, int S,
                          int nblk, int blk, int R, int* idx, int* count, cudaStream_t s);

struct FuseArgs {
  const float* xkv; int ld;       // [B*S, ld] float32 projected rows (K part then V part)
  int width;                      // 2*dkv
  const float* lam;               // [B*S, 3]
  const int* idx; const int* count; int R;
  const float* bsum; long long bsum_bstride;  // [B][nblk][width] block SUMS
  const float* carry;             // [B][nblk+1][width] EMA value at each block start
  const float* gend;              // [B][nblk][8][width] zero-carry EMA end state of each row group
  int B, S, nblk, blk, dkv;
  float alpha;
  void* k_out; void* v_out; long long kv_bstride; int out_bf16;  // [B][.. rows][dkv]
  float* state_ema;               // [B][width] <- M2[S] (nullable)
  // Full MKA (three paths) instead of the fused K/V: k_out, v_out <- the tokens' own XW_k, XW_v
  // and v2_out [B*S][dkv] float32 <- the L2 path's value M2 W_v (its EMA of XW_v); no recall gather.
  float* v2_out = nullptr;
};
cudaError_t fuse_kv(const FuseArgs& a, cudaStream_t s);

// Standalone d-space pieces.
cudaError_t ema_apply(const void* x, int x_bf16, int width, int B, int S, int nblk, int blk, float alpha,
                      const float* carry, float* m2, float* carry_out, cudaStream_t s);
cudaError_t gather_mean(const int* idx, const int* count, int R, const float* bsum, int nblk, int width, int blk,
                        int B, int S, float* m3, cudaStream_t s);

// State tail after a prefill: the unfinished block's sums.
cudaError_t prefill_tail_state(const float* xkv, int ld, int width, const void* x, int x_bf16, int d, int B, int S,
                               int blk, float* blk_sum, double* blk_x, int* pos, cudaStream_t s);

// ---------------------------------------------------------------- attention
// 64-bit words of the decode step's synchronisation area in the state: the grid barrier's arrival
// count, then per (sequence, KV group) the split-attention units finished, then per sequence the
// token-update CTAs finished.  All of them only grow; a prefill with a state, or state_init, zeroes
// them.
inline size_t decode_sync_words(int B, int Hkv) { return 1 + (size_t)B * (Hkv + 1); }

struct AttnArgs {
  const void* q; long long q_bstride; int q_ld;      // q[b][t][h*dh + i]: b*q_bstride + t*q_ld + h*dh + i
  const void* k; const void* v; long long kv_bstride; int kv_ld;  // k[b][j][g*dh + i]
  void* o; long long o_bstride; int o_ld;
  int B, S, Hq, Hkv, dh;
  float scale;
  // causal mode, when set: each row's softmax normaliser in log2 units, m + log2(l) with the
  // scores taken as scale * log2(e) * q.k, at lse[(b * Hq + h) * lse_ld + t] (for the backward)
  float* lse = nullptr; int lse_ld = 0;
  int chunk = 1;  // causal mode: (sequence, KV group) streams per chunk of the work order (set by attention_prefill_tc)
  // Block-gathered attention (set g_pairoff to select it; bf16, tcgen05 only).  The rows of a
  // work item are (token, query head) pairs that all attend to the keys of one L3 block j of
  // sequence b: the tokens of block j's list (its own tokens first when g_own, under the causal
  // mask, then the tokens that recalled it), each with the G = Hq / Hkv query heads of one KV
  // group.  No o is written: each row leaves its partial softmax result, O / l in bf16 and the
  // log2 normaliser m + log2(l), in slot `slot` of its token, for merge_partials to combine.
  const int* g_pairoff = nullptr;  // [B*nblk + 1] first tile pair of each block; [B*nblk] = all pairs
  const int* g_pinfo = nullptr;    // [all pairs] b * nblk + j of the pair's block, bit 30: second tile exists
  const int* g_ptok = nullptr;     // [all pairs][2 tpt] the pair's list entries (t << 5) | slot, -1 past the end
  int g_own = 0, nblk = 0, blk = 0, nslot = 0;
  void* part_o = nullptr;          // [B*S][nslot][Hq*dh] bf16
  float* part_lse = nullptr;       // [B*S][nslot][Hq]
};
cudaError_t attention_prefill(const AttnArgs& a, int bf16, cudaStream_t s);
// bf16 path on tcgen05 (tc_attention.cu): persistent, TMA-fed, S and P in TMEM; causal, or
// block-gathered when a.g_pairoff is set.
cudaError_t attention_prefill_tc(const AttnArgs& a, int* status, cudaStream_t s);

// ---------------------------------------------------------------- block-gathered attention (block_sparse.cu)
// Query-tile rows one token takes in the block-gathered attention: its G = Hq / Hkv heads, or an
// aligned 8-row slot for 4 < G <= 8 (one 3-D TMA box per token and 64-column half).
__host__ __device__ inline int gathered_rows_per_token(int G) { return G > 4 && G <= 8 ? 8 : G; }
// Tile pairs the block-gathered attention can run at most (block_lists' pairbj capacity).
inline size_t gathered_max_pairs(long long T, int R, int own, int tpt, long long nbj) {
  return (size_t)((T * (R + own)) / (2 * tpt) + nbj + 1);
}
// Lists, per L3 block (b, j), the tokens whose recall picked it, and the tile pairs the gathered
// attention runs for it (own tokens of the block first when own).  Entry slot = r + slot_base for
// recall rank r.  Scratch from the caller: nrec, recoff, cursor [B*nblk], pairoff [B*nblk + 1],
// list [B*S*R], pairbj [gathered_max_pairs()].  tpt: tokens per 128-row query tile
// (128 / gathered_rows_per_token(Hq / Hkv)).
// ptok, pinfo (nullable, [max pairs][2 tpt] and [max pairs]): per tile pair its list entries, own
// tokens as (t << 5) | 0, -1 past the end, and its block with bit 30 set when its second tile exists.
cudaError_t block_lists(const int* idx, const int* cnt, int B, int S, int R, int blk, int nblk, int own,
                        int slot_base, int tpt, int* nrec, int* recoff, int* cursor, int* pairoff, int* pairbj,
                        int* list, int* ptok, int* pinfo, cudaStream_t s);
struct MergeArgs {
  const void* part_o; const float* part_lse; int nslot;
  const int* cnt; int own;          // partial slots of token t: [0, cnt[t] + own)
  int B, S, Hq, Hkv, dh;
  void* o; long long o_bstride; int o_ld;   // bf16 output rows
  // full MKA (lam set): o = lam0 * o (read back) + lam1 * v2 + lam2 * merged; else o = merged
  const float* lam = nullptr; const float* v2 = nullptr;  // [B*S][3], [B*S][Hkv*dh]
};
// Combines each row's partial softmax results: w_s = 2^(lse_s - max lse), o = sum w_s O_s / sum w_s
// (0 when the row has no slot).
cudaError_t merge_partials(const MergeArgs& m, cudaStream_t s);

// ---------------------------------------------------------------- layer backward
// Causal GQA attention backward on tcgen05 (tc_attention_bwd.cu); every tensor dense, token-major.
struct AttnBwdArgs {
  const void* q; const void* k; const void* v; const void* dout;  // bf16 [B][S][Hq*dh], [B][S][Hkv*dh], dO like q
  const float* lse; const float* dsum; int lse_ld;  // [B*Hq][lse_ld >= S rounded up to 128]: forward lse, rowsum(dO*O)
  float* dq;   // [B][S][Hq*dh] float32, 32-byte aligned
  float* dkv;  // [B][S][2*Hkv*dh] float32: dK then dV per row, 32-byte aligned
  int B, S, Hq, Hkv, dh;
  float scale;
};
cudaError_t attention_backward_tc(const AttnBwdArgs& a, int* status, cudaStream_t s);
// dsum[(b * Hq + h) * ld + t] = sum_i dO * O over head h of token t (bf16 inputs).
cudaError_t attention_dsum(const void* dout, const void* o, int B, int S, int Hq, int dh, int ld, float* dsum,
                           cudaStream_t s);
// Gate and router-MLP backward (backward.cu).
struct RouterBwdArgs {
  const float* dy; int width;        // [B*S][width] dK | dV
  const float* xkv; int ld_xkv;      // the three projected sources: X [W_k | W_v] rows (stride ld_xkv),
  const float* ema; const float* m3; //   their EMA and their recalled mean ([B*S][width])
  const float* lam; float* dlam;     // [B*S][3]; dlam (nullable) <- dL/dlam
  const float* hrec; int rh;         // [B*S][2 rh] router pre-activation as hi and lo parts
  int r_inter;                       // 1: hi, lo interleaved per 128 hidden units; 0: all hi then all lo
  const float* w_r2;                 // [rh][3]
  void* dh;                          // [B*S][rh] bf16 <- dL/dh
  float* dw_r2;                      // [rh][3] += GELU(h)^T dz (zero it first)
  int B, S, route_mode, tiers;
};
cudaError_t router_backward(const RouterBwdArgs& a, cudaStream_t s);
// U = lam1 dY + EMA^T(lam2 dY) + M^T(lam3 dY) in the projected space (backward.cu).
struct MemAdjArgs {
  const float* dy; int width; const float* lam; const int* cnt;
  const int* nrec; const int* recoff; const int* list;  // recall lists of the full blocks (block_lists, own 0,
  const int* pairoff; const int* pairbj;                //   32 tokens per tile: a "pair" is a 64-entry chunk)
  int B, S, nblk, blk;
  float alpha;
  float* gsum;  // [B][nblk][width] scratch
  float* rsum;  // [B][ceil(S/blk)][width] scratch
  float* cs;    // [B][ceil(S/blk)+1][width] scratch
  void* u; int ldu;  // bf16 rows of U (stride ldu)
};
cudaError_t memory_adjoint(const MemAdjArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- decode
struct DecodeArgs {
  // packed weights
  const void* wcatT; int Ntot; int d; int x_bf16;
  const float* w_r2; const double* pT64;
  // layout of the fused projection row
  int dq, dkv, rh, nb, rh_segs;  // rh_segs: 2 for bf16 (hi+lo), 1 for f32
  int r_inter;                   // hi/lo rows interleaved per 128 hidden units (else [hi | lo])
  int B, Hq, Hkv, dh, blk, R, Lmax, maxblk;
  float alpha, scale;
  int route_mode, tiers;         // routing gate variant and active tiers (route_gate)
  const void* x_new;             // [B, d]
  void* out;                     // [B, dq]
  // state
  int* pos; void* kcache; void* vcache; float* ema; float* blk_sum; double* blk_x;
  float* summ; uint32_t* scode;
  // scratch
  float* y;                      // [B, Ntot] projection row
  float* y2 = nullptr;           // [B, Ntot] second halves of the rows the batch-1 GEMV splits (gemv_split_row on)
  float* qf;                     // [B, dq] float32 query
  float* part;                   // split-KV partials
  int nsplit;
  unsigned long long* sync;      // the decode state's grid-barrier arrival count (only grows)
  int* status;
  cudaEvent_t* prof;             // 5 events around the 4 stages, or NULL
};
// bf16: one cooperative launch of decode_fused_kernel over all SMs (nsplit = (SMs - B) / (B * Hkv)
// attention units); float32: GEMV, token update, split-KV attention and merge as four launches.
cudaError_t decode_step(const DecodeArgs& a, cudaStream_t s);

// Waits `limit_us` on an mbarrier nothing arrives at; *result = 1 if the wait (wrongly) completed.
cudaError_t selftest_wait_timeout(int limit_us, int* status, int* result, cudaStream_t s);

}  // namespace mka
