// C ABI of libmka.so: argument checks, buffer layouts and launch sequences.
// Declarations and the contract of every entry point are in include/mka.h.
#include <math.h>
#include <stdarg.h>
#include <mutex>
#include <stdio.h>
#include <string.h>
#include <string>

#include "../../include/mka.h"
#include "common.cuh"
#include "kernels.h"

using namespace mka;

// Device status block: kernels record device-side errors in word 0 (never trap); words 1-3
// hold the test-only wait-limit override (see wait_limit in common.cuh).
__device__ __align__(16) int g_mka_status[4] = {0, 0, 0, 0};

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define CUDA_TRY(expr)                                                                        \
  do {                                                                                        \
    cudaError_t e_ = (expr);                                                                  \
    if (e_ != cudaSuccess) return fail(MKA_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

int* status_ptr() {
  static std::mutex mu;
  static int* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mka_status) != cudaSuccess) return nullptr;
    ptrs[dev] = (int*)p;
  }
  return ptrs[dev];
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

inline size_t al(size_t x) { return (x + 255) & ~(size_t)255; }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

struct Dims {
  int B, S, d, Hq, Hkv, dh, rh, blk, R, nb, bf16, elem;
  int dq, dkv, width, nblk, T;
  float alpha, scale;
  int route, tiers;  // routing gate variant; active tiers (MKA_TIER_* mask, never 0)
  int paths;         // 1 FastMKA, 3 full MKA
  int block_sparse;  // Block-MKA's block-sparse attention
};

int check_cfg(const mka_config* c, Dims* o) {
  if (!c) return fail(MKA_ERR_INVALID_ARG, "cfg is NULL");
  if (c->batch < 1 || c->seq < 1) return fail(MKA_ERR_INVALID_ARG, "batch and seq must be >= 1");
  if (c->d_model < 64 || c->d_model % 64) return fail(MKA_ERR_UNSUPPORTED, "d_model must be a positive multiple of 64");
  if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads)
    return fail(MKA_ERR_INVALID_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  if (c->d_head != 64 && c->d_head != 128) return fail(MKA_ERR_UNSUPPORTED, "d_head must be 64 or 128");
  if (c->router_hidden < 8 || c->router_hidden % 8 || c->router_hidden > 1024)
    return fail(MKA_ERR_UNSUPPORTED, "router_hidden must be a multiple of 8 in [8, 1024]");
  if (!(c->ema_alpha >= 0.f && c->ema_alpha <= 1.f)) return fail(MKA_ERR_INVALID_ARG, "ema_alpha must be in [0, 1]");
  if (c->block_size < 1) return fail(MKA_ERR_INVALID_ARG, "block_size must be >= 1");
  if (c->recall_r < 1 || c->recall_r > 64) return fail(MKA_ERR_UNSUPPORTED, "recall_r must be in [1, 64]");
  if (c->hash_bits < 1 || c->hash_bits > 32) return fail(MKA_ERR_UNSUPPORTED, "hash_bits must be in [1, 32]");
  if (c->dtype != MKA_F32 && c->dtype != MKA_BF16) return fail(MKA_ERR_INVALID_ARG, "dtype must be MKA_F32 or MKA_BF16");
  if (c->route_mode < MKA_ROUTE_SOFT || c->route_mode > MKA_ROUTE_TOP2)
    return fail(MKA_ERR_INVALID_ARG, "route_mode must be one of MKA_ROUTE_*");
  if (c->tiers & ~(MKA_TIER_L1 | MKA_TIER_L2 | MKA_TIER_L3))
    return fail(MKA_ERR_INVALID_ARG, "tiers must be a mask of MKA_TIER_L1 | MKA_TIER_L2 | MKA_TIER_L3");
  if (c->attention_paths != 0 && c->attention_paths != 1 && c->attention_paths != 3)
    return fail(MKA_ERR_INVALID_ARG, "attention_paths must be 1 (FastMKA) or 3 (full MKA)");
  if (c->attention_paths == 3 && (c->dtype != MKA_BF16 || c->block_size % 128 || c->recall_r > 16))
    return fail(MKA_ERR_UNSUPPORTED, "full MKA needs bf16, a block_size that is a multiple of 128 and recall_r <= 16");
  if (c->block_sparse != 0 && c->block_sparse != 1) return fail(MKA_ERR_INVALID_ARG, "block_sparse must be 0 or 1");
  if (c->block_sparse && (c->attention_paths == 3 || c->dtype != MKA_BF16 || c->block_size % 128 || c->recall_r > 16))
    return fail(MKA_ERR_UNSUPPORTED,
                "block-sparse attention needs FastMKA, bf16, a block_size that is a multiple of 128 and recall_r <= 16");
  long long T = (long long)c->batch * c->seq;
  if (T > (1LL << 30)) return fail(MKA_ERR_UNSUPPORTED, "batch * seq too large");
  if ((c->seq + c->block_size - 1) / c->block_size > 65535) return fail(MKA_ERR_UNSUPPORTED, "seq / block_size > 65535");
  Dims& d = *o;
  d.B = c->batch;
  d.S = c->seq;
  d.d = c->d_model;
  d.Hq = c->n_q_heads;
  d.Hkv = c->n_kv_heads;
  d.dh = c->d_head;
  d.rh = c->router_hidden;
  d.blk = c->block_size;
  d.R = c->recall_r;
  d.nb = c->hash_bits;
  d.bf16 = c->dtype == MKA_BF16;
  d.elem = d.bf16 ? 2 : 4;
  d.dq = d.Hq * d.dh;
  d.dkv = d.Hkv * d.dh;
  d.width = 2 * d.dkv;
  d.nblk = d.S / d.blk;
  d.T = (int)T;
  d.alpha = c->ema_alpha;
  d.route = c->route_mode;
  d.paths = c->attention_paths == 3 ? 3 : 1;
  d.block_sparse = c->block_sparse;
  d.tiers = c->tiers ? c->tiers : (MKA_TIER_L1 | MKA_TIER_L2 | MKA_TIER_L3);
  d.scale = c->attn_scale > 0.f ? c->attn_scale : 1.f / sqrtf((float)d.dh);
  return MKA_OK;
}

// ---------------------------------------------------------------- packed weights
struct PackLayout {
  int Ntot, Npad, seg_q, seg_k, seg_v, seg_r, seg_rlo, seg_p, rh_segs;
  int router_fused;  // bf16 with 256-aligned router rows: hi/lo interleaved per 128 units, GELU.W_r2 in the GEMM epilogue
  size_t wcat, wr2, pT64, p64, wqr32, wr1T, total;
};
PackLayout pack_layout(const Dims& d) {
  PackLayout p;
  p.rh_segs = d.bf16 ? 2 : 1;
  p.seg_q = 0;
  p.seg_k = d.dq;
  p.seg_v = d.dq + d.dkv;
  p.seg_r = d.dq + 2 * d.dkv;
  p.seg_rlo = d.bf16 ? p.seg_r + d.rh : -1;
  p.seg_p = p.seg_r + p.rh_segs * d.rh;
  p.Ntot = p.seg_p + d.nb;
  p.Npad = (p.Ntot + 127) / 128 * 128;
  p.router_fused = d.bf16 && (p.seg_r % 256 == 0) && (d.rh % 128 == 0);
  size_t o = 0;
  p.wcat = o; o += al((size_t)p.Npad * d.d * d.elem);
  p.wr2 = o; o += al((size_t)d.rh * 3 * 4);
  p.pT64 = o; o += al((size_t)d.nb * d.d * 8);
  p.p64 = o; o += al((size_t)d.d * 32 * 8);
  p.wqr32 = o; o += al((size_t)d.rh * d.d * 4);
  p.wr1T = o; o += al((size_t)d.rh * d.dq * d.elem);
  p.total = o;
  return p;
}

// ---------------------------------------------------------------- prefill workspace
struct PrefillWs {
  size_t q, xkv, h1, h2, proj, lam, tcode, xsum, bsum, bend, gend, carry, scode, idx, cnt, k, v, v2;
  size_t g_nrec, g_recoff, g_cursor, g_pairoff, g_pairbj, g_list, g_ptok, g_pinfo, part_o, part_lse, total;
};
// Block-gathered attention (Block-MKA block-sparse, full MKA's recalled-block path): every L3
// block, the last partial one included, has a token list; each token keeps one partial result
// per attended block: R recalled, plus its own block for Block-MKA.
static int gathered_blocks(const Dims& d) { return (d.S + d.blk - 1) / d.blk; }
static int gathered_slots(const Dims& d) { return d.R + (d.block_sparse ? 1 : 0); }
static int gathered_tpt(const Dims& d) { return 128 / gathered_rows_per_token(d.Hq / d.Hkv); }
PrefillWs prefill_ws(const Dims& d) {
  PrefillWs w;
  size_t T = d.T, o = 0;
  w.q = o; o += al(T * d.dq * d.elem);
  w.xkv = o; o += al(T * d.width * 4);
  w.h1 = o; o += al(T * d.rh * 4);
  w.h2 = o; o += d.bf16 ? al(T * d.rh * 4) : 0;
  w.proj = o; o += al(T * d.nb * 4);
  w.lam = o; o += al(T * 3 * 4);
  w.tcode = o; o += al(T * 4);
  w.xsum = o; o += al(summary_codes_scratch(d.d, d.B, d.nblk));
  w.bsum = o; o += al((size_t)d.B * d.nblk * d.width * 4);
  w.bend = o; o += al((size_t)d.B * d.nblk * d.width * 4);
  w.gend = o; o += al((size_t)d.B * d.nblk * 8 * d.width * 4);
  w.carry = o; o += al((size_t)d.B * (d.nblk + 1) * d.width * 4);
  w.scode = o; o += al((size_t)d.B * d.nblk * 4);
  w.idx = o; o += al(T * d.R * 4);
  w.cnt = o; o += al(T * 4);
  w.k = o; o += al(T * d.dkv * d.elem);
  w.v = o; o += al(T * d.dkv * d.elem);
  w.v2 = o; o += d.paths == 3 ? al(T * d.dkv * 4) : 0;  // full MKA: the L2 path's value M2 W_v
  const bool ga = d.paths == 3 || d.block_sparse;
  const size_t nbj = ga ? (size_t)d.B * gathered_blocks(d) : 0, ns = ga ? gathered_slots(d) : 0;
  w.g_nrec = o; o += al(nbj * 4);
  w.g_recoff = o; o += al(nbj * 4);
  w.g_cursor = o; o += al(nbj * 4);
  w.g_pairoff = o; o += ga ? al((nbj + 1) * 4) : 0;
  w.g_pairbj = o; o += ga ? al(gathered_max_pairs(T, d.R, d.block_sparse, gathered_tpt(d), nbj) * 4) : 0;
  w.g_list = o; o += ga ? al(T * d.R * 4) : 0;
  const size_t maxp = ga ? gathered_max_pairs(T, d.R, d.block_sparse, gathered_tpt(d), nbj) : 0;
  w.g_ptok = o; o += al(maxp * 2 * (ga ? gathered_tpt(d) : 0) * 4);
  w.g_pinfo = o; o += al(maxp * 4);
  w.part_o = o; o += al(T * ns * d.dq * 2);
  w.part_lse = o; o += al(T * ns * d.Hq * 4);
  w.total = o;
  return w;
}

// ---------------------------------------------------------------- decode state
struct StateLayout {
  int Lmax, maxblk;
  size_t pos, sync, kc, vc, ema, blk_sum, blk_x, summ, scode, total;
};
StateLayout state_layout(const Dims& d, int Lmax) {
  StateLayout s;
  s.Lmax = Lmax;
  s.maxblk = Lmax / d.blk;
  size_t o = 0, B = d.B;
  s.pos = o; o += al(B * 4);
  s.sync = o; o += al(8 * decode_sync_words(d.B, d.Hkv));
  s.kc = o; o += al(B * Lmax * d.dkv * d.elem);
  s.vc = o; o += al(B * Lmax * d.dkv * d.elem);
  s.ema = o; o += al(B * d.width * 4);
  s.blk_sum = o; o += al(B * d.width * 4);
  s.blk_x = o; o += al(B * d.d * 8);
  s.summ = o; o += al(B * (size_t)s.maxblk * d.width * 4);
  s.scode = o; o += al(B * (size_t)s.maxblk * 4);
  s.total = o;
  return s;
}

int decode_nsplit(const Dims& d, int Lmax) {
  int sms = sm_count();
  int ns;
  // fused bf16 launch: one attention unit per CTA not busy with the token update (32 of them)
  if (d.bf16) ns = (2 * sms - 32) / (d.B * d.Hkv);
  else ns = (2 * sms + d.B * d.Hq - 1) / (d.B * d.Hq);
  int cap = (Lmax + 127) / 128;
  if (ns > cap) ns = cap;
  if (ns < 1) ns = 1;
  if (ns > 512) ns = 512;
  return ns;
}

struct DecodeWs {
  int nsplit;
  size_t y, y2, qf, part, total;
};
DecodeWs decode_ws(const Dims& d, int Lmax) {
  DecodeWs w;
  PackLayout p = pack_layout(d);
  w.nsplit = decode_nsplit(d, Lmax);
  size_t o = 0, B = d.B;
  w.y = o; o += al(B * p.Ntot * 4);
  w.y2 = o; o += al(B * p.Ntot * 4);
  w.qf = o; o += al(B * d.dq * 4);
  w.part = o; o += al(B * d.Hq * (size_t)w.nsplit * (d.dh + 4) * 4);  // records of part_rec(dh) floats
  w.total = o;
  return w;
}

inline char* P(void* base, size_t off) { return (char*)base + off; }

// ---------------------------------------------------------------- stage timing
constexpr int kMaxStages = 16;
struct Profiler {
  bool on = false;
  bool created = false;
  int n = 0;  // events recorded by the last call
  cudaEvent_t ev[kMaxStages + 1];
  cudaError_t mark(cudaStream_t s) {
    if (!on || n > kMaxStages) return cudaSuccess;
    return cudaEventRecord(ev[n++], s);
  }
};
Profiler g_prof;

inline void prof_begin() { g_prof.n = 0; }
#define STAGE(s) CUDA_TRY(g_prof.mark(s))

// ---------------------------------------------------------------- concurrent branches
// Library-owned streams of the current device for the independent memory kernels of a
// prefill (they are small enough at a few thousand tokens that running them one after
// another costs mostly launch and ramp time).  Work is forked from the caller's stream
// with an event and joined back with events before the call's later kernels, so the
// caller's stream orders everything and stream capture sees one fork/join graph.  The
// events are shared, so the enqueue sequence holds aux_mutex().
struct AuxStreams {
  cudaStream_t st[2];
  cudaEvent_t fork_pre, fork, join[3];
};
std::mutex& aux_mutex() {
  static std::mutex mu;
  return mu;
}
// Called with aux_mutex() held.  nullptr when the streams cannot be made.
AuxStreams* aux_streams() {
  static AuxStreams per_dev[64];
  static bool made[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  AuxStreams& a = per_dev[dev];
  if (!made[dev]) {
    for (int i = 0; i < 2; ++i)
      if (cudaStreamCreateWithFlags(&a.st[i], cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&a.fork_pre, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    for (int i = 0; i < 3; ++i)
      if (cudaEventCreateWithFlags(&a.join[i], cudaEventDisableTiming) != cudaSuccess) return nullptr;
    made[dev] = true;
  }
  return &a;
}

}  // namespace

int mka::set_last_error(int code, const char* msg) {
  g_err = msg;
  return code;
}

extern "C" {

const char* mka_version(void) { return "fastmka-b200 0.1 (sm_100a)"; }

int mka_selftest_wait_timeout(int limit_us, int* result, void* stream) {
  if (limit_us < 1 || limit_us > 1000000 || !result) return fail(MKA_ERR_INVALID_ARG, "limit_us in [1, 1e6] and result");
  int* st = status_ptr();
  if (!st) return fail(MKA_ERR_CUDA, "no CUDA device");
  CUDA_TRY(selftest_wait_timeout(limit_us, st, result, (cudaStream_t)stream));
  return MKA_OK;
}

int mka_set_wait_limit(unsigned long long limit_ns, int wait_classes) {
  if (wait_classes & ~(MKA_WAIT_PIPELINE | MKA_WAIT_GRID))
    return fail(MKA_ERR_INVALID_ARG, "wait_classes must be a mask of MKA_WAIT_PIPELINE and MKA_WAIT_GRID");
  int* st = status_ptr();
  if (!st) return fail(MKA_ERR_CUDA, "no CUDA device");
  int words[3] = {limit_ns ? wait_classes : 0, (int)(limit_ns & 0xffffffffull), (int)(limit_ns >> 32)};
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpy(st + 1, words, sizeof(words), cudaMemcpyHostToDevice));
  return MKA_OK;
}

int mka_profile_enable(int enable) {
  if (enable && !g_prof.created) {
    for (int i = 0; i <= kMaxStages; ++i) CUDA_TRY(cudaEventCreate(&g_prof.ev[i]));
    g_prof.created = true;
  }
  g_prof.on = enable != 0;
  g_prof.n = 0;
  return MKA_OK;
}

int mka_profile_read(float* ms, int max_stages) {
  if (!g_prof.created || g_prof.n < 2) return fail(MKA_ERR_INVALID_ARG, "no profiled call to read");
  CUDA_TRY(cudaEventSynchronize(g_prof.ev[g_prof.n - 1]));
  int stages = g_prof.n - 1;
  for (int i = 0; i < stages && i < max_stages; ++i) CUDA_TRY(cudaEventElapsedTime(&ms[i], g_prof.ev[i], g_prof.ev[i + 1]));
  return stages;
}
const char* mka_last_error(void) { return g_err.c_str(); }

int mka_status(void) {
  int* p = status_ptr();
  if (!p) return fail(MKA_ERR_CUDA, "no CUDA device");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(MKA_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
  int v = 0;
  e = cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(MKA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  int z = 0;
  cudaMemcpy(p, &z, sizeof(int), cudaMemcpyHostToDevice);
  return v;
}

size_t mka_packed_weights_size(const mka_config* cfg) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK) return 0;
  return pack_layout(d).total;
}

size_t mka_workspace_size(const mka_config* cfg) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK) return 0;
  return prefill_ws(d).total;
}

size_t mka_router_workspace_size(const mka_config* cfg) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK) return 0;
  return al((size_t)d.rh * d.dq * d.elem) + al((size_t)d.rh * 3 * 4) + al((size_t)d.T * d.rh * 4);
}

static const int kEmaChunk = 64;

size_t mka_session_ema_workspace_size(const mka_config* cfg) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK) return 0;
  size_t nch = d.S / kEmaChunk;
  return al((size_t)d.B * nch * d.d * 4) + al((size_t)d.B * (nch + 1) * d.d * 4);
}

size_t mka_longterm_recall_workspace_size(const mka_config* cfg) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK) return 0;
  size_t T = d.T;
  return al((size_t)d.nb * d.d * d.elem) + al((size_t)d.nb * d.d * 8) + al((size_t)d.d * 32 * 8) + al(T * d.nb * 4) +
         al(T * 4) + al(summary_codes_scratch(d.d, d.B, d.nblk)) + al((size_t)d.B * d.nblk * d.d * 4) +
         al((size_t)d.B * d.nblk * 4) + al(T * 4);
}

size_t mka_state_size(const mka_config* cfg, int32_t max_positions) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK || max_positions < 1) return 0;
  return state_layout(d, max_positions).total;
}

size_t mka_decode_workspace_size(const mka_config* cfg, int32_t max_positions) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK || max_positions < 1) return 0;
  return decode_ws(d, max_positions).total;
}

int mka_pack_weights(const mka_config* cfg, const mka_weights* w, void* packed, size_t packed_bytes, void* stream) {
  Dims d;
  int rc = check_cfg(cfg, &d);
  if (rc) return rc;
  if (!w || !w->w_q || !w->w_k || !w->w_v || !w->w_r1 || !w->w_r2 || !w->hash_proj || !packed)
    return fail(MKA_ERR_INVALID_ARG, "NULL weight or packed pointer");
  if (!aligned16(w->w_q) || !aligned16(w->w_k) || !aligned16(w->w_v) || !aligned16(w->w_r1) || !aligned16(packed))
    return fail(MKA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  PackLayout L = pack_layout(d);
  if (packed_bytes < L.total) return fail(MKA_ERR_WORKSPACE, "packed buffer %zu < %zu bytes", packed_bytes, L.total);
  cudaStream_t s = (cudaStream_t)stream;
  char* wc = P(packed, L.wcat);
  size_t row = (size_t)d.d * d.elem;
  CUDA_TRY(cudaMemsetAsync(wc, 0, (size_t)L.Npad * row, s));
  CUDA_TRY(transpose(w->w_q, d.d, d.dq, d.dq, wc + L.seg_q * row, d.d, d.elem, 0, s));
  CUDA_TRY(transpose(w->w_k, d.d, d.dkv, d.dkv, wc + L.seg_k * row, d.d, d.elem, 0, s));
  CUDA_TRY(transpose(w->w_v, d.d, d.dkv, d.dkv, wc + L.seg_v * row, d.d, d.elem, 0, s));
  CUDA_TRY(transpose(w->hash_proj, d.d, d.nb, d.nb, wc + L.seg_p * row, d.d, d.elem, 0, s));
  CUDA_TRY(transpose(w->hash_proj, d.d, d.nb, d.nb, P(packed, L.pT64), d.d, d.elem, 1, s));
  CUDA_TRY(widen_pad32_f64(w->hash_proj, d.d, d.nb, d.bf16, (double*)P(packed, L.p64), s));
  CUDA_TRY(widen_f32(w->w_r2, d.rh * 3, d.bf16, (float*)P(packed, L.wr2), s));
  // Router fold: (W_q W_r1)^T [rh, d] = W_r1^T [rh, dq] . W_q^T, float32 accumulation.
  CUDA_TRY(transpose(w->w_r1, d.dq, d.rh, d.rh, P(packed, L.wr1T), d.dq, d.elem, 0, s));
  Epilogue ep{};
  ep.nseg = 1;
  ep.seg[0] = OutSeg{0, d.d, P(packed, L.wqr32), d.d, 0};
  CUDA_TRY(gemm_tn_ffma(P(packed, L.wr1T), d.dq, d.bf16, w->w_q, d.dq, d.bf16, d.rh, d.d, d.dq, ep, s));
  if (d.bf16 && L.router_fused) {
    CUDA_TRY(split_hi_lo_interleaved((const float*)P(packed, L.wqr32), d.rh, d.d, wc + L.seg_r * row, s));
  } else if (d.bf16) {
    CUDA_TRY(split_hi_lo((const float*)P(packed, L.wqr32), d.rh * d.d, wc + L.seg_r * row, wc + L.seg_rlo * row, s));
  } else {
    CUDA_TRY(cudaMemcpyAsync(wc + L.seg_r * row, P(packed, L.wqr32), (size_t)d.rh * d.d * 4, cudaMemcpyDeviceToDevice, s));
  }
  return MKA_OK;
}

int mka_state_init(const mka_config* cfg, int32_t max_positions, void* state, size_t state_bytes, void* stream) {
  Dims d;
  int rc = check_cfg(cfg, &d);
  if (rc) return rc;
  if (max_positions < 1) return fail(MKA_ERR_INVALID_ARG, "max_positions must be >= 1");
  if (!state || !aligned16(state)) return fail(MKA_ERR_INVALID_ARG, "state must be a 16-byte aligned device pointer");
  StateLayout L = state_layout(d, max_positions);
  if (state_bytes < L.total) return fail(MKA_ERR_WORKSPACE, "state buffer %zu < %zu bytes", state_bytes, L.total);
  CUDA_TRY(cudaMemsetAsync(state, 0, L.total, (cudaStream_t)stream));
  return MKA_OK;
}

int mka_router(const mka_config* cfg, const void* q, const void* w_r1, const void* w_r2, float* lambda, void* ws,
               size_t ws_bytes, void* stream) {
  Dims d;
  int rc = check_cfg(cfg, &d);
  if (rc) return rc;
  if (!q || !w_r1 || !w_r2 || !lambda || !ws) return fail(MKA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(q) || !aligned16(w_r1) || !aligned16(lambda) || !aligned16(ws))
    return fail(MKA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  size_t need = mka_router_workspace_size(cfg);
  if (ws_bytes < need) return fail(MKA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  cudaStream_t s = (cudaStream_t)stream;
  char* w1T = (char*)ws;
  float* wr2 = (float*)(w1T + al((size_t)d.rh * d.dq * d.elem));
  float* h = (float*)((char*)wr2 + al((size_t)d.rh * 3 * 4));
  CUDA_TRY(transpose(w_r1, d.dq, d.rh, d.rh, w1T, d.dq, d.elem, 0, s));
  CUDA_TRY(widen_f32(w_r2, d.rh * 3, d.bf16, wr2, s));
  Epilogue ep{};
  ep.nseg = 1;
  ep.seg[0] = OutSeg{0, d.rh, h, d.rh, 0};
  if (d.bf16) CUDA_TRY(gemm_tn_bf16_tc(q, d.dq, w1T, d.dq, d.T, d.rh, d.dq, ep, status_ptr(), s));
  else CUDA_TRY(gemm_tn_ffma(q, d.dq, 0, w1T, d.dq, 0, d.T, d.rh, d.dq, ep, s));
  CUDA_TRY(router_tail(h, nullptr, d.rh, d.T, d.rh, wr2, d.route, d.tiers, lambda, s));
  return MKA_OK;
}

int mka_session_ema(const mka_config* cfg, const void* x, const float* carry_in, float* m2, float* carry_out,
                    void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  int rc = check_cfg(cfg, &d);
  if (rc) return rc;
  if (!x || !m2 || !ws) return fail(MKA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(x) || !aligned16(m2) || !aligned16(ws) || (carry_in && !aligned16(carry_in)) ||
      (carry_out && !aligned16(carry_out)))
    return fail(MKA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  size_t need = mka_session_ema_workspace_size(cfg);
  if (ws_bytes < need) return fail(MKA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  cudaStream_t s = (cudaStream_t)stream;
  int nch = d.S / kEmaChunk;
  float* bend = (float*)ws;
  float* carry = (float*)((char*)ws + al((size_t)d.B * nch * d.d * 4));
  double apb = pow((double)d.alpha, (double)kEmaChunk);
  CUDA_TRY(block_reduce(x, d.bf16, d.d, d.d, d.B, d.S, nch, kEmaChunk, d.alpha, nullptr, 0, bend, nullptr, s));
  CUDA_TRY(ema_carry(bend, d.d, d.B, nch, (float)apb, carry_in, carry, s));
  CUDA_TRY(ema_apply(x, d.bf16, d.d, d.B, d.S, nch, kEmaChunk, d.alpha, carry, m2, carry_out, s));
  return MKA_OK;
}

int mka_longterm_recall(const mka_config* cfg, const void* x, const void* hash_proj, int32_t* idx, int32_t* count,
                        float* m3, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  int rc = check_cfg(cfg, &d);
  if (rc) return rc;
  if (!x || !hash_proj || !idx || !ws) return fail(MKA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(x) || !aligned16(ws) || !aligned16(idx) || (m3 && !aligned16(m3)))
    return fail(MKA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  size_t need = mka_longterm_recall_workspace_size(cfg);
  if (ws_bytes < need) return fail(MKA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  cudaStream_t s = (cudaStream_t)stream;
  size_t T = d.T;
  char* o = (char*)ws;
  void* pT = o; o += al((size_t)d.nb * d.d * d.elem);
  double* pT64 = (double*)o; o += al((size_t)d.nb * d.d * 8);
  double* p64 = (double*)o; o += al((size_t)d.d * 32 * 8);
  float* proj = (float*)o; o += al(T * d.nb * 4);
  uint32_t* tcode = (uint32_t*)o; o += al(T * 4);
  double* xsum = (double*)o; o += al(summary_codes_scratch(d.d, d.B, d.nblk));
  float* bsum = (float*)o; o += al((size_t)d.B * d.nblk * d.d * 4);
  uint32_t* scode = (uint32_t*)o; o += al((size_t)d.B * d.nblk * 4);
  int* cnt = count ? count : (int*)o;
  CUDA_TRY(transpose(hash_proj, d.d, d.nb, d.nb, pT, d.d, d.elem, 0, s));
  CUDA_TRY(transpose(hash_proj, d.d, d.nb, d.nb, pT64, d.d, d.elem, 1, s));
  CUDA_TRY(widen_pad32_f64(hash_proj, d.d, d.nb, d.bf16, p64, s));
  Epilogue ep{};
  ep.nseg = 1;
  ep.seg[0] = OutSeg{0, d.nb, proj, d.nb, 0};
  if (d.bf16) CUDA_TRY(gemm_tn_bf16_tc(x, d.d, pT, d.d, d.T, d.nb, d.d, ep, status_ptr(), s));
  else CUDA_TRY(gemm_tn_ffma(x, d.d, 0, pT, d.d, 0, d.T, d.nb, d.d, ep, s));
  HashArgs ha{proj, d.nb, x, d.bf16, pT64, d.d, d.nb, d.d};
  CUDA_TRY(token_codes(ha, d.T, tcode, s));
  CUDA_TRY(summary_codes(x, d.bf16, d.d, d.B, d.S, d.nblk, d.blk, p64, d.nb, xsum, scode, d.nblk, s));
  CUDA_TRY(recall_select(tcode, scode, d.nblk, d.B, d.S, d.nblk, d.blk, d.R, idx, cnt, s));
  if (m3) {
    CUDA_TRY(block_reduce(x, d.bf16, d.d, d.d, d.B, d.S, d.nblk, d.blk, d.alpha, bsum, (long long)d.nblk * d.d, nullptr,
                          nullptr, s));
    CUDA_TRY(gather_mean(idx, cnt, d.R, bsum, d.nblk, d.d, d.blk, d.B, d.S, m3, s));
  }
  return MKA_OK;
}

// The prefill forward; lse (nullable) receives the attention's per-row log2 normaliser,
// [B*Hq][S rounded up to 128], for the backward.
static int prefill_forward(const mka_config* cfg, const void* packed, const void* x, void* out, float* lambda_out,
                           int32_t* recall_idx_out, void* state, size_t state_bytes, int32_t max_positions, void* ws,
                           size_t ws_bytes, void* stream, float* lse) {
  Dims d;
  int rc = check_cfg(cfg, &d);
  if (rc) return rc;
  if (!packed || !x || !out || !ws) return fail(MKA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(packed) || !aligned16(x) || !aligned16(out) || !aligned16(ws) ||
      (lambda_out && !aligned16(lambda_out)) || (recall_idx_out && !aligned16(recall_idx_out)) ||
      (state && !aligned16(state)))
    return fail(MKA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((d.paths == 3 || d.block_sparse) && ((uintptr_t)ws & 31))  // 32-byte stores into its partial results
    return fail(MKA_ERR_INVALID_ARG, "full MKA and block-sparse attention need a 32-byte aligned workspace");
  PrefillWs W = prefill_ws(d);
  if (ws_bytes < W.total) return fail(MKA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, W.total);
  StateLayout SL{};
  if (state && (d.paths == 3 || d.block_sparse))
    return fail(MKA_ERR_UNSUPPORTED, "full MKA and block-sparse attention have no decode state");
  if (state) {
    if (max_positions < d.S) return fail(MKA_ERR_CAPACITY, "max_positions %d < seq %d", max_positions, d.S);
    SL = state_layout(d, max_positions);
    if (state_bytes < SL.total) return fail(MKA_ERR_WORKSPACE, "state buffer %zu < %zu bytes", state_bytes, SL.total);
  }
  PackLayout PL = pack_layout(d);
  cudaStream_t s = (cudaStream_t)stream;
  void* q = P(ws, W.q);
  float* xkv = (float*)P(ws, W.xkv);
  float* h1 = (float*)P(ws, W.h1);
  float* h2 = d.bf16 ? (float*)P(ws, W.h2) : nullptr;
  float* proj = (float*)P(ws, W.proj);
  float* lam = lambda_out ? lambda_out : (float*)P(ws, W.lam);
  uint32_t* tcode = (uint32_t*)P(ws, W.tcode);
  double* xsum = (double*)P(ws, W.xsum);
  float* bsum = state ? (float*)P(state, SL.summ) : (float*)P(ws, W.bsum);
  long long bsum_bstride = (long long)(state ? SL.maxblk : d.nblk) * d.width;
  float* bend = (float*)P(ws, W.bend);
  float* gend = (float*)P(ws, W.gend);
  float* carry = (float*)P(ws, W.carry);
  uint32_t* scode = state ? (uint32_t*)P(state, SL.scode) : (uint32_t*)P(ws, W.scode);
  int code_bstride = state ? SL.maxblk : d.nblk;
  int* idx = recall_idx_out ? recall_idx_out : (int*)P(ws, W.idx);
  int* cnt = (int*)P(ws, W.cnt);
  void* kbuf = state ? P(state, SL.kc) : P(ws, W.k);
  void* vbuf = state ? P(state, SL.vc) : P(ws, W.v);
  long long kv_bstride = (long long)(state ? max_positions : d.S) * d.dkv;
  const void* wcat = P((void*)packed, PL.wcat);

  // 2-4: router tail, L3 codes, block sums / EMA end states, carries.  With stage timing on
  // they run one after another on the caller's stream (so each stage has its own time);
  // otherwise as concurrent branches joined before the recall: the block codes (which read X
  // only) start before the projection GEMM and share the SMs with it, the router tail and
  // the token codes, and the block sums and carries, follow the GEMM.
  HashArgs ha{proj, d.nb, x, d.bf16, (const double*)P((void*)packed, PL.pT64), d.d, d.nb, d.d};
  const double* p64 = (const double*)P((void*)packed, PL.p64);
  auto k_router = [&](cudaStream_t st) {
    return PL.router_fused
               ? router_softmax(h1, d.rh / 128, d.T, d.route, d.tiers, lam, st)
               : router_tail(h1, h2, d.rh, d.T, d.rh, (const float*)P((void*)packed, PL.wr2), d.route, d.tiers, lam, st);
  };
  auto k_tcode = [&](cudaStream_t st) { return token_codes(ha, d.T, tcode, st); };
  auto k_bsum = [&](cudaStream_t st) {
    return block_reduce(xkv, 0, d.width, d.width, d.B, d.S, d.nblk, d.blk, d.alpha, bsum, bsum_bstride, bend, gend, st);
  };
  auto k_scode = [&](cudaStream_t st) {
    return summary_codes(x, d.bf16, d.d, d.B, d.S, d.nblk, d.blk, p64, d.nb, xsum, scode, code_bstride, st);
  };
  auto k_carry = [&](cudaStream_t st) {
    return ema_carry(bend, d.width, d.B, d.nblk, (float)pow((double)d.alpha, (double)d.blk), nullptr, carry, st);
  };
  auto k_tail = [&](cudaStream_t st) {
    return prefill_tail_state(xkv, d.width, d.width, x, d.bf16, d.d, d.B, d.S, d.blk, (float*)P(state, SL.blk_sum),
                              (double*)P(state, SL.blk_x), (int*)P(state, SL.pos), st);
  };
  // A decode step ORs the bits of a block's code in when the block closes: the codes of the
  // blocks this prefill does not finish start at zero, so a prefill redefines the whole state.
  if (state && SL.maxblk > d.nblk)
    CUDA_TRY(cudaMemset2DAsync(scode + d.nblk, (size_t)SL.maxblk * 4, 0, (size_t)(SL.maxblk - d.nblk) * 4, d.B, s));
  // and the decode step's grid barrier and completion counts start from zero
  if (state) CUDA_TRY(cudaMemsetAsync(P(state, SL.sync), 0, 8 * decode_sync_words(d.B, d.Hkv), s));
  std::unique_lock<std::mutex> aux_lock(aux_mutex(), std::defer_lock);
  AuxStreams* ax = nullptr;
  if (!g_prof.on) {
    aux_lock.lock();
    ax = aux_streams();
  }
  // With L3 off (MKA_TIER_L3 not set) its weight is 0: no codes and no recall, count 0 for every token.
  const bool l3 = (d.tiers & MKA_TIER_L3) != 0;
  prof_begin();
  if (ax && l3) {  // the L3 block codes read X only: they run beside the projection GEMM
    CUDA_TRY(cudaEventRecord(ax->fork_pre, s));
    CUDA_TRY(cudaStreamWaitEvent(ax->st[0], ax->fork_pre, 0));
    CUDA_TRY(k_scode(ax->st[0]));
  }
  STAGE(s);
  // 1. projections: q | XW_k | XW_v | X(W_q W_r1) | XP
  Epilogue ep{};
  int ns = 0;
  ep.seg[ns++] = OutSeg{PL.seg_q, PL.seg_k, q, d.dq, d.bf16};
  ep.seg[ns++] = OutSeg{PL.seg_k, PL.seg_r, xkv, d.width, 0};
  ep.seg[ns++] = OutSeg{PL.seg_r, PL.seg_r + d.rh, h1, d.rh, 0};
  if (d.bf16) ep.seg[ns++] = OutSeg{PL.seg_rlo, PL.seg_rlo + d.rh, h2, d.rh, 0};
  ep.seg[ns++] = OutSeg{PL.seg_p, PL.Ntot, proj, d.nb, 0};
  ep.nseg = ns;
  if (PL.router_fused) {  // hidden layer reduced in the epilogue; h1 holds the partials
    ep.r_begin = PL.seg_r;
    ep.r_end = PL.seg_r + 2 * d.rh;
    ep.w_r2 = (const float*)P((void*)packed, PL.wr2);
    ep.zpart = h1;
  }
  if (d.bf16) CUDA_TRY(gemm_tn_bf16_tc(x, d.d, wcat, d.d, d.T, PL.Ntot, d.d, ep, status_ptr(), s));
  else CUDA_TRY(gemm_tn_ffma(x, d.d, 0, wcat, d.d, 0, d.T, PL.Ntot, d.d, ep, s));
  STAGE(s);
  if (ax) {
    CUDA_TRY(cudaEventRecord(ax->fork, s));
    CUDA_TRY(cudaStreamWaitEvent(ax->st[0], ax->fork, 0));
    CUDA_TRY(cudaStreamWaitEvent(ax->st[1], ax->fork, 0));
    CUDA_TRY(cudaEventRecord(ax->join[0], ax->st[0]));  // the block codes, started before the GEMM
    if (state) CUDA_TRY(k_tail(ax->st[0]));  // reads x and xkv only; joined at the end
    CUDA_TRY(cudaEventRecord(ax->join[2], ax->st[0]));
    CUDA_TRY(k_router(ax->st[1]));
    if (l3) CUDA_TRY(k_tcode(ax->st[1]));
    CUDA_TRY(cudaEventRecord(ax->join[1], ax->st[1]));
    CUDA_TRY(k_bsum(s));
    CUDA_TRY(k_carry(s));
    CUDA_TRY(cudaStreamWaitEvent(s, ax->join[0], 0));
    CUDA_TRY(cudaStreamWaitEvent(s, ax->join[1], 0));
  } else {
    CUDA_TRY(k_router(s));
    STAGE(s);
    if (l3) CUDA_TRY(k_tcode(s));
    STAGE(s);
    CUDA_TRY(k_bsum(s));
    STAGE(s);
    if (l3) CUDA_TRY(k_scode(s));
    STAGE(s);
    CUDA_TRY(k_carry(s));
  }
  STAGE(s);
  if (l3) {
    CUDA_TRY(recall_select(tcode, scode, code_bstride, d.B, d.S, d.nblk, d.blk, d.R, idx, cnt, s));
  } else {
    CUDA_TRY(cudaMemsetAsync(cnt, 0, (size_t)d.T * sizeof(int), s));
    if (recall_idx_out) CUDA_TRY(cudaMemsetAsync(idx, 0xff, (size_t)d.T * d.R * sizeof(int), s));
  }
  STAGE(s);
  // 5. route-fuse -> K, V
  FuseArgs fa{};
  fa.xkv = xkv; fa.ld = d.width; fa.width = d.width; fa.lam = lam; fa.idx = idx; fa.count = cnt; fa.R = d.R;
  fa.bsum = bsum; fa.bsum_bstride = bsum_bstride; fa.carry = carry; fa.gend = gend;
  fa.B = d.B; fa.S = d.S; fa.nblk = d.nblk; fa.blk = d.blk; fa.dkv = d.dkv; fa.alpha = d.alpha;
  fa.k_out = kbuf; fa.v_out = vbuf; fa.kv_bstride = kv_bstride; fa.out_bf16 = d.bf16;
  fa.state_ema = state ? (float*)P(state, SL.ema) : nullptr;
  if (d.paths == 3) fa.v2_out = (float*)P(ws, W.v2);  // K, V <- the tokens' own; v2 <- M2 W_v
  CUDA_TRY(fuse_kv(fa, s));
  STAGE(s);
  // 6. causal GQA attention over the fused K/V (Block-MKA: none; its own-block part is gathered)
  AttnArgs aa{};
  aa.q = q; aa.q_bstride = (long long)d.S * d.dq; aa.q_ld = d.dq;
  aa.k = kbuf; aa.v = vbuf; aa.kv_bstride = kv_bstride; aa.kv_ld = d.dkv;
  aa.o = out; aa.o_bstride = (long long)d.S * d.dq; aa.o_ld = d.dq;
  aa.B = d.B; aa.S = d.S; aa.Hq = d.Hq; aa.Hkv = d.Hkv; aa.dh = d.dh; aa.scale = d.scale;
  if (lse) {
    aa.lse = lse;
    aa.lse_ld = (d.S + 127) / 128 * 128;
  }
  if (!d.block_sparse) {
    if (d.bf16) CUDA_TRY(attention_prefill_tc(aa, status_ptr(), s));
    else CUDA_TRY(attention_prefill(aa, 0, s));
  }
  if (d.block_sparse || d.paths == 3) {
    // Block-MKA: each token's own block (causal) and recalled blocks; full MKA: the recalled
    // blocks' tokens, then mixed with the causal output and the L2 value.  Rows are gathered
    // per block, attended on the tensor cores, and their per-block results merged.
    const int own = d.block_sparse, nball = gathered_blocks(d), ns = gathered_slots(d);
    int* nrec = (int*)P(ws, W.g_nrec);
    int* recoff = (int*)P(ws, W.g_recoff);
    int* pairoff = (int*)P(ws, W.g_pairoff);
    int* list = (int*)P(ws, W.g_list);
    int* pairbj = (int*)P(ws, W.g_pairbj);
    int* ptok = (int*)P(ws, W.g_ptok);
    int* pinfo = (int*)P(ws, W.g_pinfo);
    CUDA_TRY(block_lists(idx, cnt, d.B, d.S, d.R, d.blk, nball, own, own, gathered_tpt(d), nrec, recoff,
                         (int*)P(ws, W.g_cursor), pairoff, pairbj, list, ptok, pinfo, s));
    AttnArgs ag = aa;
    ag.g_pairoff = pairoff; ag.g_pinfo = pinfo; ag.g_ptok = ptok;
    ag.g_own = own; ag.nblk = nball; ag.blk = d.blk; ag.nslot = ns;
    ag.part_o = P(ws, W.part_o); ag.part_lse = (float*)P(ws, W.part_lse);
    CUDA_TRY(attention_prefill_tc(ag, status_ptr(), s));
    MergeArgs mg{};
    mg.part_o = ag.part_o; mg.part_lse = ag.part_lse; mg.nslot = ns; mg.cnt = cnt; mg.own = own;
    mg.B = d.B; mg.S = d.S; mg.Hq = d.Hq; mg.Hkv = d.Hkv; mg.dh = d.dh;
    mg.o = out; mg.o_bstride = (long long)d.S * d.dq; mg.o_ld = d.dq;
    if (d.paths == 3) {
      mg.lam = lam;
      mg.v2 = (const float*)P(ws, W.v2);
    }
    CUDA_TRY(merge_partials(mg, s));
  }
  STAGE(s);
  if (ax) {
    CUDA_TRY(cudaStreamWaitEvent(s, ax->join[2], 0));
  } else if (state) {
    CUDA_TRY(k_tail(s));
    STAGE(s);
  }
  return MKA_OK;
}

int mka_prefill_forward(const mka_config* cfg, const void* packed, const void* x, void* out, float* lambda_out,
                        int32_t* recall_idx_out, void* state, size_t state_bytes, int32_t max_positions, void* ws,
                        size_t ws_bytes, void* stream) {
  return prefill_forward(cfg, packed, x, out, lambda_out, recall_idx_out, state, state_bytes, max_positions, ws,
                         ws_bytes, stream, nullptr);
}

// ---------------------------------------------------------------- training: forward + backward
// The training workspace is the prefill workspace (whose activations the backward reads: q, the
// projected sources, lambda, the EMA carries, the block sums, the recall, the fused K/V) followed
// by the attention normalisers the training forward writes and the backward's own scratch.
struct TrainWs {
  PrefillWs fw;
  int Spad, ncat, nball;
  size_t lse, dsum, dq, dy, ema, m3, hrec, dlam, dh, gsum, rsum, cs, acat;
  size_t nrec, recoff, cursor, pairoff, pairbj, list, total;
};
static TrainWs train_ws(const Dims& d) {
  TrainWs w;
  w.fw = prefill_ws(d);
  const size_t T = d.T, W = d.width;
  w.Spad = (d.S + 127) / 128 * 128;
  w.ncat = d.dq + 2 * d.dkv;      // [dq | U] columns
  w.nball = (d.S + d.blk - 1) / d.blk;
  const size_t nbj = (size_t)d.B * d.nblk;
  size_t o = w.fw.total;
  w.lse = o; o += al((size_t)d.B * d.Hq * w.Spad * 4);
  w.dsum = o; o += al((size_t)d.B * d.Hq * w.Spad * 4);
  w.dq = o; o += al(T * d.dq * 4);
  w.dy = o; o += al(T * W * 4);
  w.ema = o; o += al(T * W * 4);
  w.m3 = o; o += al(T * W * 4);
  w.hrec = o; o += al(T * 2 * d.rh * 4);
  w.dlam = o; o += al(T * 3 * 4);
  w.dh = o; o += al(T * d.rh * 2);
  w.gsum = o; o += al(nbj * W * 4);
  w.rsum = o; o += al((size_t)d.B * w.nball * W * 4);
  w.cs = o; o += al((size_t)d.B * (w.nball + 1) * W * 4);
  w.acat = o; o += al(T * w.ncat * 2);
  w.nrec = o; o += al(nbj * 4);
  w.recoff = o; o += al(nbj * 4);
  w.cursor = o; o += al(nbj * 4);
  w.pairoff = o; o += al((nbj + 1) * 4);
  w.pairbj = o; o += al(gathered_max_pairs(T, d.R, 0, 32, nbj) * 4);
  w.list = o; o += al(T * d.R * 4);
  w.total = o;
  return w;
}

static int check_train(const mka_config* cfg, Dims* d) {
  int rc = check_cfg(cfg, d);
  if (rc) return rc;
  if (!d->bf16 || d->paths != 1 || d->block_sparse)
    return fail(MKA_ERR_UNSUPPORTED, "the layer backward needs bf16 FastMKA (attention_paths 1, no block_sparse)");
  if (d->rh % 32 || d->rh > 512) return fail(MKA_ERR_UNSUPPORTED, "the layer backward needs router_hidden a multiple of 32, at most 512");
  return MKA_OK;
}

size_t mka_train_workspace_size(const mka_config* cfg) {
  Dims d;
  if (check_cfg(cfg, &d) != MKA_OK || !d.bf16 || d.paths != 1 || d.block_sparse || d.rh % 32 || d.rh > 512) return 0;
  return train_ws(d).total;
}

int mka_prefill_forward_train(const mka_config* cfg, const void* packed, const void* x, void* out, void* ws,
                              size_t ws_bytes, void* stream) {
  Dims d;
  int rc = check_train(cfg, &d);
  if (rc) return rc;
  if (!ws) return fail(MKA_ERR_INVALID_ARG, "NULL pointer");
  if ((uintptr_t)ws & 31) return fail(MKA_ERR_INVALID_ARG, "the training workspace must be 32-byte aligned");
  TrainWs W = train_ws(d);
  if (ws_bytes < W.total) return fail(MKA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, W.total);
  // rows past S of the last query tile keep a defined normaliser (the backward masks them)
  CUDA_TRY(cudaMemsetAsync(P(ws, W.lse), 0, (size_t)d.B * d.Hq * W.Spad * 4, (cudaStream_t)stream));
  return prefill_forward(cfg, packed, x, out, nullptr, nullptr, nullptr, 0, 0, ws, ws_bytes, stream,
                         (float*)P(ws, W.lse));
}

int mka_prefill_backward(const mka_config* cfg, const void* packed, const void* x, const void* out, const void* dout,
                         void* dx, float* dw_q, float* dw_k, float* dw_v, float* dw_r1, float* dw_r2,
                         float* dlambda_out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  int rc = check_train(cfg, &d);
  if (rc) return rc;
  if (!packed || !x || !out || !dout || !dx || !dw_q || !dw_k || !dw_v || !dw_r1 || !dw_r2 || !ws)
    return fail(MKA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(packed) || !aligned16(x) || !aligned16(out) || !aligned16(dout) || !aligned16(dx) ||
      !aligned16(dw_q) || !aligned16(dw_k) || !aligned16(dw_v) || !aligned16(dw_r1) || !aligned16(dw_r2) ||
      (dlambda_out && !aligned16(dlambda_out)))
    return fail(MKA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((uintptr_t)ws & 31) return fail(MKA_ERR_INVALID_ARG, "the training workspace must be 32-byte aligned");
  TrainWs W = train_ws(d);
  if (ws_bytes < W.total) return fail(MKA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, W.total);
  PackLayout PL = pack_layout(d);
  cudaStream_t s = (cudaStream_t)stream;
  const PrefillWs& F = W.fw;
  const size_t T = d.T;
  const int wd = d.width;  // 2 dkv: [dK | dV], [X W_k | X W_v]
  const bf16* wcat = (const bf16*)P((void*)packed, PL.wcat);
  float* lse = (float*)P(ws, W.lse);
  float* dsum = (float*)P(ws, W.dsum);
  float* dq = (float*)P(ws, W.dq);
  float* dy = (float*)P(ws, W.dy);
  float* ema = (float*)P(ws, W.ema);
  float* m3 = (float*)P(ws, W.m3);
  float* hrec = (float*)P(ws, W.hrec);
  float* dlam = dlambda_out ? dlambda_out : (float*)P(ws, W.dlam);
  void* dh = P(ws, W.dh);
  void* acat = P(ws, W.acat);
  const float* lam = (const float*)P(ws, F.lam);
  const int* idx = (const int*)P(ws, F.idx);
  const int* cnt = (const int*)P(ws, F.cnt);

  prof_begin();
  STAGE(s);
  // attention: D = rowsum(dO * O), then dQ and [dK | dV]
  CUDA_TRY(cudaMemsetAsync(dsum, 0, (size_t)d.B * d.Hq * W.Spad * 4, s));
  CUDA_TRY(attention_dsum(dout, out, d.B, d.S, d.Hq, d.dh, W.Spad, dsum, s));
  STAGE(s);
  AttnBwdArgs ab{};
  ab.q = P(ws, F.q); ab.k = P(ws, F.k); ab.v = P(ws, F.v); ab.dout = dout;
  ab.lse = lse; ab.dsum = dsum; ab.lse_ld = W.Spad;
  ab.dq = dq; ab.dkv = dy;
  ab.B = d.B; ab.S = d.S; ab.Hq = d.Hq; ab.Hkv = d.Hkv; ab.dh = d.dh; ab.scale = d.scale;
  CUDA_TRY(attention_backward_tc(ab, status_ptr(), s));
  STAGE(s);
  // the router's pre-activation h = X (W_q W_r1) from its packed hi / lo rows
  {
    Epilogue ep{};
    ep.nseg = 1;
    ep.seg[0] = OutSeg{0, 2 * d.rh, hrec, 2 * d.rh, 0};
    CUDA_TRY(gemm_tn_bf16_tc(x, d.d, wcat + (size_t)PL.seg_r * d.d, d.d, (int)T, 2 * d.rh, d.d, ep, status_ptr(), s));
  }
  STAGE(s);
  // the L2 and L3 values of the projected sources, as the forward fused them
  const float* xkv = (const float*)P(ws, F.xkv);
  CUDA_TRY(ema_apply(xkv, 0, wd, d.B, d.S, d.nblk, d.blk, d.alpha, (const float*)P(ws, F.carry), ema, nullptr, s));
  CUDA_TRY(gather_mean(idx, cnt, d.R, (const float*)P(ws, F.bsum), d.nblk, wd, d.blk, d.B, d.S, m3, s));
  // gate and router MLP
  CUDA_TRY(cudaMemsetAsync(dw_r2, 0, (size_t)d.rh * 3 * sizeof(float), s));
  RouterBwdArgs rb{};
  rb.dy = dy; rb.width = wd; rb.xkv = xkv; rb.ld_xkv = wd; rb.ema = ema; rb.m3 = m3;
  rb.lam = lam; rb.dlam = dlam; rb.hrec = hrec; rb.rh = d.rh; rb.r_inter = PL.router_fused;
  rb.w_r2 = (const float*)P((void*)packed, PL.wr2); rb.dh = dh; rb.dw_r2 = dw_r2;
  rb.B = d.B; rb.S = d.S; rb.route_mode = d.route; rb.tiers = d.tiers;
  CUDA_TRY(router_backward(rb, s));
  STAGE(s);
  // dq = dh W_r1^T + dq (attention, added in the epilogue), into the first dq columns of [dq | U] (bf16);
  // the packed W_r1^T [rh][dq] is the MN-major B
  {
    Epilogue ep{};
    ep.nseg = 1;
    ep.seg[0] = OutSeg{0, d.dq, acat, W.ncat, 1, dq, d.dq};
    CUDA_TRY(gemm_bf16_tc(dh, d.rh, 0, P((void*)packed, PL.wr1T), d.dq, 1, (int)T, d.dq, d.rh, ep, status_ptr(), s));
  }
  STAGE(s);
  // U = lam1 dY + EMA^T(lam2 dY) + M^T(lam3 dY), into the last 2 dkv columns
  {
    int* nrec = (int*)P(ws, W.nrec);
    int* recoff = (int*)P(ws, W.recoff);
    int* list = (int*)P(ws, W.list);
    if (d.nblk > 0)
      CUDA_TRY(block_lists(idx, cnt, d.B, d.S, d.R, d.blk, d.nblk, 0, 0, 32, nrec, recoff, (int*)P(ws, W.cursor),
                           (int*)P(ws, W.pairoff), (int*)P(ws, W.pairbj), list, nullptr, nullptr, s));
    MemAdjArgs ma{};
    ma.dy = dy; ma.width = wd; ma.lam = lam; ma.cnt = cnt; ma.nrec = nrec; ma.recoff = recoff; ma.list = list;
    ma.pairoff = (const int*)P(ws, W.pairoff); ma.pairbj = (const int*)P(ws, W.pairbj);
    ma.B = d.B; ma.S = d.S; ma.nblk = d.nblk; ma.blk = d.blk; ma.alpha = d.alpha;
    ma.gsum = (float*)P(ws, W.gsum); ma.rsum = (float*)P(ws, W.rsum); ma.cs = (float*)P(ws, W.cs);
    ma.u = (bf16*)acat + d.dq; ma.ldu = W.ncat;
    CUDA_TRY(memory_adjoint(ma, s));
  }
  STAGE(s);
  // dX = [dq | U] [W_q | W_k | W_v]^T; the packed rows [W_q | W_k | W_v]^T ([dq + 2 dkv][d]) are the MN-major B
  {
    Epilogue ep{};
    ep.nseg = 1;
    ep.seg[0] = OutSeg{0, d.d, dx, d.d, 1};
    CUDA_TRY(gemm_bf16_tc(acat, W.ncat, 0, wcat, d.d, 1, (int)T, d.d, W.ncat, ep, status_ptr(), s));
  }
  STAGE(s);
  // weight gradients: [dW_q | dW_k | dW_v] = X^T [dq | U], dW_r1 = q^T dh, with the token axis as K:
  // X, [dq | U], q and dh are the MN-major operands as they are stored
  {
    Epilogue ep{};
    ep.nseg = 3;
    ep.seg[0] = OutSeg{0, d.dq, dw_q, d.dq, 0};
    ep.seg[1] = OutSeg{d.dq, d.dq + d.dkv, dw_k, d.dkv, 0};
    ep.seg[2] = OutSeg{d.dq + d.dkv, W.ncat, dw_v, d.dkv, 0};
    CUDA_TRY(gemm_bf16_tc(x, d.d, 1, acat, W.ncat, 1, d.d, W.ncat, (int)T, ep, status_ptr(), s));
  }
  {
    Epilogue ep{};
    ep.nseg = 1;
    ep.seg[0] = OutSeg{0, d.rh, dw_r1, d.rh, 0};
    CUDA_TRY(gemm_bf16_tc(P(ws, F.q), d.dq, 1, dh, d.rh, 1, d.dq, d.rh, (int)T, ep, status_ptr(), s));
  }
  STAGE(s);
  return MKA_OK;
}

int mka_decode_step(const mka_config* cfg, const void* packed, void* state, size_t state_bytes, int32_t max_positions,
                    const void* x_new, void* out, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  int rc = check_cfg(cfg, &d);
  if (rc) return rc;
  if (!packed || !state || !x_new || !out || !ws) return fail(MKA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(packed) || !aligned16(state) || !aligned16(x_new) || !aligned16(out) || !aligned16(ws))
    return fail(MKA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (max_positions < 1) return fail(MKA_ERR_INVALID_ARG, "max_positions must be >= 1");
  if (d.paths == 3 || d.block_sparse)
    return fail(MKA_ERR_UNSUPPORTED, "full MKA and block-sparse attention have no decode step");
  if (d.B > 8) return fail(MKA_ERR_UNSUPPORTED, "decode batch must be <= 8");
  if (d.bf16 && d.Hq / d.Hkv > 16) return fail(MKA_ERR_UNSUPPORTED, "n_q_heads / n_kv_heads must be <= 16 for decode");
  StateLayout SL = state_layout(d, max_positions);
  if (state_bytes < SL.total) return fail(MKA_ERR_WORKSPACE, "state buffer %zu < %zu bytes", state_bytes, SL.total);
  DecodeWs W = decode_ws(d, max_positions);
  if (ws_bytes < W.total) return fail(MKA_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, W.total);
  PackLayout PL = pack_layout(d);
  DecodeArgs a{};
  a.wcatT = P((void*)packed, PL.wcat); a.Ntot = PL.Ntot; a.d = d.d; a.x_bf16 = d.bf16;
  a.w_r2 = (const float*)P((void*)packed, PL.wr2); a.pT64 = (const double*)P((void*)packed, PL.pT64);
  a.dq = d.dq; a.dkv = d.dkv; a.rh = d.rh; a.nb = d.nb; a.rh_segs = PL.rh_segs; a.r_inter = PL.router_fused;
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.dh = d.dh; a.blk = d.blk; a.R = d.R; a.Lmax = max_positions;
  a.maxblk = SL.maxblk; a.alpha = d.alpha; a.scale = d.scale; a.route_mode = d.route; a.tiers = d.tiers;
  a.x_new = x_new; a.out = out;
  a.pos = (int*)P(state, SL.pos); a.kcache = P(state, SL.kc); a.vcache = P(state, SL.vc);
  a.ema = (float*)P(state, SL.ema); a.blk_sum = (float*)P(state, SL.blk_sum); a.blk_x = (double*)P(state, SL.blk_x);
  a.summ = (float*)P(state, SL.summ); a.scode = (uint32_t*)P(state, SL.scode);
  a.y = (float*)P(ws, W.y); a.y2 = (float*)P(ws, W.y2); a.qf = (float*)P(ws, W.qf); a.part = (float*)P(ws, W.part); a.nsplit = W.nsplit;
  a.sync = (unsigned long long*)P(state, SL.sync);
  a.status = status_ptr();
  prof_begin();
  a.prof = g_prof.on ? g_prof.ev : nullptr;
  CUDA_TRY(decode_step(a, (cudaStream_t)stream));
  if (g_prof.on) g_prof.n = 5;
  return MKA_OK;
}

}  // extern "C"
