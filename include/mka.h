/*
 * mka.h -- C ABI of the B200 (sm_100a) FastMKA layer library, libmka.so.
 *
 * Route-Fused Memory-Keyed Attention ("MKA: Memory-Keyed Attention for
 * Efficient Long-Context Reasoning"; "notes" = the paper-notes page, "abstract"
 * = the abstract-and-tables page):
 *   lambda  = softmax(MLP(q))                          notes §2 (routing gate)
 *   L2: M2[t] = a*M2[t-1] + (1-a)*X[t-1], M2[0] = 0     notes §1 (session memory, causal)
 *   L3: R nearest strictly-past block summaries by
 *       sign-projection Hamming distance                notes §1 (long-term memory)
 *   X_fused = l1*X + l2*M2 + l3*M3; K,V = X_fused W_k,v notes §3 (FastMKA)
 *   O = one causal GQA attention over the fused K/V,
 *       online max-shift softmax                        notes §3-§4
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers unless a parameter says "host".  They are
 *     owned by the caller, contiguous, row-major and token-major ([B, S, ...]).
 *     The library never allocates and never frees.
 *   - Weights are [d_in, d_out] (y = x W).  Head-major columns: column h*d_head+i
 *     of q / O is head h, channel i; query head h reads KV group
 *     g(h) = h / (n_q_heads / n_kv_heads).
 *   - `dtype` (MKA_F32 or MKA_BF16) is the element type of X, the weights, q,
 *     K, V and O.  lambda, EMA states, summaries and projections are float32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is asynchronous on it.
 *   - Return value: MKA_OK or a negative mka_status_t for errors found on the
 *     host (arguments, sizes, alignment, launch failures).  Errors found by a
 *     kernel (a bounded wait that ran out, an index out of range, a full decode
 *     cache) are recorded in a device status word read by mka_status().  No
 *     call traps or asserts on the device.  mka_last_error() gives a message.
 *   - Alignment: every pointer must be 16-byte aligned.
 *   - Supported shapes: d_head in {64, 128}; n_q_heads % n_kv_heads == 0;
 *     d_model % 64 == 0; router_hidden % 8 == 0 and <= 1024; 1 <= hash_bits <= 32;
 *     1 <= recall_r <= 64; block_size >= 1; 0 <= ema_alpha <= 1.
 */
#ifndef MKA_H
#define MKA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MKA_API __attribute__((visibility("default")))
#else
#define MKA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MKA_OK = 0,
  MKA_ERR_INVALID_ARG = -1,    /* null / misaligned pointer, bad size or parameter */
  MKA_ERR_UNSUPPORTED = -2,    /* valid FastMKA shape this build does not implement */
  MKA_ERR_CUDA = -3,           /* a CUDA runtime call or a kernel launch failed */
  MKA_ERR_CAPACITY = -4,       /* decode cache full (device status) */
  MKA_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait ran out (device status) */
  MKA_ERR_DEVICE_BOUNDS = -6,  /* a kernel's bounds check failed (device status) */
  MKA_ERR_WORKSPACE = -7       /* workspace / buffer smaller than the size query says */
} mka_status_t;

typedef enum { MKA_F32 = 0, MKA_BF16 = 1 } mka_dtype_t;

/* Routing gate variants (abstract-and-tables page, Table 10).  From the router logits z
 * (notes §2, z = GELU(q W_r1) W_r2) over the active tiers:
 *   SOFT   lambda = softmax(z) (the layer as published);
 *   FIXED  equal weights, 1 / (number of active tiers);
 *   TOP1   all weight on the largest logit (ties to the lower tier index);
 *   TOP2   softmax over the two largest logits, 0 for the third.
 * Inactive tiers always get weight 0. */
typedef enum { MKA_ROUTE_SOFT = 0, MKA_ROUTE_FIXED = 1, MKA_ROUTE_TOP1 = 2, MKA_ROUTE_TOP2 = 3 } mka_route_t;

/* Memory tiers taking part (abstract-and-tables page, Table 9): a bit mask of L1 (the token),
 * L2 (session EMA) and L3 (recalled blocks).  0 selects all three.  With L3 off the prefill
 * skips the L3 codes and recall (recall_idx_out, if given, is filled with -1). */
#define MKA_TIER_L1 1
#define MKA_TIER_L2 2
#define MKA_TIER_L3 4

typedef struct mka_config {
  int32_t batch;         /* B */
  int32_t seq;           /* S: rows per sequence of a prefill call */
  int32_t d_model;       /* d */
  int32_t n_q_heads;     /* Hq */
  int32_t n_kv_heads;    /* Hkv */
  int32_t d_head;        /* dh */
  int32_t router_hidden; /* rh: router MLP d_q -> rh (GELU) -> 3 */
  float ema_alpha;       /* a of the L2 EMA */
  int32_t block_size;    /* b: L3 block length */
  int32_t recall_r;      /* R: blocks recalled per token */
  int32_t hash_bits;     /* nbits of the sign-projection code */
  int32_t dtype;         /* mka_dtype_t */
  float attn_scale;      /* <= 0 selects 1/sqrt(d_head) */
  int32_t route_mode;    /* mka_route_t; MKA_ROUTE_SOFT for the published layer */
  int32_t tiers;         /* MKA_TIER_* mask; 0 = all three */
  int32_t attention_paths; /* 1 (or 0): FastMKA, fused K/V and one attention (notes §3);
                              3: full MKA, three attention outputs mixed by the gate (notes §2):
                              causal over the tokens, the L2 summary value, attention over the
                              recalled L3 blocks' tokens.  3 is implemented for bf16 prefill with
                              block_size a multiple of 128, recall_r <= 16 and no decode state;
                              otherwise MKA_ERR_UNSUPPORTED */
  int32_t block_sparse;  /* 0: one full causal attention (notes §3).  1: Block-MKA's block-sparse
                            attention (notes §4-5): token t attends, in one softmax, to the keys <= t
                            of its own L3 block and to every key of its recalled blocks.  With
                            attention_paths 1 only; bf16 prefill, block_size a multiple of 128,
                            recall_r <= 16, no decode state; otherwise MKA_ERR_UNSUPPORTED */
} mka_config;

/* Raw layer weights, all in cfg->dtype, all [d_in, d_out] row-major. */
typedef struct mka_weights {
  const void* w_q;       /* [d, Hq*dh] */
  const void* w_k;       /* [d, Hkv*dh] */
  const void* w_v;       /* [d, Hkv*dh] */
  const void* w_r1;      /* [Hq*dh, rh] */
  const void* w_r2;      /* [rh, 3] */
  const void* hash_proj; /* [d, nbits]: the L3 sign-random-projection P */
} mka_weights;

/* ------------------------------------------------------------------ sizes */

/* Bytes of the packed-weight buffer that mka_pack_weights fills (0 on a bad cfg). */
MKA_API size_t mka_packed_weights_size(const mka_config* cfg);

/* Bytes of scratch that mka_prefill_forward needs for cfg (0 on a bad cfg). */
MKA_API size_t mka_workspace_size(const mka_config* cfg);

/* Bytes of scratch that mka_router / mka_session_ema / mka_longterm_recall need. */
MKA_API size_t mka_router_workspace_size(const mka_config* cfg);
MKA_API size_t mka_session_ema_workspace_size(const mka_config* cfg);
MKA_API size_t mka_longterm_recall_workspace_size(const mka_config* cfg);

/* Bytes of a decode state holding up to max_positions tokens per sequence, and
 * bytes of the scratch mka_decode_step needs. */
MKA_API size_t mka_state_size(const mka_config* cfg, int32_t max_positions);
MKA_API size_t mka_decode_workspace_size(const mka_config* cfg, int32_t max_positions);

/* ------------------------------------------------------------------ set-up */

/* Pack the raw weights into the layout the fused kernels read: the transposed
 * concatenation [W_q | W_k | W_v | W_q W_r1 | P]^T (for bf16 the folded router
 * matrix W_q W_r1 is stored as a bf16 hi/lo pair so that the router sees q at
 * float32 accuracy), W_r2 in float32, and P^T in float64 for exact sign
 * decisions.  The fold is exact in real arithmetic: (X W_q) W_r1 = X (W_q W_r1)
 * (notes §2 applies the MLP to q = X W_q).  `packed` must hold
 * mka_packed_weights_size(cfg) bytes.  Re-run after the weights change. */
MKA_API int mka_pack_weights(const mka_config* cfg, const mka_weights* w, void* packed, size_t packed_bytes,
                     void* stream);

/* Initialise a decode state (device buffer of mka_state_size bytes): empty cache,
 * M2 = 0, no finished block, position 0. */
MKA_API int mka_state_init(const mka_config* cfg, int32_t max_positions, void* state, size_t state_bytes, void* stream);

/* ------------------------------------------------------------------ the five steps */

/* Routing gate, notes §2: lambda[t] = softmax(GELU(q[t] W_r1) W_r2), one triple per
 * token shared by all heads.  q [B*S, Hq*dh] (dtype), w_r1 [Hq*dh, rh], w_r2 [rh, 3]
 * (dtype) -> lambda [B*S, 3] float32.  No biases; GELU is x*Phi(x) (erf form).
 * ws: mka_router_workspace_size(cfg) bytes. */
MKA_API int mka_router(const mka_config* cfg, const void* q, const void* w_r1, const void* w_r2, float* lambda,
               void* ws, size_t ws_bytes, void* stream);

/* L2 session memory, notes §1: M2[t] = a*M2[t-1] + (1-a)*X[t-1] per sequence, with
 * M2[0] = carry_in (zeros when NULL).  x [B, S, d] (dtype) -> m2 [B, S, d] float32.
 * carry_out (nullable) [B, d] float32 receives M2[S], the state of the next token.
 * ws: mka_session_ema_workspace_size(cfg) bytes. */
MKA_API int mka_session_ema(const mka_config* cfg, const void* x, const float* carry_in, float* m2, float* carry_out,
                    void* ws, size_t ws_bytes, void* stream);

/* L3 long-term memory, notes §1: block j = rows [j*b, (j+1)*b) of a sequence, summary
 * s_j = block mean of X; code(v) = bits [(v P)_k > 0] (bit k = projection k).  Block j
 * is eligible at row t iff (j+1)*b <= t.  For every row, the R eligible blocks with the
 * smallest (Hamming distance, j) are recalled.  Sign decisions are exact: a projection
 * whose float32 value is within the float32 error bound of zero is recomputed in
 * float64.  x [B, S, d], hash_proj [d, nbits] (dtype) ->
 *   idx   [B, S, R] int32, sorted by (distance, j), -1 padded
 *   count [B, S] int32 (nullable) = min(R, floor(t/b))
 *   m3    [B, S, d] float32 (nullable) = mean of the recalled summaries, 0 if none.
 * ws: mka_longterm_recall_workspace_size(cfg) bytes. */
MKA_API int mka_longterm_recall(const mka_config* cfg, const void* x, const void* hash_proj, int32_t* idx, int32_t* count,
                        float* m3, void* ws, size_t ws_bytes, void* stream);

/* The whole layer forward over B sequences of S rows (notes §1-§4):
 * x [B, S, d] (dtype) -> out [B, S, Hq*dh] (dtype, heads concatenated, no output
 * projection).  `packed` comes from mka_pack_weights.  Optional outputs (NULL to
 * skip): lambda_out [B*S, 3] float32, recall_idx_out [B, S, R] int32.  When `state`
 * is not NULL (mka_state_init'ed, max_positions >= S), the fused K/V rows, M2[S],
 * the finished block summaries and the unfinished block's partial sums are left in
 * it and its position is set to S, ready for mka_decode_step.  Everything a decode
 * step reads is rewritten (the codes of blocks not yet finished are zeroed), so a
 * state that was used before can be refilled without mka_state_init.
 * ws: mka_workspace_size(cfg) bytes, 16-byte aligned (32-byte aligned for full MKA and
 * block-sparse attention, whose partial results are written 32 bytes at a time). */
MKA_API int mka_prefill_forward(const mka_config* cfg, const void* packed, const void* x, void* out, float* lambda_out,
                        int32_t* recall_idx_out, void* state, size_t state_bytes, int32_t max_positions,
                        void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- training (layer backward)
 * Gradients of L = sum(dout * out) of the FastMKA prefill forward with respect to x and the trained
 * weights W_q, W_k, W_v, W_r1, W_r2 (notes §1-§4 differentiated step by step).  The L3 recall is a
 * discrete selection and is held fixed (straight-through): gradients reach x through the recalled
 * block means, not through the choice of blocks; the hash projection P is not trained.  The
 * routing gate passes gradient through its softmax (soft: over the active tiers; hard top-2: over
 * its two chosen logits); fixed and hard top-1 weights pass none.
 * Supported: bf16 FastMKA (attention_paths 1, block_sparse 0), router_hidden % 32 == 0 and <= 512;
 * otherwise MKA_ERR_UNSUPPORTED (mka_train_workspace_size returns 0).
 * Workspace: mka_train_workspace_size(cfg) bytes, 32-byte aligned, shared by the two calls below. */
MKA_API size_t mka_train_workspace_size(const mka_config* cfg);
/* The prefill forward (as mka_prefill_forward without optional outputs or state) that also keeps
 * the attention's per-row softmax normaliser and leaves in ws every activation the backward reads.
 * x [B, S, d] bf16 -> out [B, S, Hq*dh] bf16. */
MKA_API int mka_prefill_forward_train(const mka_config* cfg, const void* packed, const void* x, void* out, void* ws,
                                      size_t ws_bytes, void* stream);
/* The layer backward.  Must follow mka_prefill_forward_train of the same cfg, x and packed weights
 * on the same stream with ws untouched in between; out is that call's output.  dout [B, S, Hq*dh]
 * bf16 -> dx [B, S, d] bf16 and float32 dw_q [d, dq], dw_k [d, dkv], dw_v [d, dkv], dw_r1 [dq, rh],
 * dw_r2 [rh, 3] (overwritten, the weights' layouts of mka_weights); dlambda_out [B*S, 3] float32
 * (nullable) <- dL/dlambda.  All device pointers, 16-byte aligned. */
MKA_API int mka_prefill_backward(const mka_config* cfg, const void* packed, const void* x, const void* out,
                                 const void* dout, void* dx, float* dw_q, float* dw_k, float* dw_v, float* dw_r1,
                                 float* dw_r2, float* dlambda_out, void* ws, size_t ws_bytes, void* stream);

/* One decode step for the next token of each sequence (notes §3: the cache holds the
 * fused routed K/V).  x_new [B, d] (dtype) -> out [B, Hq*dh] (dtype).  Runs the
 * router, reads M2 and recalls from the finished blocks, appends the fused K/V row
 * at the current position, attends over cache[0..pos] (split-KV with a max-shift
 * merge), then advances M2, the block sums and the position.  The position lives
 * in device memory, so a sequence of steps can be captured in a CUDA graph.  A
 * step on a full cache records MKA_ERR_CAPACITY in the status word and changes
 * nothing.  ws: mka_decode_workspace_size(cfg, max_positions) bytes.
 * A step whose bounded device-side wait ran out records MKA_ERR_DEVICE_TIMEOUT and
 * may have applied part of its update: the state's position, cache row and memories
 * are then unspecified, and the out row too, and so are the step's grid barrier and
 * completion counts (arrival counts in the state).  Refill the state with
 * mka_prefill_forward (a prefill into a state redefines all of it, the counts
 * included) or mka_state_init before decoding on. */
MKA_API int mka_decode_step(const mka_config* cfg, const void* packed, void* state, size_t state_bytes,
                    int32_t max_positions, const void* x_new, void* out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ without caller scratch */

/* Bytes of the library's built-in scratch used by mka_session_ema_noalloc. */
#define MKA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* mka_session_ema for callers that cannot allocate device memory (no counterpart
 * in the paper; it exists for the library's users).  Some host programs cannot
 * hand the library a scratch buffer: for example a plugin running inside a host
 * application whose memory manager owns every device allocation and does not let
 * plugins call cudaMalloc, or a caller whose device memory is fully reserved up
 * front.  This call computes exactly what mka_session_ema computes, with the same
 * kernels, but takes its scratch from a fixed MKA_NOALLOC_SCRATCH_BYTES (16 MiB)
 * array inside the library's device image, held by every GPU that loads the
 * library until the process exits.  It allocates nothing and frees nothing.
 *   - Limit: shapes whose mka_session_ema_workspace_size(cfg) exceeds 16 MiB
 *     (about B * (2*floor(S/64) + 1) * d * 4 bytes) are rejected with
 *     MKA_ERR_WORKSPACE and a message naming both sizes; use mka_session_ema.
 *   - The first call on a device looks up the array's device address with that
 *     device current (cudaGetSymbolAddress) and caches it; make that first call
 *     before any stream capture.  The cache is kept per device index for the life
 *     of the process: it is not valid after cudaDeviceReset, nor while the calling
 *     thread has a context other than the device's primary context current (the
 *     library's image, and so the array, is then loaded at another address).
 *   - All calls share the one array, and each call overwrites what the previous
 *     one left there before reading it.  Calls that overlap on the GPU (on two
 *     streams or from two host threads) race on it: serialise them.
 * Arguments, layouts and errors are those of mka_session_ema. */
MKA_API int mka_session_ema_noalloc(const mka_config* cfg, const void* x, const float* carry_in, float* m2,
                                    float* carry_out, void* stream);

/* ------------------------------------------------------------------ status */

/* Synchronises the current device and returns the device status word (MKA_OK or one
 * of the device-side codes), then clears it. */
MKA_API int mka_status(void);

/* Message for the last host-side error of the calling thread ("" if none). */
MKA_API const char* mka_last_error(void);

/* Stage timing, for measurement.  While enabled, mka_prefill_forward and
 * mka_decode_step record a CUDA event on their stream before each stage and
 * after the last one.  mka_profile_read waits for the most recent call's last
 * event, writes the device milliseconds of up to max_stages of its stages into
 * the HOST array ms, and returns how many stages that call had.  Stages of a
 * prefill: 0 projection GEMM, 1 router tail, 2 token codes, 3 block sums,
 * 4 block codes, 5 EMA carries, 6 recall, 7 route-fuse, 8 attention
 * (9 decode-state tail when a state is filled).  Stages of a decode step:
 * 0 GEMV, 1 token update, 2 split-KV attention, 3 merge.  Not for use while
 * capturing a CUDA graph.  Returns a negative mka_status_t on error. */
MKA_API int mka_profile_enable(int enable);
MKA_API int mka_profile_read(float* ms, int max_stages);

/* Self-test of the device-side wait limit used by the tcgen05 kernels (not part of the
 * layer; the paper has no counterpart).  Launches one CTA that waits on an mbarrier
 * nothing arrives at, with a limit of limit_us microseconds (1 .. 1e6).  The wait gives
 * up, records MKA_ERR_DEVICE_TIMEOUT in the status word (read it with mka_status) and
 * the kernel returns.  *result (device int) is set to 0, or to 1 if the wait completed. */
MKA_API int mka_selftest_wait_timeout(int limit_us, int* result, void* stream);

/* Wait classes of mka_set_wait_limit. */
#define MKA_WAIT_PIPELINE 1 /* mbarrier waits of the TMA / tensor-core pipelines (GEMM, attention) */
#define MKA_WAIT_GRID 2     /* grid barrier and completion-count waits of the cooperative bf16 decode step */

/* Testing aid (not part of the layer; the paper has no counterpart): replaces the
 * built-in limit (2 s) of every bounded device-side wait of the classes in the mask
 * wait_classes with limit_ns nanoseconds, on the current device, for the kernels
 * launched after the call.  limit_ns = 0 restores the built-in limits.  A short
 * limit makes ordinary waits run out, so a test can drive the production kernels'
 * timeout path: they record MKA_ERR_DEVICE_TIMEOUT, let their copies and MMAs in
 * flight finish (drain waits keep their own limits), free their tensor memory and
 * return, and the context stays usable.  Synchronises the device; call it only
 * while no work of this library is running on it.  MKA_ERR_INVALID_ARG for an
 * unknown bit in wait_classes. */
MKA_API int mka_set_wait_limit(unsigned long long limit_ns, int wait_classes);

/* Library version string. */
MKA_API const char* mka_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MKA_H */
