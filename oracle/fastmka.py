"""FastMKA layer, restated step by step in float64 NumPy -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs use this module; the CUDA path shares no code with it.

Sources (both pages are titled "MKA: Memory-Keyed Attention for Efficient
Long-Context Reasoning"; "notes" is the paper-notes page, "abstract" the
abstract-and-tables page):

* notes §1 (三级分层记忆 table): L1 local = the current tokens, L2 session = a
  causal prefix summary M2[t] = Summary(X[:, 1:t, :]) that uses past tokens only,
  L3 long-term = recall of R << T past blocks through a vectorised hash index.
* notes §2 (动态路由门): lambda = softmax(MLP(q)), shape [B, S, 3], per token.
* notes §3 (FastMKA): X_fused = sum_l lambda_l * L_l; K, V = X_fused W_k, X_fused W_v;
  then one standard causal attention over the fused K/V.
* notes §4 (Block-MKA): online max-shift, running max mu, old partial sums
  rescaled by exp(mu_prev - mu_new).
* abstract page: FastMKA is "broadcast-routed" -- lambda is shared by every
  channel and head.

Readings where the pages leave a step open (the workload specification fixes
the parameters): L2 is the EMA M2[t] = a*M2[t-1] + (1-a)*X[t-1], M2[0] = 0;
L3 uses fixed blocks of b rows, summary = block mean of X, hash = signs of an
nbits-wide projection P (bit k set iff (v P)_k > 0, bit k = projection k),
block j is eligible at t iff (j+1)*b <= t, the R nearest by Hamming distance
are recalled with ties going to the lowest block index, and
M3[t] = mean of the recalled summaries (0 when none is eligible).  The router
MLP has no biases and uses the exact-erf GELU.  Query heads map to KV groups
contiguously, g(h) = h // (Hq / Hkv).  There is no positional encoding and no
output projection (the per-head outputs are concatenated).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
from scipy.special import erfc

# Hash bits whose projection lies closer to zero than this may come out either
# way on another machine: a recalled-index mismatch is excused only when the
# other side's list is the recall under some flip of such bits
# (recall_mismatch_excused).
EXCUSE_EPS = 1e-4


# ----------------------------------------------------------------------------- router
def gelu_erf(x: np.ndarray) -> np.ndarray:
    """GELU(x) = x * Phi(x) = 0.5 x (1 + erf(x / sqrt(2))) = 0.5 x erfc(-x / sqrt(2)).

    The erfc form avoids the cancellation of 1 + erf(.) for large negative x.
    """
    return 0.5 * x * erfc(-x / math.sqrt(2.0))


def softmax_rows(z: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (max subtracted first)."""
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def router_logits(q: np.ndarray, w_r1: np.ndarray, w_r2: np.ndarray) -> np.ndarray:
    """Router logits z = MLP(q) = GELU(q W_r1) W_r2 (notes §2).  q: [..., dq] -> z: [..., 3]."""
    h = q @ w_r1
    return gelu_erf(h) @ w_r2


ROUTE_MODES = ("soft", "fixed", "top1", "top2")


def route_gate(z: np.ndarray, mode: str = "soft", tiers: int = 7) -> np.ndarray:
    """Routing weights over the three memory sources from the logits z.

    notes §2: the published gate is lambda = softmax(z).  The abstract page's
    ablations (Table 9: L1+L2 only, L1+L3 only, L1 only; Table 10: fixed 1/3,
    hard top-2, hard top-1 routing) are read with the same logits: a removed
    tier is left out of the gate and gets 0; "fixed" puts equal weight on the
    active tiers; "top1" puts all weight on the largest active logit; "top2"
    takes the softmax over the two largest active logits and 0 elsewhere.  Ties
    go to the lower tier index.  tiers: bit 0 L1, bit 1 L2, bit 2 L3.
    z: [..., 3] -> lambda: [..., 3].
    """
    z = np.asarray(z, np.float64)
    act = np.array([(tiers >> i) & 1 for i in range(3)], bool)
    if not act.any() or mode not in ROUTE_MODES:
        raise ValueError("need at least one tier and a known mode")
    lam = np.zeros(z.shape)
    zz = np.where(act, z, -np.inf)
    if mode == "soft":
        e = np.where(act, np.exp(zz - zz.max(axis=-1, keepdims=True)), 0.0)
        return e / e.sum(axis=-1, keepdims=True)
    if mode == "fixed":
        lam[..., act] = 1.0 / act.sum()
        return lam
    order = np.argsort(-zz, axis=-1, kind="stable")  # largest first, lower index first on ties
    i1 = order[..., :1]
    if mode == "top1" or act.sum() == 1:
        np.put_along_axis(lam, i1, 1.0, axis=-1)
        return lam
    i2 = order[..., 1:2]
    z1, z2 = np.take_along_axis(z, i1, axis=-1), np.take_along_axis(z, i2, axis=-1)
    e = np.exp(z2 - z1)
    np.put_along_axis(lam, i1, 1.0 / (1.0 + e), axis=-1)
    np.put_along_axis(lam, i2, e / (1.0 + e), axis=-1)
    return lam


def route_margin(z: np.ndarray, mode: str = "soft", tiers: int = 7) -> np.ndarray:
    """The logit gap a hard gate decides on: largest minus second largest active
    logit for "top1", second minus third for "top2" (inf where nothing is
    decided, and for the soft and fixed gates).  z: [..., 3] -> [...]."""
    z = np.asarray(z, np.float64)
    act = np.array([(tiers >> i) & 1 for i in range(3)], bool)
    k = {"top1": 1, "top2": 2}.get(mode)
    if k is None or act.sum() <= k:
        return np.full(z.shape[:-1], np.inf)
    zs = -np.sort(-np.where(act, z, -np.inf), axis=-1)
    return zs[..., k - 1] - zs[..., k]


def router(q: np.ndarray, w_r1: np.ndarray, w_r2: np.ndarray, mode: str = "soft", tiers: int = 7) -> np.ndarray:
    """Routing gate lambda = softmax(MLP(q)) over the three memory sources.

    notes §2: one weight per token and source, shared by all heads.  MLP(q) =
    GELU(q W_r1) W_r2.  q: [..., dq] -> lambda: [..., 3].  mode / tiers select
    the ablation gates of route_gate (the defaults give the published gate).
    """
    return route_gate(router_logits(q, w_r1, w_r2), mode, tiers)


# ----------------------------------------------------------------------------- L2
def session_ema(X: np.ndarray, alpha: float, m_init: Optional[np.ndarray] = None):
    """L2 session memory as the causal EMA M2[t] = a*M2[t-1] + (1-a)*X[t-1].

    notes §1: M2[t] summarises X[:, 1:t, :] only (no leakage of token t).
    X: [B, S, d].  M2[0] = m_init (zeros by default).  Returns (M2, m_next) where
    m_next = M2[S], the state a following token would read.
    """
    B, S, d = X.shape
    M2 = np.zeros((B, S, d))
    m = np.zeros((B, d)) if m_init is None else np.array(m_init, dtype=np.float64, copy=True)
    for t in range(S):
        M2[:, t] = m
        m = alpha * m + (1.0 - alpha) * X[:, t]
    return M2, m


# ----------------------------------------------------------------------------- L3
def block_summaries(X: np.ndarray, b: int) -> np.ndarray:
    """Summary of block j = mean of rows [j*b, (j+1)*b) (full blocks only).  X: [B, S, d]."""
    B, S, d = X.shape
    n = S // b
    return X[:, : n * b].reshape(B, n, b, d).mean(axis=2)


def hash_codes(V: np.ndarray, P: np.ndarray):
    """Sign-random-projection code: bit k = [(V P)_k > 0], bit k of a uint32 is projection k.

    Returns (codes uint32 [...], projections float64 [..., nbits]).
    """
    p = V @ P
    nb = P.shape[1]
    bits = (p > 0).astype(np.uint64)
    place = np.left_shift(np.uint64(1), np.arange(nb, dtype=np.uint64))
    codes = (bits * place).sum(axis=-1).astype(np.uint32)
    return codes, p


def hamming(a, b) -> np.ndarray:
    """Number of differing bits."""
    return np.bitwise_count(np.bitwise_xor(np.asarray(a, np.uint32), np.asarray(b, np.uint32))).astype(np.int64)


def recall_select(code_t: int, summary_codes: np.ndarray, n_eligible: int, R: int) -> np.ndarray:
    """Indices of the R nearest eligible blocks, ordered by (Hamming distance, block index)."""
    if n_eligible <= 0:
        return np.zeros(0, dtype=np.int64)
    dist = hamming(code_t, summary_codes[:n_eligible])
    order = np.lexsort((np.arange(n_eligible), dist))  # last key is primary: distance, then index
    return order[:R].astype(np.int64)


def longterm_recall(x_rows: np.ndarray, positions: np.ndarray, summaries: np.ndarray, P: np.ndarray,
                    b: int, R: int):
    """L3 long-term memory for the rows of ONE sequence.

    x_rows [n, d] are the raw tokens at `positions` [n]; summaries [nblk, d] the
    block means of the whole sequence.  Block j is eligible at t iff (j+1)*b <= t.
    Returns (idx [n, R] with -1 padding, count [n], M3 [n, d], x_codes [n], x_proj [n, nb]).
    """
    n, d = x_rows.shape
    s_codes, _ = hash_codes(summaries, P)
    x_codes, x_proj = hash_codes(x_rows, P)
    idx = np.full((n, R), -1, dtype=np.int64)
    count = np.zeros(n, dtype=np.int64)
    M3 = np.zeros((n, d))
    for i, t in enumerate(positions):
        n_elig = min(int(t) // b, len(summaries))
        sel = recall_select(int(x_codes[i]), s_codes, n_elig, R)
        idx[i, : len(sel)] = sel
        count[i] = len(sel)
        if len(sel):
            M3[i] = summaries[sel].mean(axis=0)
    return idx, count, M3, x_codes, x_proj


def recall_mismatch_excused(got, x_proj_t: np.ndarray, s_proj: np.ndarray, n_eligible: int, R: int,
                            eps: float = EXCUSE_EPS, max_token_bits: int = 16) -> bool:
    """Whether the recalled list `got` is the L3 recall of token t once some of the hash bits
    that lie within eps of zero are flipped.

    notes §1 (L3 hash recall) with the sign-code reading: bit k of a code is [p_k > 0].  A bit
    whose projection has |p_k| < eps may come out either way under another summation order, so
    any recall that some such flip produces is as correct as the oracle's.  x_proj_t [nb] is
    token t's projection, s_proj [nblk, nb] the summaries'; `got` the other side's recalled
    indices in order (-1 padding ignored).  Bits further than eps from zero are fixed, so a
    near-zero component that cannot move the selection excuses nothing.

    Exact: the token's near-zero bits are enumerated (at most max_token_bits of them); a
    block's own near-zero bits can move its distance to any value in [d - u, d + v] (u of them
    differ from the token's bit, v agree), and the selection is the first min(R, n_eligible)
    blocks in (distance, index) order, so `got` is reachable iff the greedy choice -- the
    lowest distances for the blocks of `got` in its order, the highest for every other
    eligible block -- keeps that order.
    """
    got = [int(j) for j in got if int(j) >= 0]
    n_eligible = min(int(n_eligible), len(s_proj))
    if len(got) != min(R, n_eligible) or len(set(got)) != len(got) or any(j >= n_eligible for j in got):
        return False
    if not got:
        return True
    nb = len(x_proj_t)
    place = np.left_shift(np.uint64(1), np.arange(nb, dtype=np.uint64))
    sp = np.asarray(s_proj[:n_eligible], np.float64)
    s_bits = (sp > 0)
    s_free = np.abs(sp) < eps                                    # [n_eligible, nb]
    t_bits = np.asarray(x_proj_t, np.float64) > 0
    t_free = np.flatnonzero(np.abs(np.asarray(x_proj_t, np.float64)) < eps)
    if len(t_free) > max_token_bits:
        raise ValueError(f"{len(t_free)} near-zero token bits: too many to enumerate")
    others = np.setdiff1d(np.arange(n_eligible), got)
    for flips in range(1 << len(t_free)):
        tb = t_bits.copy()
        for k_i, k in enumerate(t_free):
            if (flips >> k_i) & 1:
                tb[k] = not tb[k]
        differ = s_bits != tb[None, :]                           # XOR bits
        dist = differ.sum(axis=1)
        lo = dist - (differ & s_free).sum(axis=1)                # flip free bits that differ
        hi = dist + (~differ & s_free).sum(axis=1)               # flip free bits that agree
        ok, prev = True, None
        for j in got:
            dj = int(lo[j]) if prev is None else max(int(lo[j]), prev[0] + (0 if j > prev[1] else 1))
            if dj > hi[j]:
                ok = False
                break
            prev = (dj, j)
        if ok and len(others):
            ok = bool(np.all((hi[others] > prev[0]) | ((hi[others] == prev[0]) & (others > prev[1]))))
        if ok:
            return True
    return False


def recall_mismatches(got_idx: np.ndarray, ref: dict, rows=None):
    """Counts (unexcused, excused) tokens whose recalled list `got_idx` [B, S or len(rows), R]
    differs from the oracle's `ref` (a fastmka_prefill / mka_full_prefill result); a mismatch is
    excused by recall_mismatch_excused only.  Returns the two counts and the unexcused (b, t)."""
    ref_idx = ref["idx"] if rows is None else ref["idx"][:, rows]
    pos = np.arange(ref["idx"].shape[1]) if rows is None else np.asarray(rows)
    got_idx = np.asarray(got_idx).reshape(ref_idx.shape)
    R = ref_idx.shape[-1]
    nblk = ref["summary_proj"].shape[1]
    b = ref["block"]
    unexcused, excused, where = 0, 0, []
    for bi, ti in zip(*np.nonzero((got_idx != ref_idx).any(axis=-1))):
        t = int(pos[ti])
        if recall_mismatch_excused(got_idx[bi, ti], ref["x_proj"][bi, t], ref["summary_proj"][bi],
                                   min(t // b, nblk), R):
            excused += 1
        else:
            unexcused += 1
            where.append((int(bi), t))
    return unexcused, excused, where


# ----------------------------------------------------------------------------- fuse + K/V
def fuse_sources(lam: np.ndarray, L1: np.ndarray, L2: np.ndarray, L3: np.ndarray) -> np.ndarray:
    """notes §3: X_fused = sum_l lambda_l * L_l, lambda broadcast over channels."""
    return lam[..., 0:1] * L1 + lam[..., 1:2] * L2 + lam[..., 2:3] * L3


def kv_project(X_fused: np.ndarray, w_k: np.ndarray, w_v: np.ndarray):
    """notes §3: K = X_fused W_k, V = X_fused W_v."""
    return X_fused @ w_k, X_fused @ w_v


# ----------------------------------------------------------------------------- attention
def causal_gqa_attention(q_rows: np.ndarray, positions: np.ndarray, K: np.ndarray, V: np.ndarray,
                         n_kv_heads: int, scale: float, row_chunk: int = 64) -> np.ndarray:
    """One causal attention over the fused K/V of ONE sequence (notes §3), two-pass softmax.

    O[t, h] = sum_{j <= t} softmax_j(scale * q[t,h] . K[j,g(h)]) V[j,g(h)], g(h) = h // (Hq/Hkv).
    q_rows [n, Hq, dh] at `positions` [n]; K, V [S, Hkv, dh].  Returns [n, Hq, dh].
    """
    n, Hq, dh = q_rows.shape
    G = Hq // n_kv_heads
    out = np.zeros((n, Hq, dh))
    for r0 in range(0, n, row_chunk):
        pos = positions[r0:r0 + row_chunk]
        tmax = int(pos.max()) + 1
        mask = np.arange(tmax)[None, :] > pos[:, None]          # [rows, j]: future keys
        for g in range(n_kv_heads):
            qg = q_rows[r0:r0 + row_chunk, g * G:(g + 1) * G]  # [rows, G, dh]
            s = np.einsum("rhd,jd->rhj", qg, K[:tmax, g]) * scale
            s[np.broadcast_to(mask[:, None, :], s.shape)] = -np.inf
            m = s.max(axis=-1, keepdims=True)                   # pass 1: row maximum
            p = np.exp(s - m)                                   # pass 2: weights
            out[r0:r0 + row_chunk, g * G:(g + 1) * G] = (
                np.einsum("rhj,jd->rhd", p, V[:tmax, g]) / p.sum(axis=-1, keepdims=True))
    return out


def block_sparse_gqa_attention(q_rows: np.ndarray, positions: np.ndarray, K: np.ndarray, V: np.ndarray,
                               idx: np.ndarray, count: np.ndarray, b: int, n_kv_heads: int,
                               scale: float) -> np.ndarray:
    """Block-MKA's block-sparse attention for ONE sequence (notes §4 / §5).

    Query t attends, in one softmax, to the keys j <= t of its own block (j // b == t // b) and
    to every key of the blocks L3 recalled for t (idx[i, :count[i]], all strictly past).
    q_rows [n, Hq, dh] at `positions`; idx [n, R], count [n] for the same rows; K, V [S, Hkv, dh].
    """
    n, Hq, dh = q_rows.shape
    G = Hq // n_kv_heads
    out = np.zeros((n, Hq, dh))
    for i, t in enumerate(positions):
        t = int(t)
        own = np.arange((t // b) * b, t + 1)
        rec = (idx[i, :int(count[i]), None] * b + np.arange(b)[None, :]).reshape(-1)
        keys = np.concatenate([rec, own])
        for h in range(Hq):
            g = h // G
            s = K[keys, g] @ q_rows[i, h] * scale
            p = np.exp(s - s.max())
            out[i, h] = (p @ V[keys, g]) / p.sum()
    return out


def online_softmax_attend(s: np.ndarray, Vt: np.ndarray, tile: int) -> np.ndarray:
    """notes §4: softmax(s) @ Vt with the online max-shift over tiles of `tile` keys.

    Keeps a running maximum mu; on each new tile the old partial sum and output
    are rescaled by exp(mu_prev - mu_new).  s: [n_keys]; Vt: [n_keys, dv].
    """
    mu = -np.inf
    l = 0.0
    o = np.zeros(Vt.shape[1])
    for k0 in range(0, len(s), tile):
        st = s[k0:k0 + tile]
        mu_new = max(mu, float(st.max()))
        corr = math.exp(mu - mu_new) if mu != -np.inf else 0.0
        e = np.exp(st - mu_new)
        l = l * corr + e.sum()
        o = o * corr + e @ Vt[k0:k0 + tile]
        mu = mu_new
    return o / l


# ----------------------------------------------------------------------------- whole layer
@dataclasses.dataclass
class Weights64:
    w_q: np.ndarray
    w_k: np.ndarray
    w_v: np.ndarray
    w_r1: np.ndarray
    w_r2: np.ndarray
    P: np.ndarray


def weights_f64(w_q, w_k, w_v, w_r1, w_r2, P) -> Weights64:
    f = lambda a: np.asarray(a, dtype=np.float64)
    return Weights64(f(w_q), f(w_k), f(w_v), f(w_r1), f(w_r2), f(P))


def fastmka_prefill(X: np.ndarray, w: Weights64, cfg, rows: Optional[np.ndarray] = None,
                    lam_override: Optional[np.ndarray] = None, row_chunk: int = 8192,
                    keep_d_space: bool = False, recall_fixed: Optional[tuple] = None) -> dict:
    """The FastMKA layer forward over whole sequences, in page order.

    X: [B, S, d] (any float dtype; widened to float64 a chunk of rows at a time).
    cfg supplies n_q_heads, n_kv_heads, d_head, alpha, block, recall_r, scale.
    Steps per sequence: q = X W_q; lambda = router(q); M2 = EMA(X); M3 = L3
    recall; X_fused = lambda-weighted sum of (X, M2, M3); K, V projections;
    causal GQA attention on the query rows `rows` (all rows when None); with cfg.block_sparse the
    attention is Block-MKA's block-sparse one (block_sparse_gqa_attention).
    Rows are processed in chunks only to bound memory; the EMA state is carried
    across chunks, so every value is the one the unchunked recurrence gives.
    recall_fixed = (idx [B,S,R], count [B,S]) replaces the hash selection by the given recalled
    blocks (M3 is still their mean): the discrete recall held fixed, as a gradient treats it.
    """
    B, S, d = X.shape
    Hq, Hkv, dh = cfg.n_q_heads, cfg.n_kv_heads, cfg.d_head
    b, R = cfg.block, cfg.recall_r
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    nblk = S // b
    out = {
        "rows": rows,
        "lam": np.zeros((B, S, 3)),
        "idx": np.full((B, S, R), -1, np.int64),
        "count": np.zeros((B, S), np.int64),
        "block": b,
        "x_codes": np.zeros((B, S), np.uint32),
        "x_proj": np.zeros((B, S, w.P.shape[1])),
        "summary_codes": np.zeros((B, nblk), np.uint32),
        "summary_proj": np.zeros((B, nblk, w.P.shape[1])),
        "K": np.zeros((B, S, Hkv, dh)),
        "V": np.zeros((B, S, Hkv, dh)),
        "q": np.zeros((B, len(rows), Hq, dh)),
        "O": np.zeros((B, len(rows), Hq * dh)),
        "m2_next": np.zeros((B, d)),
        "route_margin": np.zeros((B, S)),
    }
    if keep_d_space:
        for k in ("M2", "M3", "X_fused"):
            out[k] = np.zeros((B, S, d))
    for bi in range(B):
        # L3 block summaries need the whole sequence's full blocks.
        summ = np.zeros((nblk, d))
        for j0 in range(0, nblk, max(1, row_chunk // b)):
            j1 = min(nblk, j0 + max(1, row_chunk // b))
            summ[j0:j1] = block_summaries(np.asarray(X[bi:bi + 1, j0 * b:j1 * b], np.float64), b)[0]
        s_codes, s_proj = hash_codes(summ, w.P)
        out["summary_codes"][bi], out["summary_proj"][bi] = s_codes, s_proj
        m2 = np.zeros((1, d))
        for r0 in range(0, S, row_chunk):
            r1 = min(S, r0 + row_chunk)
            xc = np.asarray(X[bi:bi + 1, r0:r1], np.float64)          # [1, n, d]
            qc = xc[0] @ w.w_q                                          # q = X W_q
            mode, tiers = getattr(cfg, "route_mode", "soft"), getattr(cfg, "tiers", 7)
            z = router_logits(qc, w.w_r1, w.w_r2)
            lam = route_gate(z, mode, tiers) if lam_override is None else np.broadcast_to(
                np.asarray(lam_override, np.float64), (r1 - r0, 3))
            out["route_margin"][bi, r0:r1] = route_margin(z, mode, tiers)
            M2, m2 = session_ema(xc, cfg.alpha, m2)
            pos = np.arange(r0, r1)
            idx, cnt, M3, xcodes, xproj = longterm_recall(xc[0], pos, summ, w.P, b, R)
            if not tiers & 4:  # the L3 tier removed: no long-term memory at all (no recall, M3 = 0)
                idx, cnt, M3 = np.full_like(idx, -1), np.zeros_like(cnt), np.zeros_like(M3)
            if recall_fixed is not None:
                idx = np.asarray(recall_fixed[0][bi, r0:r1], np.int64)
                cnt = np.asarray(recall_fixed[1][bi, r0:r1], np.int64)
                M3 = np.array([summ[idx[i, :cnt[i]]].mean(axis=0) if cnt[i] else np.zeros(d)
                               for i in range(r1 - r0)]).reshape(r1 - r0, d)
            Xf = fuse_sources(lam, xc[0], M2[0], M3)
            Kc, Vc = kv_project(Xf, w.w_k, w.w_v)
            out["lam"][bi, r0:r1] = lam
            out["idx"][bi, r0:r1], out["count"][bi, r0:r1] = idx, cnt
            out["x_codes"][bi, r0:r1], out["x_proj"][bi, r0:r1] = xcodes, xproj
            out["K"][bi, r0:r1] = Kc.reshape(-1, Hkv, dh)
            out["V"][bi, r0:r1] = Vc.reshape(-1, Hkv, dh)
            sel = (rows >= r0) & (rows < r1)
            out["q"][bi, sel] = qc[rows[sel] - r0].reshape(-1, Hq, dh)
            if keep_d_space:
                out["M2"][bi, r0:r1], out["M3"][bi, r0:r1], out["X_fused"][bi, r0:r1] = M2[0], M3, Xf
        out["m2_next"][bi] = m2[0]
        if getattr(cfg, "block_sparse", 0):
            # without the L3 tier there is no recall: a token keeps its own block only
            cnt = out["count"][bi, rows] if getattr(cfg, "tiers", 7) & 4 else np.zeros(len(rows), np.int64)
            O = block_sparse_gqa_attention(out["q"][bi], rows, out["K"][bi], out["V"][bi], out["idx"][bi, rows],
                                           cnt, b, Hkv, cfg.scale)
        else:
            O = causal_gqa_attention(out["q"][bi], rows, out["K"][bi], out["V"][bi], Hkv, cfg.scale)
        out["O"][bi] = O.reshape(len(rows), Hq * dh)
    return out


def fastmka_decode(X: np.ndarray, w: Weights64, cfg) -> np.ndarray:
    """Token-at-a-time FastMKA, carrying the decode state.  Returns O [B, S, Hq*dh].

    State per sequence: the fused K/V cache, the EMA value M2 for the next
    token, the running sum of the unfinished block, and the finished block
    summaries with their codes.  Token t reads the state, appends its fused
    K/V, attends over cache[0..t], then advances the EMA and, when it closes a
    block ((t+1) % b == 0), finalises that block's summary and code.  A block is
    therefore visible exactly from t = (j+1)*b on, the strictly-past rule.
    """
    B, S, d = X.shape
    Hq, Hkv, dh = cfg.n_q_heads, cfg.n_kv_heads, cfg.d_head
    b, R = cfg.block, cfg.recall_r
    O = np.zeros((B, S, Hq * dh))
    for bi in range(B):
        Kc = np.zeros((S, Hkv, dh))
        Vc = np.zeros((S, Hkv, dh))
        m2 = np.zeros(d)
        block_sum = np.zeros(d)
        summaries, codes = [], []
        for t in range(S):
            x = np.asarray(X[bi, t], np.float64)
            q = x @ w.w_q
            lam = router(q[None], w.w_r1, w.w_r2, getattr(cfg, "route_mode", "soft"), getattr(cfg, "tiers", 7))[0]
            code_t, _ = hash_codes(x[None], w.P)
            s_arr = np.array(summaries).reshape(-1, d)
            n_rec = len(summaries) if getattr(cfg, "tiers", 7) & 4 else 0  # L3 removed: nothing recalled
            sel = recall_select(int(code_t[0]), np.array(codes, np.uint32), n_rec, R)
            M3 = s_arr[sel].mean(axis=0) if len(sel) else np.zeros(d)
            xf = fuse_sources(lam[None], x[None], m2[None], M3[None])
            k, v = kv_project(xf, w.w_k, w.w_v)
            Kc[t], Vc[t] = k.reshape(Hkv, dh), v.reshape(Hkv, dh)
            o = causal_gqa_attention(q.reshape(1, Hq, dh), np.array([t]), Kc[: t + 1], Vc[: t + 1], Hkv, cfg.scale)
            O[bi, t] = o.reshape(-1)
            m2 = cfg.alpha * m2 + (1.0 - cfg.alpha) * x
            block_sum = block_sum + x
            if (t + 1) % b == 0:
                s_new = block_sum / b
                summaries.append(s_new)
                codes.append(int(hash_codes(s_new[None], w.P)[0][0]))
                block_sum = np.zeros(d)
    return O


# ----------------------------------------------------------------------------- full MKA (three paths)
def recalled_block_attention(q_rows: np.ndarray, idx: np.ndarray, count: np.ndarray, K: np.ndarray,
                             V: np.ndarray, b: int, n_kv_heads: int, scale: float) -> np.ndarray:
    """a_3 of full MKA for ONE sequence: each query row attends to every token of its recalled blocks.

    notes §1 / §2: L3 recalls R past blocks and a_3 = softmax(q k_3^T) v_3 over them.  Read here as
    the keys and values of the recalled blocks' tokens (block j = rows [j*b, (j+1)*b), all strictly
    past, so no mask); 0 where nothing is recalled.  q_rows [n, Hq, dh]; idx [n, R] (-1 padded),
    count [n]; K, V [S, Hkv, dh].  Returns [n, Hq, dh].
    """
    n, Hq, dh = q_rows.shape
    G = Hq // n_kv_heads
    out = np.zeros((n, Hq, dh))
    for i in range(n):
        c = int(count[i])
        if c == 0:
            continue
        tok = (idx[i, :c, None] * b + np.arange(b)[None, :]).reshape(-1)
        for h in range(Hq):
            g = h // G
            s = K[tok, g] @ q_rows[i, h] * scale
            p = np.exp(s - s.max())
            out[i, h] = (p @ V[tok, g]) / p.sum()
    return out


def mka_full_prefill(X: np.ndarray, w: Weights64, cfg, rows: Optional[np.ndarray] = None,
                     lam_override: Optional[np.ndarray] = None) -> dict:
    """Full MKA over whole sequences: three attention outputs mixed by the gate (notes §2).

    O_h = sum_l lambda_l * a_l with a_l = softmax(q_h k_l^T) v_l:
      a_1  causal attention over the tokens themselves, k_1, v_1 = X W_k, X W_v (L1);
      a_2  attention over the L2 session summary of position t, one key, so weight 1 and
           a_2 = M2[t] W_v (M2 the causal EMA, M2[0] = 0);
      a_3  attention over the tokens of the blocks L3 recalls for t (recalled_block_attention).
    lambda is the routing gate (route_gate with cfg's mode and tiers) unless lam_override.
    The abstract page's Table 11 contrasts this three-path form with FastMKA.
    """
    B, S, d = X.shape
    Hq, Hkv, dh = cfg.n_q_heads, cfg.n_kv_heads, cfg.d_head
    b, R = cfg.block, cfg.recall_r
    G = Hq // Hkv
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    nb = w.P.shape[1]
    out = {"rows": rows, "lam": np.zeros((B, S, 3)), "idx": np.zeros((B, S, R), np.int64),
           "count": np.zeros((B, S), np.int64), "block": b, "x_proj": np.zeros((B, S, nb)),
           "summary_proj": np.zeros((B, S // b, nb)),
           "O": np.zeros((B, len(rows), Hq * dh)), "route_margin": np.zeros((B, S))}
    mode, tiers = getattr(cfg, "route_mode", "soft"), getattr(cfg, "tiers", 7)
    for bi in range(B):
        Xb = np.asarray(X[bi], np.float64)
        q = Xb @ w.w_q
        z = router_logits(q, w.w_r1, w.w_r2)
        lam = route_gate(z, mode, tiers) if lam_override is None else np.broadcast_to(
            np.asarray(lam_override, np.float64), (S, 3))
        K1 = (Xb @ w.w_k).reshape(S, Hkv, dh)
        V1 = (Xb @ w.w_v).reshape(S, Hkv, dh)
        M2, _ = session_ema(Xb[None], cfg.alpha)
        V2 = (M2[0] @ w.w_v).reshape(S, Hkv, dh)
        summ = block_summaries(Xb[None], b)[0]
        idx, cnt, _, _, xproj = longterm_recall(Xb, np.arange(S), summ, w.P, b, R)
        if not tiers & 4:  # the L3 tier removed: no recall
            idx, cnt = np.full_like(idx, -1), np.zeros_like(cnt)
        out["x_proj"][bi], out["summary_proj"][bi] = xproj, hash_codes(summ, w.P)[1]
        qr = q[rows].reshape(len(rows), Hq, dh)
        a1 = causal_gqa_attention(qr, rows, K1, V1, Hkv, cfg.scale)
        a2 = V2[rows][:, np.arange(Hq) // G]
        a3 = recalled_block_attention(qr, idx[rows], cnt[rows], K1, V1, b, Hkv, cfg.scale)
        lr = lam[rows]
        O = lr[:, 0, None, None] * a1 + lr[:, 1, None, None] * a2 + lr[:, 2, None, None] * a3
        out["O"][bi] = O.reshape(len(rows), Hq * dh)
        out["lam"][bi], out["idx"][bi], out["count"][bi] = lam, idx, cnt
        out["route_margin"][bi] = route_margin(z, mode, tiers)
    return out
