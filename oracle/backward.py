"""FastMKA layer backward, restated step by step in float64 NumPy -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` use this module; the CUDA path
shares no code with it.

The pages give the forward only (paper-notes page §1-§4; the abstract page reports training
throughput, Table 2).  The gradients here are those of the scalar L = sum(dO * O) with respect
to X and the trained weights W_q, W_k, W_v, W_r1, W_r2, taken through the forward of
``fastmka_prefill`` in its own order, with two readings:

* the L3 recall is a discrete selection (hash signs, Hamming ranks): it is held fixed, so the
  gradient reaches X through the recalled block means M3 but not through the choice of blocks
  (straight-through); the hash projection P is not trained;
* the routing gate is differentiated as written for each mode: the soft gate through its
  softmax over the active tiers, hard top-2 through the softmax of its two chosen logits, and
  the fixed and hard top-1 gates not at all (their weights are constants of the logits almost
  everywhere).

Step by step (per sequence), with Xf = lam1 X + lam2 M2 + lam3 M3, K = Xf W_k, V = Xf W_v:
  attention: P = softmax(scale q K^T) (causal), dV = P^T dO, dP = dO V^T,
             dS = P * (dP - rowsum(dP * P)), dq = scale dS K, dK = scale dS^T q (GQA: summed
             over the query heads of a KV group);
  fuse:      dXf = dK W_k^T + dV W_v^T, dW_k = Xf^T dK, dW_v = Xf^T dV,
             dlam_l = <dXf, source_l> per token, dX += lam1 dXf;
  L2:        M2[t] = a M2[t-1] + (1-a) X[t-1]  =>  dX[t-1] += (1-a) c[t], c[t] = lam2 dXf[t] + a c[t+1];
  L3:        M3[t] = mean_r s_{idx[t,r]}, s_j = mean of block j  =>  each recalled block j gets
             lam3 dXf[t] / count[t], spread as 1/b over the rows of block j;
  router:    z = GELU(h) W_r2, h = q W_r1: dz from the gate, dW_r2 = GELU(h)^T dz,
             dh = (dz W_r2^T) * GELU'(h), GELU'(x) = Phi(x) + x phi(x), dW_r1 = q^T dh,
             dq += dh W_r1^T;
  query:     dW_q = X^T dq, dX += dq W_q^T.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erfc

from .fastmka import Weights64, fastmka_prefill, gelu_erf, router_logits


def gelu_erf_grad(x: np.ndarray) -> np.ndarray:
    """d/dx of x * Phi(x): Phi(x) + x * phi(x)."""
    return 0.5 * erfc(-x / math.sqrt(2.0)) + x * np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def route_gate_backward(z: np.ndarray, lam: np.ndarray, dlam: np.ndarray, mode: str = "soft",
                        tiers: int = 7) -> np.ndarray:
    """dL/dz from dL/dlam for the gate of route_gate.  z, lam, dlam: [n, 3] -> dz [n, 3].

    Where lam is a softmax over a set A of logits (the active tiers for "soft", the two chosen
    ones for "top2"): dz_i = lam_i (dlam_i - sum_{k in A} lam_k dlam_k) for i in A, 0 elsewhere.
    """
    z = np.asarray(z, np.float64)
    n = z.shape[0]
    act = np.array([(tiers >> i) & 1 for i in range(3)], bool)
    dz = np.zeros((n, 3))
    if mode in ("fixed", "top1") or (mode == "top2" and act.sum() == 1):
        return dz
    if mode == "soft":
        member = np.broadcast_to(act, (n, 3))
    else:  # top2: the two largest active logits, lower index first on ties
        zz = np.where(act, z, -np.inf)
        order = np.argsort(-zz, axis=-1, kind="stable")[:, :2]
        member = np.zeros((n, 3), bool)
        np.put_along_axis(member, order, True, axis=-1)
    inner = (np.where(member, lam * dlam, 0.0)).sum(axis=-1, keepdims=True)
    return np.where(member, lam * (dlam - inner), 0.0)


def causal_gqa_attention_backward(q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray,
                                  n_kv_heads: int, scale: float):
    """Backward of causal_gqa_attention for ONE sequence with dense score matrices.

    q, dO: [S, Hq, dh]; K, V: [S, Hkv, dh].  Returns dq [S, Hq, dh], dK, dV [S, Hkv, dh].
    """
    S, Hq, dh = q.shape
    G = Hq // n_kv_heads
    future = np.arange(S)[None, :] > np.arange(S)[:, None]
    dq = np.zeros_like(q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for h in range(Hq):
        g = h // G
        s = scale * (q[:, h] @ K[:, g].T)
        s[future] = -np.inf
        p = np.exp(s - s.max(axis=-1, keepdims=True))
        p /= p.sum(axis=-1, keepdims=True)
        dV[:, g] += p.T @ dO[:, h]
        dp = dO[:, h] @ V[:, g].T
        ds = p * (dp - (dp * p).sum(axis=-1, keepdims=True))
        dq[:, h] = scale * (ds @ K[:, g])
        dK[:, g] += scale * (ds.T @ q[:, h])
    return dq, dK, dV


def session_ema_backward(dM2: np.ndarray, alpha: float) -> np.ndarray:
    """dL/dX from dL/dM2 for M2[t] = a M2[t-1] + (1-a) X[t-1], M2[0] = 0 (one sequence, [S, d])."""
    S = dM2.shape[0]
    dX = np.zeros_like(dM2)
    c = np.zeros(dM2.shape[1])
    for t in range(S - 1, 0, -1):
        c = dM2[t] + alpha * c
        dX[t - 1] += (1.0 - alpha) * c
    return dX


def longterm_recall_backward(dM3: np.ndarray, idx: np.ndarray, count: np.ndarray, b: int) -> np.ndarray:
    """dL/dX from dL/dM3 with the recalled blocks held fixed (one sequence, [S, d])."""
    S, d = dM3.shape
    dX = np.zeros_like(dM3)
    for t in range(S):
        c = int(count[t])
        for j in idx[t, :c]:
            dX[j * b:(j + 1) * b] += dM3[t] / (c * b)
    return dX


def fastmka_backward(X: np.ndarray, w: Weights64, cfg, dO: np.ndarray, fwd: dict | None = None) -> dict:
    """Gradients of sum(dO * O) for the FastMKA layer (cfg.attention_paths 1, full causal attention).

    X: [B, S, d]; dO: [B, S, Hq*dh].  fwd: fastmka_prefill(..., keep_d_space=True) of the same
    inputs (computed when None).  Returns dX [B,S,d], dW_q, dW_k, dW_v, dW_r1, dW_r2 (weight
    shapes) and, per token, dlam [B,S,3] and dq [B,S,Hq*dh] (the query gradient with the
    router's share).
    """
    B, S, d = X.shape
    Hq, Hkv, dh = cfg.n_q_heads, cfg.n_kv_heads, cfg.d_head
    mode, tiers = getattr(cfg, "route_mode", "soft"), getattr(cfg, "tiers", 7)
    if fwd is None:
        fwd = fastmka_prefill(X, w, cfg, keep_d_space=True)
    dO = np.asarray(dO, np.float64).reshape(B, S, Hq, dh)
    res = {k: np.zeros_like(v) for k, v in (("dW_q", w.w_q), ("dW_k", w.w_k), ("dW_v", w.w_v),
                                             ("dW_r1", w.w_r1), ("dW_r2", w.w_r2))}
    res["dX"] = np.zeros((B, S, d))
    res["dlam"] = np.zeros((B, S, 3))
    res["dq"] = np.zeros((B, S, Hq * dh))
    for bi in range(B):
        x = np.asarray(X[bi], np.float64)
        q = fwd["q"][bi]
        lam = fwd["lam"][bi]
        dq, dK, dV = causal_gqa_attention_backward(q, fwd["K"][bi], fwd["V"][bi], dO[bi], Hkv, cfg.scale)
        dK, dV = dK.reshape(S, Hkv * dh), dV.reshape(S, Hkv * dh)
        Xf = fwd["X_fused"][bi]
        dXf = dK @ w.w_k.T + dV @ w.w_v.T
        res["dW_k"] += Xf.T @ dK
        res["dW_v"] += Xf.T @ dV
        dlam = np.stack([(dXf * x).sum(-1), (dXf * fwd["M2"][bi]).sum(-1), (dXf * fwd["M3"][bi]).sum(-1)], -1)
        dx = lam[:, 0:1] * dXf
        dx += session_ema_backward(lam[:, 1:2] * dXf, cfg.alpha)
        dx += longterm_recall_backward(lam[:, 2:3] * dXf, fwd["idx"][bi], fwd["count"][bi], cfg.block)
        qf = q.reshape(S, Hq * dh)
        h = qf @ w.w_r1
        z = router_logits(qf, w.w_r1, w.w_r2)
        dz = route_gate_backward(z, lam, dlam, mode, tiers)
        res["dW_r2"] += gelu_erf(h).T @ dz
        dh_ = (dz @ w.w_r2.T) * gelu_erf_grad(h)
        res["dW_r1"] += qf.T @ dh_
        dqf = dq.reshape(S, Hq * dh) + dh_ @ w.w_r1.T
        res["dW_q"] += x.T @ dqf
        dx += dqf @ w.w_q.T
        res["dX"][bi] = dx
        res["dlam"][bi] = dlam
        res["dq"][bi] = dqf
    return res
