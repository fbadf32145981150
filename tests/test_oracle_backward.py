"""Pins for the oracle's layer backward: central finite differences of the oracle's own forward.

The gradient of L = sum(dO * O) is checked entry by entry against (L(w + e) - L(w - e)) / 2e,
with the recalled blocks held at those of the unperturbed forward (the straight-through
reading).  Each check takes the backward under test, so the mutation test at the bottom can
plant plausible mistakes in copies of its steps and show that a check fails for each.
"""
import math

import numpy as np
import pytest
import scipy.special

from oracle import backward as BW
from oracle import fastmka as O
from fastmka_inputs import FastMKAConfig

EPS = 1e-6
WEIGHTS = ("w_q", "w_k", "w_v", "w_r1", "w_r2")


def tiny_cfg(**kw) -> FastMKAConfig:
    base = FastMKAConfig("bwd-pin", 2, 40, 12, 4, 2, 3, 5, 0.7, 4, 3, 4, "f32", 7)
    return base.replace(**kw)


def tiny_problem(cfg, seed=5):
    rng = np.random.default_rng(seed)
    d, dq, dkv, rh, nb = cfg.d_model, cfg.dq, cfg.dkv, cfg.router_hidden, cfg.hash_bits
    w = O.weights_f64(rng.standard_normal((d, dq)) / math.sqrt(d), rng.standard_normal((d, dkv)) / math.sqrt(d),
                      rng.standard_normal((d, dkv)) / math.sqrt(d), rng.standard_normal((dq, rh)) / math.sqrt(dq),
                      rng.standard_normal((rh, 3)) * 2.0 / math.sqrt(rh), rng.standard_normal((d, nb)))
    X = rng.standard_normal((cfg.batch, cfg.seq, d))
    dO = rng.standard_normal((cfg.batch, cfg.seq, dq))
    return X, w, dO


def loss(X, w, cfg, dO, fixed):
    return float((dO * O.fastmka_prefill(X, w, cfg, recall_fixed=fixed)["O"]).sum())


def check_gradients(backward_fn, cfg, seed=5, per_tensor=6):
    """Analytic gradients from backward_fn against central differences of the forward."""
    X, w, dO = tiny_problem(cfg, seed)
    fwd = O.fastmka_prefill(X, w, cfg, keep_d_space=True)
    fixed = (fwd["idx"], fwd["count"])
    assert fixed[1].max() > 0 or not cfg.tiers & 4, "the problem must recall some blocks"
    g = backward_fn(X, w, cfg, dO, fwd)
    rng = np.random.default_rng(seed + 1)
    # X: rows of the first blocks (recalled, EMA-weighted from far), a middle row and the last row
    rows = [0, 1, cfg.block - 1, cfg.block, cfg.seq // 2, cfg.seq - 1]
    probes = [("dX", None, (int(rng.integers(cfg.batch)), r, int(rng.integers(cfg.d_model)))) for r in rows]
    for name in WEIGHTS:
        shape = getattr(w, name).shape
        probes += [("d" + name[0].upper() + name[1:], name, tuple(int(rng.integers(n)) for n in shape))
                   for _ in range(per_tensor)]
    for gname, wname, ix in probes:
        if wname is None:
            Xp, Xm = X.copy(), X.copy()
            Xp[ix] += EPS
            Xm[ix] -= EPS
            fd = (loss(Xp, w, cfg, dO, fixed) - loss(Xm, w, cfg, dO, fixed)) / (2 * EPS)
        else:
            base = getattr(w, wname)
            vals = []
            for sgn in (1.0, -1.0):
                arr = base.copy()
                arr[ix] += sgn * EPS
                wp = O.Weights64(**{**{k: getattr(w, k) for k in WEIGHTS + ("P",)}, wname: arr})
                vals.append(loss(X, wp, cfg, dO, fixed))
            fd = (vals[0] - vals[1]) / (2 * EPS)
        an = g[gname][ix]
        assert abs(an - fd) <= 1e-6 * (1.0 + abs(fd)), f"{gname}{ix}: analytic {an:.9g} vs difference {fd:.9g}"


@pytest.mark.parametrize("kw", [{}, {"route_mode": "top2"}, {"tiers": 3}, {"tiers": 5}, {"alpha": 0.0},
                                {"n_kv_heads": 4}],
                         ids=["soft", "top2", "L1+L2", "L1+L3", "alpha0", "mha"])
def test_gradients_match_central_differences(kw):
    check_gradients(BW.fastmka_backward, tiny_cfg(**kw))


def test_hard_gates_pass_no_gradient_to_the_router():
    """Fixed and hard top-1 weights are constants of the logits: W_r1, W_r2 get no gradient."""
    for mode in ("fixed", "top1"):
        cfg = tiny_cfg(route_mode=mode)
        X, w, dO = tiny_problem(cfg)
        g = BW.fastmka_backward(X, w, cfg, dO)
        assert not g["dW_r1"].any() and not g["dW_r2"].any()
        check_gradients(BW.fastmka_backward, cfg, per_tensor=3)


def test_attention_backward_is_the_softmax_jacobian():
    """One head, one query row: dq = scale * sum_j p_j (dp_j - sum_k p_k dp_k) K_j, from the
    softmax Jacobian diag(p) - p p^T written out."""
    rng = np.random.default_rng(3)
    S, dh = 6, 4
    q, K, V, dO = (rng.standard_normal((S, 1, dh)) for _ in range(4))
    scale = 0.7
    dq, dK, dV = BW.causal_gqa_attention_backward(q, K, V, dO, 1, scale)
    t = S - 1
    s = scale * K[:, 0] @ q[t, 0]
    p = np.exp(s - s.max())
    p /= p.sum()
    J = np.diag(p) - np.outer(p, p)
    dp = V[:, 0] @ dO[t, 0]
    np.testing.assert_allclose(dq[t, 0], scale * (J @ dp) @ K[:, 0], rtol=1e-12)
    # row 0 sees only key 0: p = 1, so it sends dO[0] to V[0] and nothing to q[0]
    np.testing.assert_allclose(dq[0, 0], 0.0, atol=1e-15)


def test_ema_adjoint_is_the_transpose():
    """session_ema_backward equals the transpose of the EMA written as an explicit S x S matrix."""
    rng = np.random.default_rng(4)
    S, a = 9, 0.6
    M = np.zeros((S, S))
    for t in range(1, S):
        for k in range(t):
            M[t, k] = (1 - a) * a ** (t - 1 - k)
    dM2 = rng.standard_normal((S, 3))
    np.testing.assert_allclose(BW.session_ema_backward(dM2, a), M.T @ dM2, rtol=1e-13)


# ---------------------------------------------------------------------------- planted mistakes
_RECALL_BWD, _GATE_BWD, _ATTN_BWD = BW.longterm_recall_backward, BW.route_gate_backward, BW.causal_gqa_attention_backward


def _mut_ema_current(dM2, alpha):
    S = dM2.shape[0]
    dX = np.zeros_like(dM2)
    c = np.zeros(dM2.shape[1])
    for t in range(S - 1, 0, -1):
        c = dM2[t] + alpha * c
        dX[t] += (1.0 - alpha) * c  # reads X[t] instead of X[t-1]
    return dX


def _mut_recall_no_count(dM3, idx, count, b):
    return _RECALL_BWD(dM3 * np.maximum(count, 1)[:, None], idx, count, b)


def _mut_gelu_grad_phi_only(x):
    return 0.5 * scipy.special.erfc(-x / math.sqrt(2.0))


def _mut_gate_sign(z, lam, dlam, mode="soft", tiers=7):
    return -_GATE_BWD(z, lam, dlam, mode, tiers)


def _mut_attention_no_scale(q, K, V, dO, n_kv_heads, scale):
    dq, dK, dV = _ATTN_BWD(q, K, V, dO, n_kv_heads, scale)
    return dq / scale, dK, dV


def test_planted_backward_mistakes_are_caught(monkeypatch):
    cfg = tiny_cfg()
    for attr, bad in (("session_ema_backward", _mut_ema_current), ("longterm_recall_backward", _mut_recall_no_count),
                      ("gelu_erf_grad", _mut_gelu_grad_phi_only), ("route_gate_backward", _mut_gate_sign),
                      ("causal_gqa_attention_backward", _mut_attention_no_scale)):
        with monkeypatch.context() as m:
            m.setattr(BW, attr, bad)
            with pytest.raises(AssertionError):
                check_gradients(BW.fastmka_backward, cfg)
    check_gradients(BW.fastmka_backward, cfg)  # and the unplanted backward passes
