"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs.

Tolerances (stated once, used by every parity test):
  lambda          max relative error <= 1e-3
  recall indices  bit-exact; a mismatch is excused only where the GPU's list is
                  the recall under a flip of hash bits with |p| < 1e-4 (counted, reported)
  float32 outputs max-abs error <= 1e-4
  bf16 outputs    relative L2 error <= 1e-2 and max-abs error <= 3e-2
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from fastmka_inputs import FastMKAConfig, FastMKAInputs, make_inputs, to_f64

LAMBDA_RTOL = 1e-3
F32_ATOL = 1e-4
BF16_REL_L2 = 1e-2
BF16_ATOL = 3e-2


def oracle_weights(inp: FastMKAInputs):
    return oracle.weights_f64(*(to_f64(t) for t in (inp.w_q, inp.w_k, inp.w_v, inp.w_r1, inp.w_r2, inp.hash_proj)))


def oracle_prefill(cfg: FastMKAConfig, inp: FastMKAInputs, rows=None, seq=None):
    S = cfg.seq if seq is None else seq
    X = inp.x[:, :S].float().numpy()
    if getattr(cfg, "attention_paths", 1) == 3:
        return oracle.mka_full_prefill(X, oracle_weights(inp), cfg.replace(seq=S), rows=rows)
    return oracle.fastmka_prefill(X, oracle_weights(inp), cfg.replace(seq=S), rows=rows)


def gpu_weights(inp: FastMKAInputs, device="cuda"):
    return {k: v.to(device) for k, v in inp.tensors().items() if k != "x"}


def gpu_prefill(cfg: FastMKAConfig, inp: FastMKAInputs, seq=None, with_state=0, device="cuda"):
    """Runs mka_prefill_forward; returns (O, lambda, idx, layer, state)."""
    import route_kv_memory_b200 as mka
    S = cfg.seq if seq is None else seq
    c = cfg.replace(seq=S)
    layer = mka.FastMKALayer(c, gpu_weights(inp, device), device)
    x = inp.x[:, :S].contiguous().to(device)
    out = torch.empty(cfg.batch, S, cfg.dq, dtype=x.dtype, device=device)
    lam = torch.empty(cfg.batch * S, 3, dtype=torch.float32, device=device)
    idx = torch.empty(cfg.batch, S, cfg.recall_r, dtype=torch.int32, device=device)
    state = layer.new_state(with_state) if with_state else None
    layer.prefill(x, out, lam, idx, state, with_state)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0
    return out, lam, idx, layer, state


def check_lambda(lam_gpu: torch.Tensor, lam_ref: np.ndarray):
    """Relative error of every nonzero weight; a weight the gate sets to 0 (a removed tier, a hard
    gate's unchosen source) must be exactly 0 on the GPU too."""
    g = lam_gpu.detach().cpu().double().numpy().reshape(lam_ref.shape)
    zero = lam_ref == 0
    assert (g[zero] == 0).all(), "a weight the gate sets to 0 is nonzero on the GPU"
    rel = np.abs(g - lam_ref)[~zero] / np.abs(lam_ref)[~zero]
    rmax = float(rel.max()) if rel.size else 0.0
    assert rmax <= LAMBDA_RTOL, f"lambda max rel err {rmax:.3e}"
    return rmax


def check_recall(idx_gpu: torch.Tensor, out_ref: dict, rows=None, allow_excused: bool = True):
    """Bit-exact recalled indices.  A mismatching token is excused only when the GPU's list is the
    recall under some flip of hash bits whose projection lies within 1e-4 of zero
    (oracle.recall_mismatch_excused).  Returns (unexcused, excused) mismatching tokens; with
    allow_excused=False excused ones fail too (the GPU decides every sign exactly)."""
    g = idx_gpu.detach().cpu().numpy().astype(np.int64)
    if rows is not None:
        g = g.reshape(out_ref["idx"].shape)[:, rows]
    unexcused, excused, where = oracle.recall_mismatches(g, out_ref, rows)
    assert unexcused == 0, f"{unexcused} tokens recall different blocks (excused: {excused}); first {where[:8]}"
    assert allow_excused or excused == 0, f"{excused} excused recall mismatches"
    return unexcused, excused


def out_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    diff = o_gpu - o_ref
    max_abs = float(np.abs(diff).max())
    rel_l2 = float(np.linalg.norm(diff) / np.linalg.norm(o_ref))
    return max_abs, rel_l2


def check_out(o_gpu: torch.Tensor, o_ref: np.ndarray, dtype: str, rows=None):
    g = o_gpu.detach().float().cpu().double().numpy()
    if rows is not None:
        g = g[:, rows]
    g = g.reshape(o_ref.shape)
    max_abs, rel_l2 = out_errors(g, o_ref)
    if dtype == "f32":
        assert max_abs <= F32_ATOL, f"f32 max-abs {max_abs:.3e}"
    else:
        assert rel_l2 <= BF16_REL_L2 and max_abs <= BF16_ATOL, f"bf16 rel-L2 {rel_l2:.3e} max-abs {max_abs:.3e}"
    return max_abs, rel_l2


def bf16_round(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def lazy_rescales(q: np.ndarray, K: np.ndarray, scale: float, tile: int = 128, threshold: float = 8.0) -> int:
    """Row-tiles of one sequence at which a tiled online softmax that moves its reference maximum only when
    it is exceeded by more than 2^threshold (log2 units) moves it after the row's first tile.  Counted from
    the oracle's q [S, Hq, dh] and K [S, Hkv, dh]."""
    S, Hq, dh = q.shape
    G = Hq // K.shape[1]
    c = scale * 1.4426950408889634
    n = 0
    for h in range(Hq):
        s = (q[:, h] @ K[:, h // G].T) * c
        for t in range(S):
            m = -np.inf
            for j in range(t // tile + 1):
                mx = s[t, j * tile:min(t + 1, (j + 1) * tile)].max()
                if mx > m + threshold:
                    n += m != -np.inf
                    m = mx
    return n
