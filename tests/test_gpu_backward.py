"""GPU parity of the layer backward (mka_prefill_forward_train + mka_prefill_backward) against the
oracle's float64 backward on the same bf16-rounded inputs and output gradient.

The oracle computes its own recall, and the GPU's recalled indices must equal it bit for bit; the
backward then holds that recall fixed (straight-through) on both sides.

Tolerance: relative L2 error <= 2e-2 per gradient tensor.  The GPU differentiates its own bf16
forward (q, K, V, O rounded) with bf16 operands on the tensor cores (P and dS of the attention
backward, the combined query gradient and U before the dX and weight-gradient products, dh);
each rounding is <= 2^-9 relative and about five of them chain on the way to dX, so errors of
0.5-1% are expected, and 2e-2 leaves room without hiding a wrong term (a dropped path or a wrong
scale moves a gradient by far more).
"""
import numpy as np
import pytest
import torch

import oracle
from fastmka_inputs import CONFIGS, FastMKAConfig, make_inputs
from gpu_util import check_out, gpu_weights, lazy_rescales, oracle_weights

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 2e-2
GRADS = ("dX", "dW_q", "dW_k", "dW_v", "dW_r1", "dW_r2", "dlam")


def small(name, **kw):
    base = dict(batch=1, seq=256, d_model=256, n_q_heads=4, n_kv_heads=2, d_head=64, router_hidden=64, alpha=0.9,
                block=32, recall_r=2, hash_bits=16, dtype="bf16", seed=200)
    base.update(kw)
    return FastMKAConfig(name, **base)


def output_gradient(cfg, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(cfg.batch, cfg.seq, cfg.dq, generator=g).to(torch.bfloat16)


def gpu_backward(cfg, inp, dout):
    import route_kv_memory_b200 as mka
    layer = mka.FastMKALayer(cfg, gpu_weights(inp))
    x = inp.x[:, :cfg.seq].contiguous().cuda()
    out = torch.empty(cfg.batch, cfg.seq, cfg.dq, dtype=x.dtype, device="cuda")
    layer.forward_train(x, out)
    f32 = dict(dtype=torch.float32, device="cuda")
    grads = {"dx": torch.empty_like(x), "dw_q": torch.empty(cfg.d_model, cfg.dq, **f32),
             "dw_k": torch.empty(cfg.d_model, cfg.dkv, **f32), "dw_v": torch.empty(cfg.d_model, cfg.dkv, **f32),
             "dw_r1": torch.empty(cfg.dq, cfg.router_hidden, **f32), "dw_r2": torch.empty(cfg.router_hidden, 3, **f32)}
    dlam = torch.empty(cfg.batch * cfg.seq, 3, **f32)
    layer.backward(x, out, dout.cuda(), grads, dlam)
    # the recall the forward used (the plain prefill computes the same one)
    idx = torch.empty(cfg.batch, cfg.seq, cfg.recall_r, dtype=torch.int32, device="cuda")
    out2 = torch.empty_like(out)
    layer.prefill(x, out2, None, idx)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0
    assert torch.equal(out, out2), "the training forward's output differs from the plain forward's"
    g = {"dX": grads["dx"], "dW_q": grads["dw_q"], "dW_k": grads["dw_k"], "dW_v": grads["dw_v"],
         "dW_r1": grads["dw_r1"], "dW_r2": grads["dw_r2"], "dlam": dlam.view(cfg.batch, cfg.seq, 3)}
    return out, {k: v.float().cpu().double().numpy() for k, v in g.items()}, idx.cpu().numpy().astype(np.int64)


def oracle_backward(cfg, inp, dout, idx_gpu):
    """The oracle's forward with its own recall, then its backward; the GPU's recall must be the same."""
    X = inp.x[:, :cfg.seq].float().numpy()
    w = oracle_weights(inp)
    fwd = oracle.fastmka_prefill(X, w, cfg, keep_d_space=True)
    if cfg.tiers & 4:  # with L3 off its weight is 0 and the GPU computes no recall (indices -1)
        mism = np.flatnonzero((idx_gpu != fwd["idx"]).any(-1).reshape(-1))
        assert mism.size == 0, f"{mism.size} tokens recall different blocks on the GPU (first {mism[:8]})"
    return fwd, oracle.fastmka_backward(X, w, cfg, dout.float().numpy().astype(np.float64), fwd)


def check_grads(cfg, seed=7, ramp=None):
    inp = make_inputs(cfg)
    if ramp is not None:  # scale the inputs up along the sequence by 1 -> ramp
        import dataclasses
        r = torch.linspace(1.0, ramp, cfg.seq)
        x = inp.x.float()
        x[:, :cfg.seq] *= r[None, :, None]
        inp = dataclasses.replace(inp, x=x.to(inp.x.dtype))
    dout = output_gradient(cfg, seed)
    out, g, idx = gpu_backward(cfg, inp, dout)
    fwd, ref = oracle_backward(cfg, inp, dout, idx)
    if ramp is not None:  # the forward's reference maximum really moves after a row's first tile
        assert lazy_rescales(fwd["q"][0], fwd["K"][0], 1.0 / np.sqrt(cfg.d_head)) > 200
    if ramp is None:
        check_out(out, fwd["O"], "bf16")
    else:  # outputs of several units: the relative bound only (the absolute one assumes unit scale)
        o = out.float().cpu().double().numpy().reshape(fwd["O"].shape)
        assert np.linalg.norm(o - fwd["O"]) <= 1e-2 * np.linalg.norm(fwd["O"])
    errs = {}
    for k in GRADS:
        a, r = g[k].reshape(ref[k].shape), ref[k]
        errs[k] = float(np.linalg.norm(a - r) / max(np.linalg.norm(r), 1e-30))
    print(cfg.name, " ".join(f"{k} {v:.2e}" for k, v in errs.items()))
    for k, e in errs.items():
        assert e <= GRAD_REL_L2, f"{k}: relative L2 error {e:.3e}"
    return errs


CASES = [
    small("bwd_dh64_split_router"),
    small("bwd_dh128_interleaved_router_ragged", batch=2, seq=300, d_model=512, n_q_heads=4, n_kv_heads=1,
          d_head=128, router_hidden=128, block=64, recall_r=3, hash_bits=32, seed=201),
    small("bwd_gqa7", seq=384, n_q_heads=14, n_kv_heads=2, d_head=128, router_hidden=128, block=128, recall_r=2,
          hash_bits=32, seed=202),
    small("bwd_top2", route_mode="top2", seed=203),
    small("bwd_l1_l2_only", tiers=3, seed=204),
    small("bwd_short_no_blocks", seq=24, block=32, seed=205),
    small("bwd_mha_dh128", seq=320, n_q_heads=2, n_kv_heads=2, d_head=128, router_hidden=128, block=64, seed=206),
    small("bwd_blocks_of_256", batch=2, seq=600, n_q_heads=8, n_kv_heads=2, d_head=64, block=256, recall_r=2,
          seed=207),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_layer_backward(cfg):
    check_grads(cfg)


def test_layer_backward_rescaled_softmax():
    """Inputs scaled up along the sequence (x 1 -> 3): the forward's tiled softmax moves its reference
    maximum (and rescales O) in many row-tiles, so the row normalisers it leaves for the backward must
    account for the moves."""
    check_grads(small("bwd_rescaled", seq=512, d_head=128, router_hidden=128, block=64, seed=208), ramp=3.0)


@pytest.mark.slow
def test_layer_backward_qwen7b_shape_one_sequence():
    """The Qwen layer shape (28/4 heads, d_h 128, d 3584, router 256) on one 1024-token sequence."""
    check_grads(CONFIGS["qwen7b_4k"].replace(batch=1, seq=1024))
