"""The production kernels' timeout path, driven by a short device-side wait limit.

mka_set_wait_limit (a testing aid) shortens the built-in limit of the bounded
waits, so ordinary waits run out: the kernels must record MKA_ERR_DEVICE_TIMEOUT,
let their copies and MMAs in flight finish, free their tensor memory and return,
leaving the context usable.  Each test then runs the same layer with the built-in
limits and checks it against the oracle.  No wait here is made endless: every
wait ends on its own limit, and no kernel traps.
"""
import numpy as np
import pytest
import torch

from fastmka_inputs import FastMKAConfig, make_inputs
from gpu_util import check_lambda, check_out, check_recall, gpu_weights, oracle_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mka():
    import route_kv_memory_b200 as m
    return m


def _cfg(name, **kw):
    base = dict(batch=2, seq=384, d_model=256, n_q_heads=4, n_kv_heads=2, d_head=128, router_hidden=128, alpha=0.9,
                block=64, recall_r=3, hash_bits=32, dtype="bf16", seed=90)
    base.update(kw)
    return FastMKAConfig(name, **base)


def _run_limited(mka, limit_ns, classes, fn):
    """Runs fn() with the given wait limit, restores the built-in limits, returns the device status."""
    assert mka.mka_status() == 0
    mka.mka_set_wait_limit(limit_ns, classes)
    try:
        fn()
        torch.cuda.synchronize()
        return mka.mka_status()
    finally:
        mka.mka_set_wait_limit(0, 0)


def test_prefill_and_training_waits_run_out_then_the_layer_recovers(mka):
    """The projection GEMM (CTA pairs), the attention and the attention-backward kernels with a
    1 ns pipeline-wait limit: every wait that is not satisfied at once runs out."""
    cfg = _cfg("timeout_prefill")
    inp = make_inputs(cfg)
    layer = mka.FastMKALayer(cfg, gpu_weights(inp))
    x = inp.x.cuda()
    out = torch.empty(cfg.batch, cfg.seq, cfg.dq, dtype=x.dtype, device="cuda")
    layer.prefill(x, out)                    # set-up outside the limited calls
    torch.cuda.synchronize()
    assert mka.mka_status() == 0

    st = _run_limited(mka, 1, mka.MKA_WAIT_PIPELINE, lambda: layer.prefill(x, out))
    assert st == mka.MKA_ERR_DEVICE_TIMEOUT, st

    f32 = dict(dtype=torch.float32, device="cuda")
    grads = {"dx": torch.empty_like(x), "dw_q": torch.empty(cfg.d_model, cfg.dq, **f32),
             "dw_k": torch.empty(cfg.d_model, cfg.dkv, **f32), "dw_v": torch.empty(cfg.d_model, cfg.dkv, **f32),
             "dw_r1": torch.empty(cfg.dq, cfg.router_hidden, **f32), "dw_r2": torch.empty(cfg.router_hidden, 3, **f32)}
    dout = torch.randn(cfg.batch, cfg.seq, cfg.dq, generator=torch.Generator().manual_seed(3)).to(x.dtype).cuda()
    layer.forward_train(x, out)
    layer.backward(x, out, dout, grads)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0

    def train_step():
        layer.forward_train(x, out)
        layer.backward(x, out, dout, grads)
    st = _run_limited(mka, 1, mka.MKA_WAIT_PIPELINE, train_step)
    assert st == mka.MKA_ERR_DEVICE_TIMEOUT, st

    # built-in limits again, same context and layer: the whole layer against the oracle
    lam = torch.empty(cfg.batch * cfg.seq, 3, **f32)
    idx = torch.empty(cfg.batch, cfg.seq, cfg.recall_r, dtype=torch.int32, device="cuda")
    layer.prefill(x, out, lam, idx)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0
    ref = oracle_prefill(cfg, inp)
    check_lambda(lam, ref["lam"])
    check_recall(idx, ref, allow_excused=False)
    check_out(out, ref["O"], "bf16")


def test_decode_grid_barrier_runs_out_then_a_refilled_state_decodes(mka):
    """The cooperative decode step with a 1 ns grid-barrier limit: CTAs that reach a barrier early
    give up and leave, and the barrier's arrival count is left mid-barrier.  The state is then
    refilled by a prefill, without mka_state_init: the refill must reset the barrier too, or the
    next steps would pass their barriers early and decode wrong rows."""
    cfg = _cfg("timeout_decode", seq=1100, n_q_heads=8, block=64, recall_r=4, seed=91)
    inp = make_inputs(cfg)
    ctx, n_new, lmax = 1000, 64, 1200
    layer = mka.FastMKALayer(cfg.replace(seq=ctx), gpu_weights(inp))
    x = inp.x.cuda()
    pre = torch.empty(cfg.batch, ctx, cfg.dq, dtype=x.dtype, device="cuda")
    state = layer.new_state(lmax)
    layer.prefill(x[:, :ctx].contiguous(), pre, state=state, max_positions=lmax)
    o = torch.empty(cfg.batch, cfg.dq, dtype=x.dtype, device="cuda")
    layer.decode(state, lmax, x[:, ctx].contiguous(), o)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0

    for _ in range(2):   # two timed-out steps in a row
        st = _run_limited(mka, 1, mka.MKA_WAIT_GRID, lambda: layer.decode(state, lmax, x[:, ctx].contiguous(), o))
        assert st == mka.MKA_ERR_DEVICE_TIMEOUT, st

    layer.prefill(x[:, :ctx].contiguous(), pre, state=state, max_positions=lmax)
    outs = []
    for t in range(ctx, ctx + n_new):
        ot = torch.empty(cfg.batch, cfg.dq, dtype=x.dtype, device="cuda")
        layer.decode(state, lmax, x[:, t].contiguous(), ot)
        outs.append(ot)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0
    ref = oracle_prefill(cfg.replace(seq=ctx + n_new), inp, rows=np.arange(ctx, ctx + n_new))
    max_abs, rel = check_out(torch.stack(outs, 1), ref["O"], "bf16")
    print(f"decode after two timed-out steps and a refill: rel-L2 {rel:.2e} max-abs {max_abs:.2e}")
