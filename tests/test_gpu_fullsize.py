"""Parity at the full workload sizes, in the launch configuration bench.py times.

lambda and the recalled block indices are compared on every row; the layer
output on a strided row sample (the oracle computes the linear parts for all
rows, the attention only for the sampled rows).  The oracle takes a minute or
so per workload on the host cores.
"""
import numpy as np
import pytest
import torch

from fastmka_inputs import CONFIGS, make_inputs, sample_rows
from gpu_util import check_lambda, check_out, check_recall, gpu_prefill, gpu_weights, oracle_prefill

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("name,max_rows", [("qwen7b_32k", 96), ("llama8b_128k", 64)])
def test_prefill_full_size(name, max_rows):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg)
    rows = sample_rows(cfg.seq, cfg.block, max_rows=max_rows)
    out, lam, idx, *_ = gpu_prefill(cfg, inp)
    out_h, lam_h, idx_h = out.cpu(), lam.cpu(), idx.cpu()
    del out, lam, idx
    torch.cuda.empty_cache()
    ref = oracle_prefill(cfg, inp, rows=rows)
    lam_err = check_lambda(lam_h, ref["lam"])
    # the GPU decides every hash sign exactly (fp64 where the fp32 value is in doubt): no
    # mismatch at all, excused or not
    _, excused = check_recall(idx_h, ref, allow_excused=False)
    max_abs, rel = check_out(out_h, ref["O"], cfg.dtype, rows=rows)
    print(f"{name}: lambda rel {lam_err:.2e}, recall excused {excused}, O rel-L2 {rel:.2e} max-abs {max_abs:.2e}")


@pytest.mark.parametrize("ctx", [4096, 32768, 131072, 262144])
def test_decode_full_context(ctx):
    """Qwen decode: prefill `ctx` rows into a state, decode 256 tokens; check a sample of them."""
    import route_kv_memory_b200 as mka
    base = CONFIGS["qwen7b_decode"]
    n_new = base.decode_new
    cfg = base.replace(seq=ctx + n_new, decode_new=0)
    inp = make_inputs(cfg)
    lmax = ctx + n_new
    layer = mka.FastMKALayer(cfg.replace(seq=ctx), gpu_weights(inp))
    x = inp.x.cuda()
    pre = torch.empty(1, ctx, cfg.dq, dtype=x.dtype, device="cuda")
    state = layer.new_state(lmax)
    layer.prefill(x[:, :ctx].contiguous(), pre, state=state, max_positions=lmax)
    outs = []
    for t in range(ctx, ctx + n_new):
        o = torch.empty(1, cfg.dq, dtype=x.dtype, device="cuda")
        layer.decode(state, lmax, x[:, t].contiguous(), o)
        outs.append(o)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0
    got = torch.stack(outs, 1).cpu()
    del pre, state, x, outs
    torch.cuda.empty_cache()
    pick = np.unique(np.linspace(0, n_new - 1, 12).round().astype(np.int64))
    ref = oracle_prefill(cfg, inp, rows=ctx + pick)
    max_abs, rel = check_out(got[:, pick], ref["O"], "bf16")
    print(f"decode ctx {ctx}: rel-L2 {rel:.2e} max-abs {max_abs:.2e}")
