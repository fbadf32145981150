"""mka_session_ema_noalloc: the session-memory EMA for callers that cannot allocate device memory.

Some users cannot hand the library a scratch buffer (a plugin inside a host
application that owns every device allocation, or a caller whose device memory is
reserved up front).  For them the library keeps a fixed 16 MiB scratch array in its
own device image.  This test calls that entry point through the C ABI and checks it
against mka_session_ema, which takes a caller buffer, on two calls in a row (the
second call must not depend on what the first left in the shared array).  The file
is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from fastmka_inputs import FastMKAConfig, make_inputs

pytestmark = pytest.mark.gpu

ATOL = 1e-4  # the float32 tolerance of the EMA parity tests


def _cfg(dtype, seq, seed):
    return FastMKAConfig("noalloc", 2, seq, 256, 4, 2, 64, 64, 0.95, 32, 2, 16, dtype, seed)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_matches_caller_scratch_on_two_calls(dtype):
    import route_kv_memory_b200 as mka
    for call, (seq, seed) in enumerate([(300, 71), (517, 72)]):
        cfg = _cfg(dtype, seq, seed)
        inp = make_inputs(cfg)
        c = mka.make_config(cfg)
        x = inp.x.cuda()
        carry_in = torch.randn(cfg.batch, cfg.d_model, generator=torch.Generator().manual_seed(seed)).cuda()
        ref_m2 = torch.empty(cfg.batch, seq, cfg.d_model, device="cuda")
        ref_out = torch.empty(cfg.batch, cfg.d_model, device="cuda")
        ws = mka.buffer(mka.mka_session_ema_workspace_size(c))
        mka.mka_session_ema(c, x, carry_in, ref_m2, ref_out, ws)
        m2 = torch.full_like(ref_m2, float("nan"))
        out = torch.full_like(ref_out, float("nan"))
        rc = mka._lib.mka_session_ema_noalloc(ctypes.byref(c), ctypes.c_void_p(x.data_ptr()),
                                               ctypes.c_void_p(carry_in.data_ptr()), ctypes.c_void_p(m2.data_ptr()),
                                               ctypes.c_void_p(out.data_ptr()),
                                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == mka.MKA_OK, mka._lib.mka_last_error()
        torch.cuda.synchronize()
        assert np.abs((m2 - ref_m2).cpu().numpy()).max() <= ATOL, f"call {call}"
        assert np.abs((out - ref_out).cpu().numpy()).max() <= ATOL, f"call {call}"


@pytest.mark.parametrize("seq,with_carry", [(40, True), (300, False), (40, False)])
def test_noalloc_short_sequences_and_no_carries(seq, with_carry):
    """Sequences shorter than one 64-row chunk (no chunk end states) and calls without carry_in /
    carry_out, against mka_session_ema on the same arguments."""
    import route_kv_memory_b200 as mka
    cfg = _cfg("f32", seq, 80 + seq)
    inp = make_inputs(cfg)
    c = mka.make_config(cfg)
    x = inp.x.cuda()
    cin = torch.randn(cfg.batch, cfg.d_model, generator=torch.Generator().manual_seed(seq)).cuda() if with_carry else None
    ref_m2 = torch.empty(cfg.batch, seq, cfg.d_model, device="cuda")
    ref_out = torch.empty(cfg.batch, cfg.d_model, device="cuda") if with_carry else None
    ws = mka.buffer(mka.mka_session_ema_workspace_size(c))
    mka.mka_session_ema(c, x, cin, ref_m2, ref_out, ws)
    m2 = torch.full_like(ref_m2, float("nan"))
    out = torch.full_like(ref_out, float("nan")) if with_carry else None
    ptr = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    rc = mka._lib.mka_session_ema_noalloc(ctypes.byref(c), ptr(x), ptr(cin), ptr(m2), ptr(out),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == mka.MKA_OK, mka._lib.mka_last_error()
    torch.cuda.synchronize()
    assert np.abs((m2 - ref_m2).cpu().numpy()).max() <= ATOL
    if with_carry:
        assert np.abs((out - ref_out).cpu().numpy()).max() <= ATOL


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import route_kv_memory_b200 as mka
    cfg = FastMKAConfig("big", 4, 65536, 4096, 32, 8, 128, 256, 0.99, 256, 16, 32, "bf16", 0)
    c = mka.make_config(cfg)
    assert mka.mka_session_ema_workspace_size(c) > (16 << 20)
    p = ctypes.c_void_p(256)
    rc = mka._lib.mka_session_ema_noalloc(ctypes.byref(c), p, None, p, None, None)
    assert rc == mka.MKA_ERR_WORKSPACE
    assert b"16777216" in mka._lib.mka_last_error()
