"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol include/mka.h declares, sizes its buffers, and rejects bad arguments on
the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_build_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("mka_build", os.path.join(ROOT, "route_kv_memory_b200", "_build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def mka():
    load_build_module().build_library()
    import route_kv_memory_b200 as m
    return m


def header_functions():
    src = open(os.path.join(ROOT, "include", "mka.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mka_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_five_steps():
    fns = header_functions()
    for name in ("mka_router", "mka_session_ema", "mka_longterm_recall", "mka_prefill_forward", "mka_decode_step"):
        assert name in fns


def test_library_exports_every_declared_symbol(mka):
    lib = ctypes.CDLL(mka.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name
    assert sorted(mka.EXPORTED) == header_functions()


def test_version_and_empty_error(mka):
    assert "sm_100a" in mka.mka_version()


def qwen_cfg(mka, **kw):
    from fastmka_inputs import CONFIGS
    c = mka.make_config(CONFIGS["qwen7b_4k"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_sizes(mka):
    c = qwen_cfg(mka)
    T, dq, dkv = 2 * 4096, 3584, 512
    ws = mka.mka_workspace_size(c)
    assert ws >= T * dq * 2 + T * 2 * dkv * 4 + 2 * T * dkv * 2
    assert mka.mka_packed_weights_size(c) >= 5152 * 3584 * 2
    st = mka.mka_state_size(c, 131072)
    assert st >= 2 * 2 * 131072 * dkv * 2          # K and V caches, 2 sequences
    assert mka.mka_decode_workspace_size(c, 131072) > 0
    assert mka.mka_router_workspace_size(c) > 0
    assert mka.mka_session_ema_workspace_size(c) > 0
    assert mka.mka_longterm_recall_workspace_size(c) > 0


@pytest.mark.parametrize("field,value", [
    ("d_head", 96), ("n_kv_heads", 5), ("hash_bits", 33), ("recall_r", 0), ("router_hidden", 12), ("d_model", 100),
    ("dtype", 7), ("block_size", 0), ("batch", 0), ("route_mode", 4), ("route_mode", -1), ("tiers", 8),
    ("attention_paths", 2), ("attention_paths", 4), ("block_sparse", 2),
])
def test_bad_configs_size_zero(mka, field, value):
    c = qwen_cfg(mka, **{field: value})
    assert mka.mka_workspace_size(c) == 0
    assert mka.mka_packed_weights_size(c) == 0


def test_routing_fields_follow_attn_scale(mka):
    """The routing fields were appended to mka_config; the earlier fields keep their offsets, and a
    zero-initialised tiers field selects all three tiers (the published layer)."""
    fields = [f[0] for f in mka.mka_config._fields_]
    assert fields[-5:] == ["attn_scale", "route_mode", "tiers", "attention_paths", "block_sparse"]
    assert ctypes.sizeof(mka.mka_config) == 17 * 4
    for mode in range(4):
        for tiers in range(8):
            assert mka.mka_workspace_size(qwen_cfg(mka, route_mode=mode, tiers=tiers)) > 0


def test_full_mka_limits(mka):
    """Three attention paths: bf16 prefill with block_size % 128 == 0; no decode state."""
    assert mka.mka_workspace_size(qwen_cfg(mka, attention_paths=3)) > mka.mka_workspace_size(qwen_cfg(mka))
    assert mka.mka_workspace_size(qwen_cfg(mka, attention_paths=3, block_size=64)) == 0
    assert mka.mka_workspace_size(qwen_cfg(mka, attention_paths=3, dtype=mka.MKA_F32)) == 0
    assert mka.mka_workspace_size(qwen_cfg(mka, block_sparse=1)) > 0
    assert mka.mka_workspace_size(qwen_cfg(mka, block_sparse=1, attention_paths=3)) == 0


def test_training_limits(mka):
    """The layer backward: bf16 FastMKA only, router_hidden % 32 == 0 and <= 512."""
    assert mka.mka_train_workspace_size(qwen_cfg(mka)) > mka.mka_workspace_size(qwen_cfg(mka))
    for kw in ({"dtype": mka.MKA_F32}, {"attention_paths": 3}, {"block_sparse": 1}, {"router_hidden": 48},
               {"router_hidden": 1024}):
        assert mka.mka_train_workspace_size(qwen_cfg(mka, **kw)) == 0, kw
    lib, a = mka._lib, ctypes.c_void_p(0x1000)
    c = qwen_cfg(mka, dtype=mka.MKA_F32)
    assert lib.mka_prefill_forward_train(ctypes.byref(c), a, a, a, a, 1 << 40, None) == mka.MKA_ERR_UNSUPPORTED
    c = qwen_cfg(mka)
    assert lib.mka_prefill_forward_train(ctypes.byref(c), a, a, a, ctypes.c_void_p(0x1010), 1 << 40,
                                         None) == mka.MKA_ERR_INVALID_ARG
    assert lib.mka_prefill_backward(ctypes.byref(c), a, a, a, a, a, a, a, a, a, a, None, a, 16,
                                    None) == mka.MKA_ERR_WORKSPACE
    assert lib.mka_prefill_backward(ctypes.byref(c), a, a, a, None, a, a, a, a, a, a, None, a, 1 << 40,
                                    None) == mka.MKA_ERR_INVALID_ARG


def test_host_side_errors_before_any_device_call(mka):
    lib = mka._lib
    c = qwen_cfg(mka)
    assert lib.mka_router(ctypes.byref(c), None, None, None, None, None, 0, None) == mka.MKA_ERR_INVALID_ARG
    assert b"NULL" in lib.mka_last_error()
    bad = qwen_cfg(mka, d_head=96)
    assert lib.mka_prefill_forward(ctypes.byref(bad), None, None, None, None, None, None, 0, 0, None, 0,
                                   None) == mka.MKA_ERR_UNSUPPORTED
    assert b"d_head" in lib.mka_last_error()
    # misaligned pointers are refused on the host
    p = ctypes.c_void_p(0x1001)
    assert lib.mka_session_ema(ctypes.byref(c), p, None, p, None, p, 1 << 30, None) == mka.MKA_ERR_INVALID_ARG
    # workspace too small
    a = ctypes.c_void_p(0x1000)
    assert lib.mka_session_ema(ctypes.byref(c), a, None, a, None, a, 16, None) == mka.MKA_ERR_WORKSPACE
    assert lib.mka_decode_step(ctypes.byref(qwen_cfg(mka, batch=9)), a, a, 1 << 40, 16, a, a, a, 1 << 40,
                               None) == mka.MKA_ERR_UNSUPPORTED
    # the gathered attention (block-sparse, full MKA) writes its partials 32 bytes at a time
    for kw in ({"block_sparse": 1}, {"attention_paths": 3}):
        assert lib.mka_prefill_forward(ctypes.byref(qwen_cfg(mka, **kw)), a, a, a, None, None, None, 0, 0,
                                       ctypes.c_void_p(0x1010), 1 << 40, None) == mka.MKA_ERR_INVALID_ARG
        assert b"32-byte" in lib.mka_last_error()


def test_product_path_has_no_fallback():
    """The binding loads libmka.so or raises; it never imports the oracle."""
    src = open(os.path.join(ROOT, "route_kv_memory_b200", "__init__.py")).read()
    assert "oracle" not in src.replace("no CPU fallback", "")
    assert "raise ImportError" in src


def test_set_wait_limit_rejects_unknown_classes_on_the_host(mka):
    """The testing aid checks its mask before it touches a device."""
    assert mka._lib.mka_set_wait_limit(1000, 4) == mka.MKA_ERR_INVALID_ARG
    assert b"wait_classes" in mka._lib.mka_last_error()
