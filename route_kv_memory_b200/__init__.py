"""Python binding of libmka.so, the B200 FastMKA layer library (see include/mka.h).

Argument marshalling only: every function below passes device pointers, sizes
and the current CUDA stream to the C entry point of the same name, and every
step of the layer runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams.  There is no fallback: if libmka.so is missing or fails to
load, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmka.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python route_kv_memory_b200/_build.py` "
                      "(or __graft_entry__.build()); this package has no CPU fallback")
_lib = ctypes.CDLL(LIB_PATH)

MKA_OK = 0
MKA_ERR_INVALID_ARG = -1
MKA_ERR_UNSUPPORTED = -2
MKA_ERR_CUDA = -3
MKA_ERR_CAPACITY = -4
MKA_ERR_DEVICE_TIMEOUT = -5
MKA_ERR_DEVICE_BOUNDS = -6
MKA_ERR_WORKSPACE = -7
MKA_F32 = 0
MKA_BF16 = 1
# routing gate variants (mka_route_t) and memory tiers (MKA_TIER_*)
ROUTE_MODES = {"soft": 0, "fixed": 1, "top1": 2, "top2": 3}
MKA_TIER_L1, MKA_TIER_L2, MKA_TIER_L3 = 1, 2, 4

EXPORTED = [
    "mka_packed_weights_size", "mka_workspace_size", "mka_router_workspace_size", "mka_session_ema_workspace_size",
    "mka_longterm_recall_workspace_size", "mka_state_size", "mka_decode_workspace_size", "mka_pack_weights",
    "mka_state_init", "mka_router", "mka_session_ema", "mka_longterm_recall", "mka_prefill_forward",
    "mka_decode_step", "mka_status", "mka_last_error", "mka_version", "mka_profile_enable", "mka_profile_read",
    "mka_session_ema_noalloc", "mka_selftest_wait_timeout", "mka_train_workspace_size", "mka_prefill_forward_train",
    "mka_prefill_backward", "mka_set_wait_limit",
]


class mka_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("seq", ctypes.c_int32), ("d_model", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("d_head", ctypes.c_int32),
        ("router_hidden", ctypes.c_int32), ("ema_alpha", ctypes.c_float), ("block_size", ctypes.c_int32),
        ("recall_r", ctypes.c_int32), ("hash_bits", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("attn_scale", ctypes.c_float), ("route_mode", ctypes.c_int32), ("tiers", ctypes.c_int32),
        ("attention_paths", ctypes.c_int32), ("block_sparse", ctypes.c_int32),
    ]


class mka_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_q", "w_k", "w_v", "w_r1", "w_r2", "hash_proj")]


_vp, _sz, _i32, _cfgp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.POINTER(mka_config)
_SIGS = {
    "mka_packed_weights_size": (_sz, [_cfgp]),
    "mka_workspace_size": (_sz, [_cfgp]),
    "mka_router_workspace_size": (_sz, [_cfgp]),
    "mka_session_ema_workspace_size": (_sz, [_cfgp]),
    "mka_longterm_recall_workspace_size": (_sz, [_cfgp]),
    "mka_state_size": (_sz, [_cfgp, _i32]),
    "mka_decode_workspace_size": (_sz, [_cfgp, _i32]),
    "mka_pack_weights": (ctypes.c_int, [_cfgp, ctypes.POINTER(mka_weights), _vp, _sz, _vp]),
    "mka_state_init": (ctypes.c_int, [_cfgp, _i32, _vp, _sz, _vp]),
    "mka_router": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mka_session_ema": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mka_longterm_recall": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mka_prefill_forward": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i32, _vp, _sz, _vp]),
    "mka_decode_step": (ctypes.c_int, [_cfgp, _vp, _vp, _sz, _i32, _vp, _vp, _vp, _sz, _vp]),
    "mka_train_workspace_size": (_sz, [_cfgp]),
    "mka_prefill_forward_train": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mka_prefill_backward": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                            _vp]),
    "mka_status": (ctypes.c_int, []),
    "mka_last_error": (ctypes.c_char_p, []),
    "mka_version": (ctypes.c_char_p, []),
    "mka_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "mka_session_ema_noalloc": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _vp]),
    "mka_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int, _vp, _vp]),
    "mka_set_wait_limit": (ctypes.c_int, [ctypes.c_ulonglong, ctypes.c_int]),
    "mka_profile_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float), ctypes.c_int]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


class MKAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where} failed with status {code}: {_lib.mka_last_error().decode()}")


def _check(code: int, where: str) -> None:
    if code != MKA_OK:
        raise MKAError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("FastMKA tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("FastMKA tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_config(cfg, seq: Optional[int] = None, batch: Optional[int] = None) -> mka_config:
    """mka_config from any object with the FastMKA workload fields (see fastmka_inputs.FastMKAConfig)."""
    return mka_config(
        batch=cfg.batch if batch is None else batch, seq=cfg.seq if seq is None else seq, d_model=cfg.d_model,
        n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads, d_head=cfg.d_head, router_hidden=cfg.router_hidden,
        ema_alpha=cfg.alpha, block_size=cfg.block, recall_r=cfg.recall_r, hash_bits=cfg.hash_bits,
        dtype=MKA_F32 if cfg.dtype == "f32" else MKA_BF16,
        attn_scale=cfg.attn_scale if cfg.attn_scale is not None else 0.0,
        route_mode=ROUTE_MODES[getattr(cfg, "route_mode", "soft")], tiers=getattr(cfg, "tiers", 7),
        attention_paths=getattr(cfg, "attention_paths", 1), block_sparse=getattr(cfg, "block_sparse", 0))


# ------------------------------------------------------------------ sizes
def mka_packed_weights_size(c: mka_config) -> int:
    return _lib.mka_packed_weights_size(ctypes.byref(c))


def mka_workspace_size(c: mka_config) -> int:
    return _lib.mka_workspace_size(ctypes.byref(c))


def mka_router_workspace_size(c: mka_config) -> int:
    return _lib.mka_router_workspace_size(ctypes.byref(c))


def mka_session_ema_workspace_size(c: mka_config) -> int:
    return _lib.mka_session_ema_workspace_size(ctypes.byref(c))


def mka_longterm_recall_workspace_size(c: mka_config) -> int:
    return _lib.mka_longterm_recall_workspace_size(ctypes.byref(c))


def mka_state_size(c: mka_config, max_positions: int) -> int:
    return _lib.mka_state_size(ctypes.byref(c), max_positions)


def mka_decode_workspace_size(c: mka_config, max_positions: int) -> int:
    return _lib.mka_decode_workspace_size(ctypes.byref(c), max_positions)


# ------------------------------------------------------------------ set-up
def mka_pack_weights(c: mka_config, w_q, w_k, w_v, w_r1, w_r2, hash_proj, packed: torch.Tensor, stream=None) -> None:
    w = mka_weights(*(t.data_ptr() for t in (w_q, w_k, w_v, w_r1, w_r2, hash_proj)))
    for t in (w_q, w_k, w_v, w_r1, w_r2, hash_proj):
        _ptr(t)
    _check(_lib.mka_pack_weights(ctypes.byref(c), ctypes.byref(w), _ptr(packed), packed.numel() * packed.element_size(),
                                 _stream(stream)), "mka_pack_weights")


def mka_state_init(c: mka_config, max_positions: int, state: torch.Tensor, stream=None) -> None:
    _check(_lib.mka_state_init(ctypes.byref(c), max_positions, _ptr(state), state.numel() * state.element_size(),
                               _stream(stream)), "mka_state_init")


# ------------------------------------------------------------------ the five steps
def mka_router(c: mka_config, q, w_r1, w_r2, lam, ws, stream=None) -> None:
    _check(_lib.mka_router(ctypes.byref(c), _ptr(q), _ptr(w_r1), _ptr(w_r2), _ptr(lam), _ptr(ws),
                           ws.numel() * ws.element_size(), _stream(stream)), "mka_router")


def mka_session_ema(c: mka_config, x, carry_in, m2, carry_out, ws, stream=None) -> None:
    _check(_lib.mka_session_ema(ctypes.byref(c), _ptr(x), _ptr(carry_in), _ptr(m2), _ptr(carry_out), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "mka_session_ema")


def mka_session_ema_noalloc(c: mka_config, x, carry_in, m2, carry_out, stream=None) -> None:
    """mka_session_ema without a caller scratch buffer (uses the library's fixed 16 MiB device array)."""
    _check(_lib.mka_session_ema_noalloc(ctypes.byref(c), _ptr(x), _ptr(carry_in), _ptr(m2), _ptr(carry_out),
                                        _stream(stream)), "mka_session_ema_noalloc")


def mka_longterm_recall(c: mka_config, x, hash_proj, idx, count, m3, ws, stream=None) -> None:
    _check(_lib.mka_longterm_recall(ctypes.byref(c), _ptr(x), _ptr(hash_proj), _ptr(idx), _ptr(count), _ptr(m3),
                                    _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "mka_longterm_recall")


def mka_prefill_forward(c: mka_config, packed, x, out, lambda_out, recall_idx_out, state, max_positions: int, ws,
                        stream=None) -> None:
    sb = 0 if state is None else state.numel() * state.element_size()
    _check(_lib.mka_prefill_forward(ctypes.byref(c), _ptr(packed), _ptr(x), _ptr(out), _ptr(lambda_out),
                                    _ptr(recall_idx_out), _ptr(state), sb, max_positions, _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)), "mka_prefill_forward")


def mka_train_workspace_size(c: mka_config) -> int:
    return _lib.mka_train_workspace_size(ctypes.byref(c))


def mka_prefill_forward_train(c: mka_config, packed, x, out, ws, stream=None) -> None:
    _check(_lib.mka_prefill_forward_train(ctypes.byref(c), _ptr(packed), _ptr(x), _ptr(out), _ptr(ws),
                                          ws.numel() * ws.element_size(), _stream(stream)), "mka_prefill_forward_train")


def mka_prefill_backward(c: mka_config, packed, x, out, dout, dx, dw_q, dw_k, dw_v, dw_r1, dw_r2, dlambda_out, ws,
                         stream=None) -> None:
    _check(_lib.mka_prefill_backward(ctypes.byref(c), _ptr(packed), _ptr(x), _ptr(out), _ptr(dout), _ptr(dx),
                                     _ptr(dw_q), _ptr(dw_k), _ptr(dw_v), _ptr(dw_r1), _ptr(dw_r2), _ptr(dlambda_out),
                                     _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "mka_prefill_backward")


def mka_decode_step(c: mka_config, packed, state, max_positions: int, x_new, out, ws, stream=None) -> None:
    _check(_lib.mka_decode_step(ctypes.byref(c), _ptr(packed), _ptr(state), state.numel() * state.element_size(),
                                max_positions, _ptr(x_new), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)), "mka_decode_step")


def mka_status() -> int:
    return _lib.mka_status()


def mka_profile_enable(enable: bool) -> None:
    _check(_lib.mka_profile_enable(1 if enable else 0), "mka_profile_enable")


def mka_profile_read(max_stages: int = 16) -> list:
    """Device milliseconds of each stage of the most recent profiled call."""
    buf = (ctypes.c_float * max_stages)()
    n = _lib.mka_profile_read(buf, max_stages)
    if n < 0:
        raise MKAError(n, "mka_profile_read")
    return [buf[i] for i in range(min(n, max_stages))]


def mka_selftest_wait_timeout(limit_us: int, result: torch.Tensor, stream=None) -> None:
    _check(_lib.mka_selftest_wait_timeout(limit_us, _ptr(result), _stream(stream)), "mka_selftest_wait_timeout")


MKA_WAIT_PIPELINE, MKA_WAIT_GRID = 1, 2


def mka_set_wait_limit(limit_ns: int, wait_classes: int) -> None:
    """Testing aid: the limit of the device-side waits of the given classes (0 restores the built-in one)."""
    _check(_lib.mka_set_wait_limit(limit_ns, wait_classes), "mka_set_wait_limit")


def mka_version() -> str:
    return _lib.mka_version().decode()


def buffer(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device byte buffer (torch's caching allocator aligns to at least 512 B)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


class FastMKALayer:
    """Convenience owner of the packed weights and scratch of one layer configuration.

    Allocation happens here (torch device memory); every computation goes through the C ABI.
    """

    def __init__(self, cfg, weights: dict, device="cuda", stream=None):
        self.cfg = cfg
        self.c = make_config(cfg)
        self.device = device
        self.packed = buffer(mka_packed_weights_size(self.c), device)
        mka_pack_weights(self.c, weights["w_q"], weights["w_k"], weights["w_v"], weights["w_r1"], weights["w_r2"],
                         weights["hash_proj"], self.packed, stream)
        self._ws = {}

    def workspace(self, c: mka_config) -> torch.Tensor:
        key = ("prefill", c.batch, c.seq)
        if key not in self._ws:
            self._ws[key] = buffer(mka_workspace_size(c), self.device)
        return self._ws[key]

    def prefill(self, x: torch.Tensor, out: torch.Tensor, lambda_out=None, recall_idx_out=None, state=None,
                max_positions: int = 0, stream=None) -> torch.Tensor:
        c = make_config(self.cfg, seq=x.shape[1], batch=x.shape[0])
        mka_prefill_forward(c, self.packed, x, out, lambda_out, recall_idx_out, state, max_positions,
                            self.workspace(c), stream)
        return out

    def train_workspace(self, c: mka_config) -> torch.Tensor:
        key = ("train", c.batch, c.seq)
        if key not in self._ws:
            self._ws[key] = buffer(mka_train_workspace_size(c), self.device)
        return self._ws[key]

    def forward_train(self, x: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
        """The prefill forward, keeping in this layer's training workspace what backward() reads."""
        c = make_config(self.cfg, seq=x.shape[1], batch=x.shape[0])
        mka_prefill_forward_train(c, self.packed, x, out, self.train_workspace(c), stream)
        return out

    def backward(self, x: torch.Tensor, out: torch.Tensor, dout: torch.Tensor, grads: dict, dlambda_out=None,
                 stream=None) -> dict:
        """Gradients of sum(dout * out) after forward_train(x, out) on the same stream: grads holds
        dx (like x) and float32 dw_q, dw_k, dw_v, dw_r1, dw_r2 in the weights' shapes."""
        c = make_config(self.cfg, seq=x.shape[1], batch=x.shape[0])
        mka_prefill_backward(c, self.packed, x, out, dout, grads["dx"], grads["dw_q"], grads["dw_k"], grads["dw_v"],
                             grads["dw_r1"], grads["dw_r2"], dlambda_out, self.train_workspace(c), stream)
        return grads

    def new_state(self, max_positions: int, batch: Optional[int] = None, stream=None) -> torch.Tensor:
        c = make_config(self.cfg, batch=batch)
        st = buffer(mka_state_size(c, max_positions), self.device)
        mka_state_init(c, max_positions, st, stream)
        return st

    def decode(self, state, max_positions: int, x_new, out, stream=None) -> torch.Tensor:
        c = make_config(self.cfg, seq=1, batch=x_new.shape[0])
        key = ("decode", c.batch, max_positions)
        if key not in self._ws:
            self._ws[key] = buffer(mka_decode_workspace_size(c, max_positions), self.device)
        mka_decode_step(c, self.packed, state, max_positions, x_new, out, self._ws[key], stream)
        return out
