"""Seeded synthetic inputs for the FastMKA layer.

This module is shared by the CPU oracle (``oracle/``) and by the CUDA path's
tests and benchmark.  It holds workload shapes and seeded random draws only:
none of the layer's arithmetic lives here.

Workloads (shapes of the Qwen2.5-7B / Llama-3.1-8B attention layers named in
the MKA paper's experimental setup, "MKA: Memory-Keyed Attention for
Efficient Long-Context Reasoning", paper-notes page, section "实验设置"):

* ``tiny_f32``       fp32, batch 1, seq 256, d_model 256, 4 q-heads, 2 kv-heads, d_h 64
* ``qwen7b_4k``      bf16, batch 2, seq 4096, d_model 3584, 28/4 heads, d_h 128
* ``qwen7b_32k``     the same layer at seq 32768
* ``llama8b_128k``   bf16, batch 1, seq 131072, d_model 4096, 32/8 heads, d_h 128
* ``qwen7b_decode``  Qwen-shaped decode: a 131072-position prefix, then 256 new tokens

Draw order (one ``torch.Generator('cpu')`` per workload, seeded):
X ~ N(0,1) [B, S_total, d]; W_q = N(0,1)/sqrt(d) [d, dq]; W_k, W_v = N(0,1)/sqrt(d)
[d, dkv]; W_r1 = N(0,1)/sqrt(dq) [dq, rh]; W_r2 = N(0,1)/sqrt(rh) [rh, 3];
P = N(0,1) [d, nbits] (the hash projection is unscaled).  bf16 workloads round
every drawn tensor to bf16 (round-to-nearest-even) once; both sides consume the
rounded values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class FastMKAConfig:
    name: str
    batch: int
    seq: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    d_head: int
    router_hidden: int
    alpha: float
    block: int
    recall_r: int
    hash_bits: int
    dtype: str  # "f32" or "bf16"
    seed: int
    attn_scale: Optional[float] = None  # None -> 1/sqrt(d_head)
    decode_new: int = 0  # tokens decoded one at a time after a prefix of `seq`
    route_mode: str = "soft"  # routing gate variant: "soft", "fixed", "top1", "top2"
    tiers: int = 7  # active memory tiers: bit 0 L1, bit 1 L2, bit 2 L3
    attention_paths: int = 1  # 1: FastMKA (fused K/V, one attention); 3: full MKA (three attention paths)
    block_sparse: int = 0  # 1: Block-MKA's block-sparse attention (own block + recalled blocks)

    @property
    def dq(self) -> int:
        return self.n_q_heads * self.d_head

    @property
    def dkv(self) -> int:
        return self.n_kv_heads * self.d_head

    @property
    def scale(self) -> float:
        return self.attn_scale if self.attn_scale is not None else 1.0 / math.sqrt(self.d_head)

    @property
    def seq_total(self) -> int:
        return self.seq + self.decode_new

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    def replace(self, **kw) -> "FastMKAConfig":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, FastMKAConfig] = {
    "tiny_f32": FastMKAConfig("tiny_f32", 1, 256, 256, 4, 2, 64, 64, 0.9, 32, 2, 16, "f32", 0),
    "qwen7b_4k": FastMKAConfig("qwen7b_4k", 2, 4096, 3584, 28, 4, 128, 256, 0.99, 128, 8, 32, "bf16", 1),
    "qwen7b_32k": FastMKAConfig("qwen7b_32k", 2, 32768, 3584, 28, 4, 128, 256, 0.99, 128, 8, 32, "bf16", 2),
    "llama8b_128k": FastMKAConfig("llama8b_128k", 1, 131072, 4096, 32, 8, 128, 256, 0.995, 256, 16, 32, "bf16", 3),
    # Decode: 512 summaries at 131072 positions fixes the block at 256 (see the design notes).
    "qwen7b_decode": FastMKAConfig("qwen7b_decode", 1, 131072, 3584, 28, 4, 128, 256, 0.99, 256, 8, 32, "bf16", 4,
                                   decode_new=256),
}


@dataclasses.dataclass
class FastMKAInputs:
    """CPU tensors in the workload dtype (torch.float32 or torch.bfloat16)."""
    x: torch.Tensor      # [B, S_total, d]
    w_q: torch.Tensor    # [d, dq]
    w_k: torch.Tensor    # [d, dkv]
    w_v: torch.Tensor    # [d, dkv]
    w_r1: torch.Tensor   # [dq, rh]
    w_r2: torch.Tensor   # [rh, 3]
    hash_proj: torch.Tensor  # [d, nbits]

    def tensors(self) -> Dict[str, torch.Tensor]:
        return {f.name: getattr(self, f.name) for f in dataclasses.fields(self)}


def torch_dtype(cfg: FastMKAConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def make_inputs(cfg: FastMKAConfig, seq_total: Optional[int] = None) -> FastMKAInputs:
    """Draw the seeded inputs of `cfg` (see the module docstring for the order)."""
    g = torch.Generator("cpu").manual_seed(cfg.seed)
    S = cfg.seq_total if seq_total is None else seq_total
    d, dq, dkv, rh, nb = cfg.d_model, cfg.dq, cfg.dkv, cfg.router_hidden, cfg.hash_bits
    x = torch.randn(cfg.batch, S, d, generator=g, dtype=torch.float32)
    w_q = torch.randn(d, dq, generator=g) / math.sqrt(d)
    w_k = torch.randn(d, dkv, generator=g) / math.sqrt(d)
    w_v = torch.randn(d, dkv, generator=g) / math.sqrt(d)
    w_r1 = torch.randn(dq, rh, generator=g) / math.sqrt(dq)
    w_r2 = torch.randn(rh, 3, generator=g) / math.sqrt(rh)
    p = torch.randn(d, nb, generator=g)
    dt = torch_dtype(cfg)
    return FastMKAInputs(*(t.to(dt).contiguous() for t in (x, w_q, w_k, w_v, w_r1, w_r2, p)))


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (possibly bf16) CPU tensor to a float64 ndarray."""
    return t.detach().to("cpu", torch.float64).numpy()


def sample_rows(S: int, block: int, max_rows: Optional[int] = None) -> np.ndarray:
    """Strided query-row sample for large workloads.

    All rows t < 2b; rows b*k-1, b*k, b*k+1 for every 8th block k; every
    (S/512)-th row; the last row.  `max_rows` thins the result evenly (keeping
    the first and last rows) when a bounded sample is needed.
    """
    rows = set(range(min(S, 2 * block)))
    nblk = S // block
    for k in range(0, nblk + 1, 8):
        for t in (block * k - 1, block * k, block * k + 1):
            if 0 <= t < S:
                rows.add(t)
    stride = max(1, S // 512)
    rows.update(range(0, S, stride))
    rows.add(S - 1)
    out = np.array(sorted(rows), dtype=np.int64)
    if max_rows is not None and len(out) > max_rows:
        pick = np.unique(np.linspace(0, len(out) - 1, max_rows).round().astype(np.int64))
        out = out[pick]
    return out


__all__ = ["FastMKAConfig", "FastMKAInputs", "CONFIGS", "make_inputs", "to_f64", "sample_rows", "torch_dtype"]
