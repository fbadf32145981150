"""CPU oracle for the FastMKA layer -- TEST INFRASTRUCTURE, not product code.

A plain, slow, float64 NumPy restatement of Route-Fused Memory-Keyed Attention
("MKA: Memory-Keyed Attention for Efficient Long-Context Reasoning"; paper-notes
page sections 1-4 and the abstract page).  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its
``--impl reference`` arm) may import it.  The CUDA path never imports, links or
calls anything here, and nothing here imports the CUDA path.

Pins (see ``tests/test_oracle_pins.py``) tie every function to facts the pages
and mathematics fix: router rows sum to one, the EMA closed form, the
strictly-past recall rule checked by brute force, lambda=(1,0,0) reducing to
textbook causal attention, the online max-shift equalling the two-pass softmax,
causality under future perturbation, decode == prefill rows, and closed forms of
the routing-gate variants (fixed, hard top-1 / top-2, removed tiers).
"""
from .fastmka import (  # noqa: F401
    gelu_erf, softmax_rows, router, router_logits, route_gate, route_margin, ROUTE_MODES, session_ema, block_summaries, hash_codes, hamming,
    recall_select, longterm_recall, fuse_sources, kv_project, causal_gqa_attention,
    online_softmax_attend, fastmka_prefill, fastmka_decode, Weights64, weights_f64,
    recalled_block_attention, mka_full_prefill, block_sparse_gqa_attention,
    EXCUSE_EPS, recall_mismatch_excused, recall_mismatches,
)
from .backward import (  # noqa: F401
    fastmka_backward, causal_gqa_attention_backward, session_ema_backward, longterm_recall_backward,
    route_gate_backward, gelu_erf_grad,
)
