"""Float64 CPU oracle for batched attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs, never by the library. It
shares no code with the CUDA path. See ``paged_ref.py`` for what it computes,
the passages it follows and the readings it takes.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force on tiny inputs, a library special case, closed forms, a hand-worked
golden example and invariants); none is "parity unpinned".
"""
from .paged_ref import (  # noqa: F401
    LN2,
    append_paged_kv,
    attend,
    dequantize_kv,
    e4m3_to_f64,
    gather_pages,
    kv_lengths,
    merge_state,
    merge_states,
    mla_attend,
    mla_paged_attention,
    mla_paged_attention_rows,
    paged_attention,
    paged_attention_quantized_kv,
    paged_attention_rows,
    softmax_rows,
    visible,
)
