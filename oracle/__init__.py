"""CPU float64 oracle for memory-efficient attention — test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` import this package. It never imports the CUDA package and the CUDA package never
imports it. Pins that tie it to the pages and to mathematics live in ``tests/test_oracle_pins.py``.

Parity unpinned (beyond limits and symmetry checks): the non-causal ALiBi form
``-slope * |p_i - j|`` and bottom-right causal alignment for 1 < L_q != L_k.
"""
from .core import (  # noqa: F401
    alibi_slopes,
    attention,
    attention_backward,
    attention_bruteforce,
    attention_probs,
    attention_rows,
    decode,
    e4m3_decode,
    lse_merge,
    paged_gather,
    segment_positions,
    split_attention_chunks,
)
