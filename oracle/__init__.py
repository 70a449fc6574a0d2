"""Slow, plain fp64 CPU oracle for exact softmax attention (test infrastructure).

This package is TEST INFRASTRUCTURE ONLY.  It may be imported by ``tests/``,
by ``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / ``--impl
reference`` legs of ``bench.py``; nothing on the product path imports it,
and it imports nothing from the product package.

Every function computes the plain definition of attention (materialised
score matrix, two-pass softmax, dense products) in float64, one head at a
time, so that a reader can check it against the source pages by eye.  See
``oracle/attention.py`` for the citations.
"""

from .attention import (  # noqa: F401
    allowed_mask,
    block_mask_elements,
    alibi_bias,
    head_scores,
    head_forward,
    head_backward,
    attention_forward,
    attention_backward,
    attention_forward_rows,
    bwd_preprocess,
)
