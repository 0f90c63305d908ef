"""Plain, slow, obviously correct CPU oracle of the Llama-style decode forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product path (the CUDA library and its Python binding) never does and shares no
code with it.

It computes what the megakernel computes, written out from its definition in
float32 (the stated precision of the parity oracle) or float64 (used by the
self-checks), with numpy.  See :mod:`oracle.llama`.
"""

from .llama import (  # noqa: F401
    OracleModel,
    argmax_lowest,
    attention_decode,
    rmsnorm,
    rope_apply,
    rope_inv_freq,
    silu,
    softmax,
    top2_margin,
    weights_to_numpy,
)
