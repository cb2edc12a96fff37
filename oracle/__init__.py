"""CPU oracle for the gated MLA hot path — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the method computes, written from
the pages' formulas.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never calls it and shares no code with it; the two meet only
through the seeded inputs of ``gated_mla_qk_b200.synth``.

Every function is pinned by ``-m "not gpu"`` tests in ``tests/test_oracle_*.py``
against closed forms, invariants, library routines (torch SDPA, torch RMSNorm,
torch's bf16 cast) and brute force on tiny inputs.  No function here is
"parity unpinned".
"""
from .mla import (  # noqa: F401
    bf16_round,
    rms_norm,
    up_proj,
    attention,
    attention_rows,
    head_maxlogit,
    attention_lse,
    attention_backward,
    qkclip,
    decode_absorbed,
    decode_materialised,
    layer_forward,
)
