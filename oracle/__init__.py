"""fp64 CPU oracle for DiT joint attention and the KV-chunk log-sum-exp merge.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import, call, link or
run anything in this package.  The product path (``long_sequence_attention_b200``)
never touches it and shares no code with it; the only common module is
``workloads`` (seeded input generators, no attention arithmetic).

Contents
--------
``attention``      plain definition of non-causal softmax attention with an explicit
                   full softmax row, in fp64, over a KV range [k0, k1).
``merge``          exact log-sum-exp combination of per-chunk partials, fp64.
``fp8``            E4M3 decode / saturating round-to-nearest-even encode and the
                   per-tensor absmax quantisation, written from the format definition.
``brute``          an independent triple-loop C implementation in ``long double`` for
                   tiny shapes (``brute_attention.c``), used to pin ``attention``.
``neighborhood``   3-D neighborhood attention on a T x Y x X token grid (the NATTEN
                   na3d operation): clamped fixed-size windows, explicit softmax, fp64.

Parity status: every function here is pinned by ``tests/test_oracle.py`` (brute force,
closed forms, invariants, a library cross-check and planted-mistake checks).
"""

from .attn import attention, softmax_rows, merge, NEG_INF  # noqa: F401
from . import fp8  # noqa: F401
from . import neighborhood  # noqa: F401
