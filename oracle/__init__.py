"""CPU oracle for Hybrid Linear Attention over Gated DeltaNet.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import, call or run
anything in this package.  The GPU library never does, shares no code with it, and
has no CPU fallback.

* ``hla_oracle``      -- fp64 definition: token rule, literal chunk transitions, the
                         WY/UT form (for comparison), gated composition, prefill,
                         decode.
* ``routing_recipe``  -- the bit-level binary32 routing recipe (pools, gates).
* ``brute``           -- pure-Python explicit-matrix brute force for tiny inputs.

Parity status: every function is pinned by ``tests/test_oracle_*.py`` against closed
forms, special cases, exact rational brute force, fp64 library routines or the
mathematics; nothing here is "parity unpinned" except absolute outputs of a trained
model, which no page prints.
"""
from . import hla_oracle, routing_recipe, brute  # noqa: F401
