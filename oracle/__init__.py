"""Plain fp64 CPU oracle for the SALA hybrid attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may import,
call or link this package: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (``hybrid_sparse_linear_lightning_b200/csrc``) and
imports nothing from the library package; the only common module is the
seeded input generator ``hybrid_sparse_linear_lightning_b200.workloads``,
which holds no arithmetic of the method.

Every function states the passage of the pages it follows.  The pages name the
two attention kinds (InfLLM-V2 block-sparse, Lightning linear attention), the
1:3 layer mix, QK normalisation, HyPE (RoPE in linear layers, NoPE in sparse
layers) and an output gate after each block, but print no formula; where a
step is open, the plainest reading is taken and stated beside the code.

Pin status: every public function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, library routines, brute force, invariants).  The choices that
the pages leave open (no normaliser in the linear layer, the block-score rule,
the RMSNorm epsilon) are readings, not facts printed on the pages.
"""
from .sala_oracle import *  # noqa: F401,F403
