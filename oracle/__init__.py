"""fp64 CPU oracle for the token-pruned attention path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package. The product path
(``token_pruned_sparse_b200``) never imports it, and it never imports the
product path: the two share no code. Only the seeded input generators
(``token_pruned_sparse_b200.synth``, which holds none of the method's
arithmetic) feed both.

Parity status per function (see each docstring for the pins):
  lipar_score, select_threshold, select_topk, group_split, schedule_active,
  kv_sync, pruned_attn, scatter_out  -- pinned by tests/test_oracle_pins.py
  euler_update, lse_merge, lipar_score_motion,
  timeripple_delta/_reuse/_token_score/_theta,
  rope_rotate, kv_rerotate             -- pinned likewise (hand-worked
                                         fixtures, closed forms, invariants,
                                         complex-number form)
  philox4x32_10 raw stream            -- pinned by the published
                                         known-answer vectors (Salmon et al.,
                                         SC'11), and its normals statistically.
"""
from .tps_oracle import *  # noqa: F401,F403
from .tps_oracle import __all__  # noqa: F401
