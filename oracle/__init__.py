"""CPU oracle for partitioned attention with selective attention-state reuse.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline / reference arm may import this package; the product path
(the CUDA library and its Python binding) never does, and this package never
imports the product.  It is plain, slow and fp64 on purpose: every function is
the definition written out, with library primitives (matmul, exp, log, sort)
as steps and no blocking or fusion beyond what the definition states.

Sources (pages, by title and section):
  * "DiTango: Cost-Effective Parallel Diffusion Generation with Selective
    Attention State Reuse", technical summary ("Riepilogo Tecnico"):
      - Metodologia (spatial locality of attention contributions);
      - 1. Anchor-Guided Selection Planner (error model with partition
        importance w, anchor steps, group strategy "Strategia per Gruppi");
      - 2. State-Centric Parallel Runtime, "Composizione dello Stato"
        (attention state = output + log-sum-exp, composed associatively and
        commutatively; cached instead of raw KV), "Calcolo dello Stato di
        Gruppo" and "Composizione Dinamica dei Gruppi" (group states; cached
        states merged recursively into coarser groups).
  * "Efficient-vDiT: Efficient Video Diffusion Transformers With Attention
    Tile", abstract (tile-style repeating pattern, sparse 3D attention linear
    in the number of frames).

Parity status per function:
  attention.partial_state, attention.merge_states, attention.dense_attention,
  masks.*, plan.select, plan.mass_scores, step.*, groups.*
  -- pinned (tests/test_oracle_*.py)
  error_plan.* -- its rules and their invariants pinned
  (tests/test_oracle_error_plan.py); the error model's predictive quality
  -- parity unpinned: the pages give no formula and no values.
  The quality of reuse (how far a reuse step drifts from an all-fresh step)
  -- parity unpinned: the pages print no error values; it is reported only.
"""
from .attention import partial_state, merge_states, dense_attention  # noqa: F401
from .masks import pair_mask, slot_table, token_allowed, frame_of  # noqa: F401
from .plan import mass_scores, select, budget_target, PLAN_SKIP, PLAN_FRESH, PLAN_REUSE  # noqa: F401
from . import step, groups, error_plan  # noqa: F401
