"""CPU oracle of the speculative-decoding verify step -- TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the verify step computes, used to check the
CUDA kernels.  Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import it; the product path (the ``verify_step_b200`` package and its CUDA library) never
does, and shares no code with it.

Modules
  philox     Philox4x32-10 and the uniforms of the acceptance rule
  attention  verify attention (k+1 causal queries, paged GQA cache, sliding or global)
             and the drafter's read-only cross-attention into the same cache
  lm_head    dense LM head and the clustered two-stage drafter head
  accept     lossless acceptance, correction and bonus draws (T > 0) and greedy (T = 0)
  commit     committed length, committed slots, rollback and next hidden row
  drafter    the drafter's dense layers around its cross-attention (one link of the chain)
  target     the target's layers over the k+1 verified positions (multi-layer verify)

Parity status: every function is pinned by tests/test_oracle_*.py against closed forms,
invariants, library routines, brute-force enumeration or published known answers, except
agreement with real Gemma 4 / vLLM / FlashInfer outputs (no weights or traces exist here).
"""
from . import accept, attention, commit, drafter, lm_head, philox, target  # noqa: F401
