"""CPU oracle for the Split-KV hot path — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package. The CUDA library never calls it, links it or shares a
line of code with it, and it never imports the CUDA binding.

Every function here is a plain, slow restatement of what the method computes,
in float64 NumPy (integers for costs and plans), written from *Split-KV:
Efficient Context Parallelism for Training Diffusion Drafters* (Abstract):

* ``attention``  — the exact block-sparse cross-attention of anchor-sampled draft
  blocks over a long context (direct single-pass definition), its chunk-local
  partials, their exact log-sum-exp merge, and the gradients.
* ``schedule``   — the realized masked-attention cost of each context chunk work
  item and the cost-aware longest-processing-time-first (LPT) plan, plus the
  cost-blind equal split and an exhaustive optimum for pins.

Readings taken where the pages are silent are stated in each function's
docstring. Parity status: every function is pinned by ``tests/test_oracle_*.py``
against independent facts (library routines on explicit masks, closed forms,
invariants, brute force, exhaustive search, Graham's bound).
"""
from . import attention, schedule  # noqa: F401
