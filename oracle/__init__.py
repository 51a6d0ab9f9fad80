"""fp64 CPU oracle for Split-KV block-sparse anchor attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package: only
the tests, the smoke check and the bench's CPU-baseline leg may call it.  It
shares no code with the CUDA path (no kernels, headers, helpers or tables).

Sources (the two pages on the method):

* [digest]  "Split-KV: Efficient Context Parallelism for Training Diffusion
  Drafters", paper digest page, Abstract.
* [news]    "Split-KV speeds diffusion drafter training by keeping long-context
  data local", news page, sections "Why short queries change the problem",
  "Exchange the smaller side" and "Balance actual attention work".

What is computed, and where the pages leave a step open (each reading is also
listed in the repository's design notes):

* mask ([news] "Why short queries change the problem"): block b, opened by
  anchor a_b in packed sample s, attends to the preceding context of its own
  sample, keys [S_s, a_b) (the anchor itself excluded), plus all bs tokens of
  its own block.  Reading: the block's tokens are the draft block's own keys
  and values (Kb, Vb, one row per draft token), every row of a block sees all
  bs of them, and all rows of a block share one context interval.
* exact combine ([news] "Exchange the smaller side"; [digest]): partial
  attention over disjoint key sets merged with their normalisation statistics
  (running max m, sum l) reproduces unsplit softmax attention.  A partial with
  no allowed key has m = -inf, l = 0, O = 0 and contributes nothing.
* cost and LPT ([news] "Balance actual attention work"; [digest]): a chunk's
  cost is its realised attention usage (allowed query-key pairs); LPT sorts
  items by cost, longest first, and gives each to the least-loaded eligible
  worker; "eligible" keeps item counts equal in the equal-count mode.

Modules: mask (intervals, chunk entries, pair counts), attention (forward,
backward, chunk partials, merge), lpt (work items, LPT, contiguous baseline,
imbalance), context_parallel (chunk ownership over ranks, a rank's partial
result and backward share, the combine over ranks).  All floating point is
float64.
"""

from . import mask, attention, lpt, context_parallel  # noqa: F401
