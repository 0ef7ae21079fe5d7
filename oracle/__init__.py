"""CPU oracle of the score-then-select sparse decode step.

TEST INFRASTRUCTURE ONLY. Tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline
leg (and its ``--impl reference`` arm) are the only code that may import it. It shares no
code, header, table or constant generator with the CUDA path, and never calls it.

Pins (what each part is checked against, in tests/test_oracle_*.py):
  formats   - hand-derived E2M1 / UE4M3 / BF16 values from the format definitions,
              round trips, nearest-even midpoints, exact rational rounding;
  writer    - identity projection, single-entry projections, a summation-order case whose
              answer differs by order, the float32 dot-product error bound;
  score     - group-mean linearity; rank = d with P = I equals the exact group-mean score;
              block max against loops;
  select    - exhaustive subset search on tiny inputs, invariants, budget >= blocks;
  attention - brute-force dense softmax attention with math.fsum when the budget covers
              every block; one-hot selection; split-count invariance of the LSE combine;
  NVFP4     - factored block-scaled dot product against dequantise-then-dot; exactly
              representable round trips; the per-element error bound; kept blocks by
              exhaustive search; planted needle selected;
  binary    - an exactly representable rotated case whose estimate is the exact score; the
              mean over random rotations and query roundings against the exact score
              (unbiasedness); identity and signed-permutation rotations; bit packing;
  top-p     - exhaustive subset search on tiny inputs; closed forms for uniform and
              geometric masses; the budget cap; forced blocks;
  semantic  - Lloyd's objective never increases; converged partitions are fixed points;
              exactly placed keys recovered; one token per cluster = token level; cluster
              score = mean member score; full budget = dense attention; planted cluster.
Parity unpinned: the aggregation of per-head NVFP4 scores into one block score (max over
the group's heads), and the semantic blocks' clustering (Lloyd's k-means, evenly spaced
seeds), are readings the pages leave open; only their implementations are pinned.
"""
from . import formats, method, step  # noqa: F401
