"""CPU oracle for frame/block-sparse video attention (LVSA and LoSA).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import anything in this package.  The
CUDA library and its Python binding never import it, and this package
imports nothing from them: the two share no code.

Plain, slow, obviously correct code: numpy in float64 (integers exact), one
function per step of the method, each citing the passage it follows.  The
sources are two web pages:

* [LVSA] "LVSA: Training-Free Sparse Attention for Long Video Diffusion"
  (gist.science explainer of arXiv 2605.31057), technical summary, section 2
  "Method" (core mechanism A(t) = G u W(t); rotating global anchors;
  expanded adaptive window; computational complexity).
* [LoSA] "LoSA (Near-Lossless Sparse Attention)" article (ai.ros.co.jp,
  2026-08-14), sections "LoSA's innovative approach" (99% mass constraint,
  about 40% of block interactions removable, high-mass support stable over
  denoising steps) and "Balancing efficiency and quality" (one dense step
  measures exact inter-block mass; per head and query block the minimal
  key/value block set holding 99% of the mass is kept; the index is frozen
  and reused at every later step).

Where the pages leave a step open the reading taken is stated in the
function's docstring.  Every function here is pinned by tests that do not
re-type its formula: hand-derived fixtures, closed forms, invariants, a
library routine on special cases, and brute force on tiny inputs.
"""
from . import lvsa, tiles, attention, losa  # noqa: F401
