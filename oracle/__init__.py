"""CPU oracle for the DraftAttention2 hot path — TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, deliberately unoptimised restatement of what the
low-resolution-guided mixed-precision block-sparse attention computes.  It runs
in fp64 with numpy and exists to check the CUDA library.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and reference
legs) may import it; the product path never does.  It shares no code, tables or
helpers with ``mixed_precision_block_b200``; both sides only share the seeded
input generator in ``mixed_precision_block_b200/synth.py``, which holds none of
the method's arithmetic.

Sources (cited by page title and section throughout):

* "DraftAttention2 abstract" — the abstract on the paper card
  *DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided
  Mixed-Precision Attention*.
* "DraftAttention2 reading note" — the Chinese reading note on the same paper
  (title *DraftAttention2：用低分草稿引导的混合精度注意力加速视频扩散*): its
  "Method overview" section and bullets 1-4, the Figure 2 and Figure 3
  captions, and its "How are the experiments designed" and "Key results"
  sections.
* "DraftAttention abstract" — the abstract of the v1 paper *DraftAttention:
  Fast Video Diffusion via Low-Resolution Attention Guidance*.

Where the pages leave a step open, the reading adopted is stated next to the
code that implements it.  Functions whose result is not pinned by a test to
something other than this package say "parity unpinned" in their docstring.

Parity unpinned (covered only by tolerance, nothing on the pages pins them):
the accumulation order of the tensor-core products, the GPU's exponential, and
the bf16 rounding order of P in the 16-bit phase (``attention.py``).
"""

from .problem import Problem, CONFIGS  # noqa: F401
from . import geometry, formats, prep, draft, rank, attention, pipeline  # noqa: F401
