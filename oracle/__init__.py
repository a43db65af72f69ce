"""CPU oracle for the FP8 ViT block, merger and tower forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package.  The CUDA library
never calls it and it never calls the CUDA library: the two share no code,
tables or constants beyond the seeded input generator.

The oracle is plain numpy in fp64 (plus fp32 exactly where the method's own
integer decisions are taken: the FP8 scale and the value that is rounded to an
E4M3 code).  It is written for readability, not speed.

Modules
-------
numerics : bf16 and OCP FP8 E4M3 ("E4M3FN") rounding written from their
           definitions (round-to-nearest-even, saturating at 448).
vit      : the stages of the block (LayerNorm+quant, FP8 block-128 GEMM,
           2D rotary, varlen attention, GELU+quant), the 2x2 merger and the
           27-block tower with its DeepStack taps.

Pinning: every stage function is checked against something other than itself
in ``tests/test_oracle_pins.py`` (closed forms, exhaustive code tables, library
casts, brute-force loops, invariants).  The block, merger and tower have no
published values; their wiring is pinned in ``tests/test_oracle_compositions.py``
by closed forms and invariants of the method (zero-weight blocks reduce to their
residual adds, the taps follow blocks 8, 16, 24 and 27, packed images equal
images alone, the merger normalises four concatenated rows and maps each group
of four rows to one output row), and their arithmetic through the pinned stages.
"""
from . import numerics, vit  # noqa: F401
