"""CPU oracle for the STAPLE embedding-augmented SwiGLU FFN layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs may import this package.  The CUDA
library never calls it and shares no code with it; the two meet only through
the seeded generators in ``synthetic``.

Everything here is the plain definition of what the layer computes, in fp64
numpy (matmul, sort and unique are library primitives used as single steps),
written from these sources:

  [ABS]   the paper's abstract, "STAPLE: Static Sparse Upcycling of Pretrained
          Checkpoints via Embedding Modules" (arXiv 2610.12599; as listed on
          hot.jian.ing, mlsanity.com and thelatestinai.com)
  [AIS]   ai4snews summary "Pretrained models gain sparse capacity without
          retraining: a zero-initialized memory path lifts ten-task average by
          1.20 points", sections Synopsis / Interpretation
  [RADIO] AI Radio episode "STAPLE: Static Sparse Upcycling of Pretrained
          Checkpoints via Embedding Modules", paper-summary segments
  [TLA]   thelatestinai.com listing of arXiv 2610.12599: Figure 4 caption,
          Table 4 (serving efficiency on one B200) and the unnumbered
          retrieval-path table (Prefill / Decode rows)

Readings taken where the pages are silent are listed in the docstrings of the
functions that depend on them.
"""
from .staple_oracle import *  # noqa: F401,F403
from .staple_oracle import __all__  # noqa: F401
