"""fp64 CPU oracle for GPTQ single-layer quantization.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import or run anything in this
package.  The CUDA library never calls it and shares no code with it; the only
thing both sides share is the seeded input generator
(``post_weight_quantization_05_b200.synth``), which holds none of the method's
arithmetic.
"""
from .gptq import *  # noqa: F401,F403
