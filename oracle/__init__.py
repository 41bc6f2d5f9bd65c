"""CPU oracle for CRISP sparse prefill — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the CRISP paper ("Cliff-awaRe
Input-adaptive Sparse Prefilling with Structural-Mass-Motivated Routing")
computes: proxy attention (Algorithm 2), C_struct routing (Eq. 2), the JSD
router of its Appendix A (Algorithm 5), sink-aware vertical-slash selection
(Algorithm 3, Eq. 3-4), the gamma-cumulative selections (Algorithms 4 and 6)
and masked attention (Eq. 1).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never calls it and
shares no code with it.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test against
an independent fact (brute force, a closed form, an invariant or a
hand-computed case); none is "parity unpinned".
"""
from .crisp import *  # noqa: F401,F403
from .crisp import __all__  # noqa: F401
