"""Float64 CPU oracle for the SSD (Mamba-2) forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The CUDA
library never calls it and shares no code with it.

The oracle is the plain definition of the scalar-times-identity selective SSM
run as a sequential recurrence ("Transformers are SSMs", paperlayer.ai summary,
§2.4, §3.4.1 and App. B.2.1), written in C (``ssd_oracle.c``) and driven from
``oracle.py``.  ``oracle_backward`` is the gradient of the same recurrence by the
chain rule; ``oracle_feature_map`` and ``oracle_forward_ext`` add the feature maps and
the denominator normalisation of §7.3 around it.  Every function here is pinned by ``tests/test_oracle_pins.py``; none
is "parity unpinned".
"""

from .oracle import (FMAP_BASED, FMAP_NONE, FMAP_REBASED, FMAP_RELU,  # noqa: F401
                     FMAP_SILU, build, oracle_backward, oracle_feature_map, oracle_forward,
                     oracle_forward_ext, oracle_step, oracle_threads)
