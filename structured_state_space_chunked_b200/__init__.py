"""B200-native forward pass of the chunked SSD (Mamba-2) scan.

The compute path is ``libssd_b200.so`` (CUDA kernels for sm_100a behind the C-ABI
declared in ``include/ssd.h``).  ``ssd`` is the thin Python binding over that
library; ``inputs`` draws the seeded synthetic workloads.  Importing this package
does not load the CUDA library; the first call into ``ssd`` does, and it raises
if the library is missing.
"""

__all__ = ["inputs", "ssd", "build"]
