"""B200-native DSA sparse-attention step: lightning indexer -> top-k -> sparse MLA.

``binding`` exposes the C ABI of libdsa (include/dsa.h) to Python with the same
function names; ``workloads`` draws the seeded synthetic inputs; ``build``
compiles the library for sm_100a in-tree.
"""
from . import workloads  # noqa: F401  (numpy only; never loads the CUDA library)

__all__ = ["workloads", "binding", "build"]
