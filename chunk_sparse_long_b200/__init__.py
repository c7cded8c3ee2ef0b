"""HiLS attention forward on B200 (sm_100a): C-ABI library + thin binding.

``chunk_sparse_long_b200.hils`` is the binding; ``build`` compiles the
library in-tree.  Importing the package does not load the CUDA library.
"""
__all__ = ["hils", "build"]
