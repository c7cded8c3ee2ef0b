"""HiLS attention on B200 (sm_100a): C-ABI library + thin binding.

``chunk_sparse_long_b200.hils`` is the binding of include/hils.h: the prefill
and decode forward, the prefill backward with the chunk selection held fixed
(``prefill_backward``), and the calls of the context-parallel decode step.
``chunk_sparse_long_b200.cp`` runs that step over a torch.distributed group
(``cp.Decoder``).  ``build`` compiles the library in-tree.  Importing the
package does not load the CUDA library.
"""
__all__ = ["hils", "build", "cp"]
