"""fp64 CPU oracle of the KATA causal forward — test infrastructure only.

Imported only by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py``.  The product path (the CUDA library and its binding)
never imports, links or calls anything here.
"""
