"""CPU oracle (float64) for the MoE layer forward.

TEST INFRASTRUCTURE: imported only by the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py``.  The product path
(the CUDA library and its Python binding) never imports it.
"""
