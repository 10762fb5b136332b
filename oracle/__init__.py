"""KDA CPU oracle -- TEST INFRASTRUCTURE ONLY.

Plain fp64 CPU implementations used to check the CUDA library: the token-by-token
recurrence (``oracle.oracle``, C via ctypes) and a naive chunkwise form
(``oracle.chunkwise``, NumPy).  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  It shares no
code with the CUDA path, and the CUDA path never imports it.

Parity status: every function here is pinned by ``tests/test_oracle.py`` (brute
force products, closed forms, special cases and invariants fixed by the
definition).
"""
