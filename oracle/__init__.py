"""CPU oracles for causal self-attention (test infrastructure only).

``oracle.oracle`` is the fp64 NumPy definition and ``oracle.brute`` is an
independent pure-Python loop version for tiny sizes. Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
them. The CUDA library never does, and it shares no code with them.
"""
