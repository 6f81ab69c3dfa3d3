"""CPU oracles for causal self-attention (test infrastructure only).

``oracle.oracle`` is the fp64 NumPy definition and ``oracle.brute`` is an
independent pure-Python loop version for tiny sizes. ``oracle.linear`` is the
fp64 definition of the block's two dense layers around attention (c_attn,
c_proj), and ``oracle.fp8`` the per-tensor e4m3 quantiser that the FP8
forward's inputs are checked with. Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
them. The CUDA library never does, and it shares no code with them.
"""
