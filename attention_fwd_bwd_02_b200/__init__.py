"""B200-native fused attention (forward and backward) for sm_100a.

The compute path is the C-ABI library ``libfa_b200.so`` (CUDA kernels under
``csrc/``); ``attention_fwd_bwd_02_b200.fa`` is the thin ctypes binding over
it.  The library is loaded on first use and its absence is an error: there
is no CPU or PyTorch fallback.
"""
