"""BitNet b1.58 BitLinear forward on B200 (sm_100a).

The compute path is the C-ABI library ``libbitlinear.so`` (hand-written CUDA
kernels); :mod:`bitlinear_b1_fwd_b200.binding` marshals torch tensors into it.
"""
__version__ = "0.1.0"
