"""RotateAttention INT4 attention forward for B200 (sm_100a).

The compute path is the C-ABI library ``librotate_attn.so`` (hand-written
CUDA); ``api`` is its thin Python binding.  Importing the package loads
nothing: ``synth`` (seeded inputs) and ``schedule`` (FP16/INT4 dispatch) are
host-only helpers.
"""
