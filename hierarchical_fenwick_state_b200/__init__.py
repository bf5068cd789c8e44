"""B200-native log-linear attention forward (Mamba-2 form).

The compute path is the C-ABI library ``libllattn.so`` built from ``csrc/``
(hand-written sm_100a CUDA); ``binding`` marshals torch tensors into it.
Importing this package does not load the library; ``binding.lib()`` does, and
raises if it is missing.
"""
__all__ = ["inputs", "binding"]
