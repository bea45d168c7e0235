"""B200-native (sm_100a) fused exact attention, forward and backward.

The compute lives in ``libattn.so`` (CUDA kernels behind the C ABI declared in
``include/attn.h``).  ``capi`` binds those entry points with ctypes under the
same names; ``ops`` wraps them for torch tensors (``attn_fwd``, ``attn_bwd``,
``attention``).  ``inputs`` holds the seeded synthetic-input generator.
"""
__version__ = "1.0.0"


def __getattr__(name):
    if name in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attention"):
        from . import ops
        return getattr(ops, name)
    raise AttributeError(name)
