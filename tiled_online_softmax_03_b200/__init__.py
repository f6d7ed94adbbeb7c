"""B200-native (sm_100a) exact attention forward with the tiled online softmax.

The compute path is the C-ABI library ``libfa.so`` (hand-written CUDA for
sm_100a, declared in include/fa.h). ``binding`` marshals torch tensors into its
calls; importing it loads the library and fails loudly when it is missing.
"""

__all__ = ["fa_fwd", "fa_bwd", "fa_fwd_fp8", "fa_fwd_bias", "fa_fwd_splitkv", "fa_fwd_splitkv_static", "fa_fwd_from_host",
           "splitkv_workspace_bytes", "FaError", "load_library",
           "device_status"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
