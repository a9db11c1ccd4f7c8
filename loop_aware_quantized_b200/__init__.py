"""LoopKV fused decode attention over a per-(loop, layer) mixed-precision KV
cache, for NVIDIA B200 (sm_100a).

The work runs in ``libloopkv.so`` (hand-written CUDA kernels behind the C ABI
of ``include/loopkv.h``); ``loopkv`` is its Python binding.  The binding is
imported on first use of a name below, and that import fails if the library
has not been built: there is no other code path.
"""

_EXPORTS = ("LOOPKV_BF16", "LOOPKV_Q2", "LOOPKV_Q4", "LOOPKV_RES2", "LOOPKV_SHARE", "LoopKVError", "Plan",
            "plan_optimize", "query_sizes", "vq_decode", "vq_encode")


def __getattr__(name):
    if name in _EXPORTS:
        from . import loopkv
        return getattr(loopkv, name)
    raise AttributeError(name)
