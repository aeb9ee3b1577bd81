"""B200-native LatentMoE layer forward pass.

``lmoe`` is the Python binding of the C-ABI library ``liblmoe.so`` (imported
lazily so that the workload generator and the cost model load without it).
"""
__all__ = ["lmoe", "workloads", "costmodel"]


def __getattr__(name):
    if name == "lmoe":
        from . import lmoe
        return lmoe
    raise AttributeError(name)
