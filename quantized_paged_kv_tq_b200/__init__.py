"""TurboQuant paged KV cache for B200 (sm_100a).

The compute path lives in ``libtq.so`` (hand-written CUDA behind a C ABI,
declared in ``include/tq.h``).  ``quantized_paged_kv_tq_b200.tq`` is the thin
ctypes binding; importing it loads the library and fails loudly when it is
missing.  ``workloads`` draws the seeded synthetic inputs.
"""
__all__ = ["tq", "workloads"]


def __getattr__(name):
    if name == "tq":
        from . import tq
        return tq
    if name == "workloads":
        from . import workloads
        return workloads
    raise AttributeError(name)
