"""TurboQuant paged KV cache for B200 (sm_100a).

The compute path lives in ``libtq.so`` (hand-written CUDA behind a C ABI,
declared in ``include/tq.h``):

* ``quantized_paged_kv_tq_b200.tq`` -- the thin ctypes binding; importing it
  loads the library and fails loudly when it is missing.
* ``quantized_paged_kv_tq_b200.workloads`` -- seeded synthetic inputs.
* ``quantized_paged_kv_tq_b200.build`` -- nvcc build of ``libtq.so``.
"""
