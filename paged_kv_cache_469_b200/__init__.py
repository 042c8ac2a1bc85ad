"""Paged KV-cache attention for B200 (sm_100a).

The compute lives in ``libpa.so`` (CUDA kernels behind the C ABI declared in
``include/pa.h``); this package builds it and marshals arguments to it:

- ``build``: compiles ``libpa.so`` in-tree with nvcc for sm_100a.
- ``lib``: ctypes binding, one function per C entry point:
  ``reshape_and_cache``, ``attention_varlen``, ``attention_varlen_write_cache``
  (the cache write and attention of one step in one call), ``plan_step`` (one
  scheduler step's block allocation, ``seq_lens``, ``query_start_loc`` and
  slot mapping on the GPU), and the workspace helpers.
- ``block_pool``: the same bookkeeping on the host (free queue,
  ``allocate_slots``, block tables, slot mapping, super-sequence offsets).
- ``step``: ``DeviceStep``, one step's tensors on the device, with CUDA-graph
  capture of the step.
- ``inputs``: seeded synthetic workloads (random draws only).
- ``run_workload``: runs a named workload's steps (for profiling).
"""
