"""PagedAttention decode for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libpa.so`` (hand-written CUDA,
declared in ``include/paged_attention.h``); ``ops`` is its thin Python
binding: ``decode``, ``decode_append`` (slot write fused into decode),
``decode_noalloc``, ``prefill`` (several query tokens per sequence),
``reshape_and_cache`` and ``copy_blocks``.  ``block_allocator`` and
``workloads`` build seeded inputs on the host, ``capacity`` restates the
pages' capacity arithmetic, and ``scheduler`` simulates the
continuous-batching loop that drives the GPU path step by step.
"""
__version__ = "0.2.0"
