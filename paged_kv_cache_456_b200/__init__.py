"""PagedAttention decode for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libpa.so`` (hand-written CUDA);
``ops`` is its thin Python binding.  ``block_allocator`` and ``workloads``
build seeded inputs on the host.
"""
__version__ = "0.1.0"
