"""fp64 CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does; the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over
(sequence, head)); ``brute.py`` restates the attention definition in pure
Python for tiny inputs.  This module only compiles the C file with gcc and
marshals numpy arrays into it.

Parity of every function here is pinned by ``tests/test_oracle_pins.py``
against things other than itself: torch's scaled-dot-product attention on a
contiguous gather (a library special case), closed forms (one token, constant
V, zero query), invariants (block permutation, prefix sharing, split-K
identity) and hand-derived values under ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_oracle.so")

_DT = {"f32": 0, "bf16": 1}
_lib: Optional[ctypes.CDLL] = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB, extra=()) -> str:
    """Compile ``oracle.c`` (gcc -O2 -fopenmp) into a shared library."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *extra, src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    p, i, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
    lib.oracle_paged_decode.argtypes = [p, p, p, p, p, p] + [i] * 8 + [d, i]
    lib.oracle_paged_decode.restype = i
    lib.oracle_paged_decode_partitioned.argtypes = [p, p, p, p, p, p] + [i] * 8 + [d, i, i]
    lib.oracle_paged_decode_partitioned.restype = i
    lib.oracle_paged_prefill.argtypes = [p, p, p, p, p, p, p] + [i] * 9 + [d, i]
    lib.oracle_paged_prefill.restype = i
    lib.oracle_reshape_and_cache.argtypes = [p, p, p, p, p] + [i] * 6
    lib.oracle_reshape_and_cache.restype = i
    lib.oracle_copy_blocks.argtypes = [p, p, p] + [i] * 6
    lib.oracle_copy_blocks.restype = i
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = i
    return lib


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """The compiled oracle (built on first use)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def num_threads() -> int:
    return int(load().oracle_num_threads())


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype=None) -> np.ndarray:
    return np.ascontiguousarray(a if dtype is None else np.asarray(a, dtype=dtype))


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, *, scale: float,
                 dtype: str, max_context_len: Optional[int] = None,
                 partition_size: int = 0, lib: Optional[ctypes.CDLL] = None):
    """fp64 attention output ``[S][Hq][D]`` and the error bits.

    ``q``: ``[S][Hq][D]``; caches ``[N][Hkv][block_size][D]`` as float32, or
    as int16/uint16 bf16 bit patterns when ``dtype == "bf16"``.  With
    ``partition_size > 0`` the split-K form with log-sum-exp merge is used.
    """
    lib = lib or load()
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    tables = _c(block_tables, np.int32)
    lens = _c(context_lens, np.int32)
    S, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape and tables.shape[0] == S
    if max_context_len is None:
        max_context_len = int(lens.max()) if S else 0
    out = np.zeros((S, Hq, D), dtype=np.float64)
    args = [_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(tables), _ptr(lens),
            S, Hq, Hkv, D, bs, tables.shape[1], N, int(max_context_len), float(scale), _DT[dtype]]
    if partition_size > 0:
        err = lib.oracle_paged_decode_partitioned(*args, int(partition_size))
    else:
        err = lib.oracle_paged_decode(*args)
    return out, int(err)


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, *, scale: float,
                  dtype: str, max_context_len: Optional[int] = None,
                  lib: Optional[ctypes.CDLL] = None):
    """fp64 causal attention of several query tokens per sequence, the last
    ``Q_s = query_start[s+1] - query_start[s]`` of its ``context_lens[s]``
    tokens.  ``q``: ``[query_start[S]][Hq][D]``; returns ``(out, err_bits)``."""
    lib = lib or load()
    q, k_cache, v_cache = _c(q), _c(k_cache), _c(v_cache)
    tables = _c(block_tables, np.int32)
    lens = _c(context_lens, np.int32)
    qs = _c(query_start, np.int32)
    T, Hq, D = q.shape
    N, Hkv, bs, D2 = k_cache.shape
    S = lens.shape[0]
    assert D2 == D and v_cache.shape == k_cache.shape and tables.shape[0] == S
    assert qs.shape[0] == S + 1
    if max_context_len is None:
        max_context_len = int(lens.max()) if S else 0
    out = np.zeros((T, Hq, D), dtype=np.float64)
    err = lib.oracle_paged_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(tables),
                                   _ptr(lens), _ptr(qs), S, T, Hq, Hkv, D, bs, tables.shape[1], N,
                                   int(max_context_len), float(scale), _DT[dtype])
    return out, int(err)


def reshape_and_cache(k_cache, v_cache, key, value, slot_mapping, *,
                      lib: Optional[ctypes.CDLL] = None) -> int:
    """Slot write into ``k_cache``/``v_cache`` in place; returns the error bits."""
    lib = lib or load()
    for a in (k_cache, v_cache):
        assert a.flags["C_CONTIGUOUS"]
    key, value = _c(key), _c(value)
    slots = _c(slot_mapping, np.int64)
    N, Hkv, bs, D = k_cache.shape
    return int(lib.oracle_reshape_and_cache(_ptr(k_cache), _ptr(v_cache), _ptr(key), _ptr(value),
                                            _ptr(slots), int(slots.shape[0]), Hkv, D, bs, N,
                                            k_cache.itemsize))


def copy_blocks(k_cache, v_cache, block_mapping, *, lib: Optional[ctypes.CDLL] = None) -> int:
    """Whole-block copies ``dst <- src`` in place; returns the error bits."""
    lib = lib or load()
    for a in (k_cache, v_cache):
        assert a.flags["C_CONTIGUOUS"]
    pairs = _c(block_mapping, np.int32).reshape(-1, 2)
    N, Hkv, bs, D = k_cache.shape
    return int(lib.oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), int(pairs.shape[0]),
                                      Hkv, D, bs, N, k_cache.itemsize))


def workload_step(w, partition_size: int = 0, lib: Optional[ctypes.CDLL] = None):
    """The whole hot path of a workload on its compact pool, in step order:
    copy-on-write copies, the slot write of the new tokens, then attention.
    Returns ``(out_fp64, k_pool_after, v_pool_after, err_bits)``."""
    k = w.k_pool.copy()
    v = w.v_pool.copy()
    err = 0
    if w.block_mapping_compact is not None:
        err |= copy_blocks(k, v, w.block_mapping_compact, lib=lib)
    if w.new_key is not None:
        err |= reshape_and_cache(k, v, w.new_key, w.new_value, w.slot_mapping_compact, lib=lib)
    if getattr(w, "query_start", None) is not None:
        out, e = paged_prefill(w.q, k, v, w.tables_compact, w.context_lens, w.query_start,
                               scale=w.scale, dtype=w.dtype, lib=lib)
    else:
        out, e = paged_decode(w.q, k, v, w.tables_compact, w.context_lens, scale=w.scale,
                              dtype=w.dtype, partition_size=partition_size, lib=lib)
    return out, k, v, err | e
