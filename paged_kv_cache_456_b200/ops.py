"""Python binding of ``libpa.so`` (include/paged_attention.h).

Argument marshalling only: tensors are turned into device pointers and sizes
and handed to the C ABI on the current CUDA stream.  Every step of the path
runs in the library's CUDA kernels; there is no fallback.  If the library has
not been built, :func:`library` raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

# PA_LIBRARY selects another build of the library (e.g. a tuning variant)
_LIB_PATH = os.environ.get("PA_LIBRARY") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libpa.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA = range(5)
PA_F32, PA_BF16 = 0, 1

ERRBIT_BLOCK_ID = 1
ERRBIT_CONTEXT_LEN = 2
ERRBIT_SLOT = 4
ERRBIT_PAIR = 8
ERRBIT_TIMEOUT = 16
ERRBIT_QUERY = 32
ERRBIT_GROUP = 64

EXPORTED = ("pa_status_str", "pa_decode_workspace_size", "pa_decode_workspace_init",
            "pa_decode_launch_config", "pa_decode", "pa_decode_noalloc", "pa_decode_append",
            "pa_prefill", "pa_prefill_workspace_size", "pa_prefill_launch_config",
            "pa_reshape_and_cache", "pa_copy_blocks", "pa_shared_prefix_plan",
            "pa_shared_prefix_plan_tree",
            "pa_shared_prefix_workspace_size", "pa_decode_shared_prefix")

# size of the library's fixed scratch array used by pa_decode_noalloc
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_str(status)}")
        self.status = status


_lib: Optional[ctypes.CDLL] = None


def library(path: Optional[str] = None) -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m paged_kv_cache_456_b200.build`"
                           " (the CUDA library is the only implementation)")
    lib = ctypes.CDLL(p)
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    lib.pa_status_str.argtypes = [i]
    lib.pa_status_str.restype = ctypes.c_char_p
    lib.pa_decode_workspace_size.argtypes = [i] * 7 + [ctypes.POINTER(sz)]
    lib.pa_decode_workspace_size.restype = i
    lib.pa_decode_workspace_init.argtypes = [vp, sz, vp]
    lib.pa_decode_workspace_init.restype = i
    lib.pa_decode_launch_config.argtypes = [i] * 7 + [ctypes.POINTER(i)] * 4
    lib.pa_decode_launch_config.restype = i
    lib.pa_decode.argtypes = [vp] * 6 + [i] * 8 + [f, i, i, vp, sz, vp, vp]
    lib.pa_decode.restype = i
    lib.pa_decode_noalloc.argtypes = [vp] * 6 + [i] * 8 + [f, i, i, vp, vp]
    lib.pa_prefill_launch_config.restype = i
    lib.pa_prefill_launch_config.argtypes = [i] * 8 + [ctypes.POINTER(i)] * 4
    lib.pa_prefill_workspace_size.restype = i
    lib.pa_prefill_workspace_size.argtypes = [i] * 8 + [ctypes.POINTER(sz)]
    lib.pa_prefill.restype = i
    lib.pa_prefill.argtypes = [vp] * 7 + [i] * 9 + [f, i, i, vp, sz, vp, vp]
    lib.pa_decode_append.restype = i
    lib.pa_decode_append.argtypes = [vp] * 8 + [i] * 8 + [f, i, i, vp, sz, vp, vp]
    lib.pa_decode_noalloc.restype = i
    lib.pa_reshape_and_cache.argtypes = [vp] * 5 + [i] * 6 + [vp, vp]
    lib.pa_reshape_and_cache.restype = i
    lib.pa_copy_blocks.argtypes = [vp] * 3 + [i] * 6 + [vp, vp]
    lib.pa_copy_blocks.restype = i
    ip = ctypes.POINTER(i)
    lib.pa_shared_prefix_plan.argtypes = [vp, vp] + [i] * 4 + [vp, vp, vp, ip, ip]
    lib.pa_shared_prefix_plan.restype = i
    lib.pa_shared_prefix_plan_tree.argtypes = [vp, vp] + [i] * 4 + [vp, vp, vp, ip, ip]
    lib.pa_shared_prefix_plan_tree.restype = i
    lib.pa_shared_prefix_workspace_size.argtypes = [i] * 9 + [ctypes.POINTER(sz)]
    lib.pa_shared_prefix_workspace_size.restype = i
    lib.pa_decode_shared_prefix.argtypes = [vp] * 11 + [i] * 10 + [f, i, i, vp, sz, vp, vp]
    lib.pa_decode_shared_prefix.restype = i
    if path is None:
        _lib = lib
    return lib


def status_str(status: int) -> str:
    return library().pa_status_str(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        raise PagedAttentionError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float32:
        return PA_F32
    raise TypeError(f"unsupported element type {t.dtype} (float32 or bfloat16)")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libpa must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------
def workspace_size(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                   max_context_len: int, partition_size: int = 0,
                   dtype: torch.dtype = torch.bfloat16) -> int:
    out = ctypes.c_size_t(0)
    code = PA_BF16 if dtype == torch.bfloat16 else PA_F32
    _check(library().pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              max_context_len, partition_size, code,
                                              ctypes.byref(out)), "pa_decode_workspace_size")
    return int(out.value)


def make_workspace(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                   max_context_len: int, partition_size: int = 0,
                   dtype: torch.dtype = torch.bfloat16, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size ``pa_decode`` needs."""
    n = workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                       partition_size, dtype)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def make_prefill_workspace(num_seqs: int, num_query_tokens: int, num_q_heads: int,
                           num_kv_heads: int, head_dim: int, max_context_len: int,
                           partition_size: int = 0, dtype: torch.dtype = torch.bfloat16,
                           device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size ``pa_prefill`` needs."""
    n = ctypes.c_size_t(0)
    _check(library().pa_prefill_workspace_size(
        num_seqs, num_query_tokens, num_q_heads, num_kv_heads, head_dim, int(max_context_len),
        int(partition_size), PA_BF16 if dtype == torch.bfloat16 else PA_F32, ctypes.byref(n)),
        "pa_prefill_workspace_size")
    return torch.zeros(max(n.value, 16), dtype=torch.uint8, device=device)


def launch_config(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                  max_context_len: int, partition_size: int = 0,
                  dtype: torch.dtype = torch.bfloat16) -> dict:
    vals = [ctypes.c_int(0) for _ in range(4)]
    code = PA_BF16 if dtype == torch.bfloat16 else PA_F32
    _check(library().pa_decode_launch_config(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                             max_context_len, partition_size, code,
                                             *[ctypes.byref(v) for v in vals]),
           "pa_decode_launch_config")
    return dict(zip(("grid", "warps_per_cta", "pipeline_depth", "smem_bytes"),
                    (v.value for v in vals)))


def prefill_launch_config(num_seqs: int, num_query_tokens: int, num_q_heads: int,
                          num_kv_heads: int, head_dim: int, max_context_len: int,
                          partition_size: int = 0, dtype: torch.dtype = torch.bfloat16) -> dict:
    vals = [ctypes.c_int(0) for _ in range(4)]
    code = PA_BF16 if dtype == torch.bfloat16 else PA_F32
    _check(library().pa_prefill_launch_config(num_seqs, num_query_tokens, num_q_heads,
                                              num_kv_heads, head_dim, max_context_len,
                                              partition_size, code,
                                              *[ctypes.byref(v) for v in vals]),
           "pa_prefill_launch_config")
    return dict(zip(("grid", "warps_per_cta", "pipeline_depth", "smem_bytes"),
                    (v.value for v in vals)))


def decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           block_tables: torch.Tensor, context_lens: torch.Tensor, *, scale: float,
           max_context_len: int, workspace: torch.Tensor, partition_size: int = 0,
           err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """PagedAttention decode into ``out`` ``[S][Hq][D]``; see ``pa_decode``."""
    S, Hq, D = q.shape
    N, Hkv, bs, _ = k_cache.shape
    _check(library().pa_decode(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        S, Hq, Hkv, D, bs, block_tables.shape[1], N, int(max_context_len), float(scale),
        int(partition_size), _dtype_code(q), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(err_flag), _stream(stream)), "pa_decode")
    return out


def decode_append(out: torch.Tensor, q: torch.Tensor, key: torch.Tensor, value: torch.Tensor,
                  k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                  context_lens: torch.Tensor, *, scale: float, max_context_len: int,
                  workspace: torch.Tensor, partition_size: int = 0,
                  err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Write each sequence's newest ``key``/``value`` row ``[S][Hkv][D]`` into its
    cache slot and decode over it in the same launch; see ``pa_decode_append``."""
    S, Hq, D = q.shape
    N, Hkv, bs, _ = k_cache.shape
    _check(library().pa_decode_append(
        _ptr(out), _ptr(q), _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), _ptr(context_lens), S, Hq, Hkv, D, bs, block_tables.shape[1], N,
        int(max_context_len), float(scale), int(partition_size), _dtype_code(q), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(err_flag), _stream(stream)),
        "pa_decode_append")
    return out


def prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
            block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor, *,
            scale: float, max_context_len: int, workspace: torch.Tensor, partition_size: int = 0,
            err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Causal attention of ``q`` ``[T][Hq][D]``, the last ``query_start[s+1] -
    query_start[s]`` tokens of each sequence, into ``out``; see ``pa_prefill``.
    The workspace is sized for ``T`` query rows (``make_workspace(T, ...)``)."""
    T, Hq, D = q.shape
    N, Hkv, bs, _ = k_cache.shape
    _check(library().pa_prefill(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        _ptr(query_start), block_tables.shape[0], T, Hq, Hkv, D, bs, block_tables.shape[1], N,
        int(max_context_len), float(scale), int(partition_size), _dtype_code(q),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(err_flag),
        _stream(stream)), "pa_prefill")
    return out


def decode_noalloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                   v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
                   *, scale: float, max_context_len: int, partition_size: int = 0,
                   err_flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``decode`` for callers that cannot allocate device memory: the scratch
    comes from the library's fixed array (``NOALLOC_SCRATCH_BYTES``), shared by
    every call; see ``pa_decode_noalloc``."""
    S, Hq, D = q.shape
    N, Hkv, bs, _ = k_cache.shape
    _check(library().pa_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        S, Hq, Hkv, D, bs, block_tables.shape[1], N, int(max_context_len), float(scale),
        int(partition_size), _dtype_code(q), _ptr(err_flag), _stream(stream)), "pa_decode_noalloc")
    return out


# ---------------------------------------------------------------------------
# cache maintenance
# ---------------------------------------------------------------------------
def reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                      err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """Write ``key``/``value`` ``[T][Hkv][D]`` into the cache slots of ``slot_mapping``."""
    T = key.shape[0]
    N, Hkv, bs, D = k_cache.shape
    _check(library().pa_reshape_and_cache(
        _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D, bs, N,
        _dtype_code(k_cache), _ptr(err_flag), _stream(stream)), "pa_reshape_and_cache")


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_mapping: torch.Tensor,
                err_flag: Optional[torch.Tensor] = None, stream=None) -> None:
    """Copy whole blocks ``src -> dst`` for each row of ``block_mapping`` ``[M][2]``."""
    N, Hkv, bs, D = k_cache.shape
    _check(library().pa_copy_blocks(
        _ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), block_mapping.shape[0], Hkv, D, bs, N,
        _dtype_code(k_cache), _ptr(err_flag), _stream(stream)), "pa_copy_blocks")


# ---------------------------------------------------------------------------
# prefix-deduplicated decode
# ---------------------------------------------------------------------------
@dataclass
class SharedPrefixGroups:
    """Groups of sequences that share their leading blocks (``pa_shared_prefix_plan``):
    group g's members are ``seqs[start[g]:start[g+1]]`` and share ``blocks[g]`` blocks."""
    seqs: np.ndarray
    start: np.ndarray
    blocks: np.ndarray

    @property
    def num_groups(self) -> int:
        return len(self.blocks)

    @property
    def num_listed(self) -> int:
        return len(self.seqs)

    def to(self, device="cuda"):
        """(seqs, start, blocks) as int32 device tensors."""
        return tuple(torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
                     for a in (self.seqs, self.start, self.blocks))


def shared_prefix_plan(block_tables: np.ndarray, context_lens: np.ndarray,
                       min_shared_blocks: int = 1, tree: bool = False) -> SharedPrefixGroups:
    """Find the groups on the host (the library's planner; no device needed):
    one group per first block, or with ``tree`` groups chosen on the trie of
    block paths (``pa_shared_prefix_plan_tree``)."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cl = np.ascontiguousarray(context_lens, dtype=np.int32)
    S = int(cl.shape[0])
    if bt.ndim != 2 or bt.shape[0] != S:
        raise ValueError("block_tables must be [num_seqs][max_blocks_per_seq]")
    seqs = np.zeros(max(S, 1), dtype=np.int32)
    start = np.zeros(S + 1, dtype=np.int32)
    blocks = np.zeros(max(S, 1), dtype=np.int32)
    ng, nl = ctypes.c_int(0), ctypes.c_int(0)
    vp = ctypes.c_void_p
    fn = "pa_shared_prefix_plan_tree" if tree else "pa_shared_prefix_plan"
    _check(getattr(library(), fn)(
        vp(bt.ctypes.data), vp(cl.ctypes.data), S, int(bt.shape[1]), 16, int(min_shared_blocks),
        vp(seqs.ctypes.data), vp(start.ctypes.data), vp(blocks.ctypes.data), ctypes.byref(ng),
        ctypes.byref(nl)), fn)
    return SharedPrefixGroups(seqs[:nl.value].copy(), start[:ng.value + 1].copy(),
                              blocks[:ng.value].copy())


def shared_prefix_workspace_size(num_seqs: int, num_listed: int, num_q_heads: int,
                                 num_kv_heads: int, head_dim: int, max_blocks_per_seq: int,
                                 max_context_len: int, partition_size: int = 0,
                                 dtype: torch.dtype = torch.bfloat16) -> int:
    out = ctypes.c_size_t(0)
    _check(library().pa_shared_prefix_workspace_size(
        num_seqs, num_listed, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
        int(max_context_len), int(partition_size),
        PA_BF16 if dtype == torch.bfloat16 else PA_F32, ctypes.byref(out)),
        "pa_shared_prefix_workspace_size")
    return int(out.value)


def make_shared_prefix_workspace(num_seqs: int, num_listed: int, num_q_heads: int,
                                 num_kv_heads: int, head_dim: int, max_blocks_per_seq: int,
                                 max_context_len: int, partition_size: int = 0,
                                 dtype: torch.dtype = torch.bfloat16, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of the size ``pa_decode_shared_prefix`` needs."""
    n = shared_prefix_workspace_size(num_seqs, num_listed, num_q_heads, num_kv_heads, head_dim,
                                     max_blocks_per_seq, max_context_len, partition_size, dtype)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def decode_shared_prefix(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor,
                         v_cache: torch.Tensor, block_tables: torch.Tensor,
                         context_lens: torch.Tensor, groups, *, scale: float,
                         max_context_len: int, workspace: torch.Tensor,
                         key: Optional[torch.Tensor] = None, value: Optional[torch.Tensor] = None,
                         partition_size: int = 0, err_flag: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """Decode that reads each group's shared blocks once; ``groups`` is the
    (seqs, start, blocks) device triple of :meth:`SharedPrefixGroups.to`.  With
    ``key``/``value`` the newest rows are also written, as in :func:`decode_append`."""
    seqs, start, blocks = groups
    S, Hq, D = q.shape
    N, Hkv, bs, _ = k_cache.shape
    _check(library().pa_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), _ptr(context_lens), _ptr(seqs), _ptr(start), _ptr(blocks),
        int(blocks.numel()), int(seqs.numel()), S, Hq, Hkv, D, bs, block_tables.shape[1], N,
        int(max_context_len), float(scale), int(partition_size), _dtype_code(q), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(err_flag), _stream(stream)),
        "pa_decode_shared_prefix")
    return out
