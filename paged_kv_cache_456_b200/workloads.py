"""Seeded synthetic inputs for paged decode attention.

This module builds the inputs that both the CPU oracle and the CUDA path
consume.  It holds none of the attention arithmetic: it draws lengths and
values, lays them out in a paged KV pool through :class:`BlockAllocator`,
and plants NaN sentinels in every slot that no live token owns, so that a
kernel reading a slot it should not read produces NaN.

Workload shapes
---------------
The five named workloads follow one layer of a decode step:

* ``tiny``: 4 sequences of 1, 15, 16 and 33 tokens, 4 query heads = 4 KV
  heads, head size 64, fp32, a 16-block pool, scale 1/8.
* ``7b``: 64 sequences, 32 = 32 heads, head size 128, bf16, 20000-block pool;
  the newest token of every sequence is written by the slot write before
  attention.
* ``gqa70b``: 256 sequences, 64 query / 8 KV heads, head size 128, bf16,
  40000-block pool.
* ``prefix_cow``: 128 sequences share a 2048-token prefix (128 blocks with
  reference count 128) plus private suffixes of floor(Exp(mean 300)) tokens;
  32 / 8 heads, head size 128, bf16, 4096-block pool; 64 of the sequences
  copy-on-write the last shared block before attention.
* ``long``: 8 sequences of 32768 tokens, 32 / 8 heads, head size 128, bf16,
  16384-block pool (exactly full), partition size 512 tokens.

Sequence lengths of ``7b`` and ``gqa70b`` follow the skewed traffic of the
host simulation in "What vLLM Is and Why It Exists" (section "Code"):
``n = min(4096, 100 + floor(X))`` with ``X ~ Exp(mean 400)``.

Draw order (one ``numpy.random.default_rng(seed)`` stream): lengths, pool
permutation (the allocator's free list), copy-on-write choice, q, K pool, V
pool.  q, K and V are N(0, 1) in float32, rounded to bf16 to nearest-even for
bf16 workloads.

Two views of one pool
---------------------
Only the blocks some table or copy pair references hold data.  They are kept
densely in ``k_pool``/``v_pool`` (``[U][Hkv][16][D]``, "compact" ids
``0..U-1``), and ``used_blocks[c]`` gives the physical id of compact block
``c`` in the full pool of ``num_blocks`` blocks that the GPU sees.  Compact
tables and physical tables describe the same tokens; paged attention does not
depend on where a block sits.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

from .block_allocator import BlockAllocator, blocks_for_tokens

BLOCK_SIZE = 16
BF16_NAN_BITS = np.int16(0x7FC0)

WORKLOAD_NAMES = ("tiny", "7b", "gqa70b", "prefix_cow", "long", "prefill")


# ---------------------------------------------------------------------------
# element encodings
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even); returns the 16-bit patterns as int16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    out = ((u + bias) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out.view(np.int16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (int16/uint16) to float32."""
    b = np.ascontiguousarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Values of a stored array as float64 (bf16 patterns widened exactly)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def _cast(x32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x32) if dtype == "bf16" else x32.astype(np.float32)


def _nan_value(dtype: str):
    return BF16_NAN_BITS if dtype == "bf16" else np.float32(np.nan)


# ---------------------------------------------------------------------------
# the workload record
# ---------------------------------------------------------------------------
@dataclasses.dataclass
class Workload:
    name: str
    dtype: str                      # "f32" or "bf16"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int                 # physical pool size the GPU sees
    scale: float
    partition_size: int
    context_lens: np.ndarray        # int32 [S]
    used_blocks: np.ndarray         # int64 [U] physical id of each compact block
    k_pool: np.ndarray              # [U][Hkv][16][D] state before the step
    v_pool: np.ndarray
    tables_compact: np.ndarray      # int32 [S][Tmax], -1 past each sequence's blocks
    q: np.ndarray                   # [S][Hq][D]
    new_key: Optional[np.ndarray] = None         # [T][Hkv][D]
    new_value: Optional[np.ndarray] = None
    slot_mapping_compact: Optional[np.ndarray] = None   # int64 [T]
    block_mapping_compact: Optional[np.ndarray] = None  # int32 [M][2] (src, dst)
    refcount: Optional[np.ndarray] = None        # physical refcounts after the build
    block_size: int = BLOCK_SIZE
    # several query tokens per sequence: q is then [T][Hq][D], the query rows
    # of sequence s are query_start[s] .. query_start[s+1]-1 (its last tokens)
    query_start: Optional[np.ndarray] = None     # int32 [S + 1]

    # -- shapes ------------------------------------------------------------
    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.tables_compact.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    # -- physical view -----------------------------------------------------
    def _phys(self, compact: np.ndarray) -> np.ndarray:
        out = np.where(compact >= 0, self.used_blocks[np.maximum(compact, 0)], -1)
        return out.astype(compact.dtype)

    @property
    def block_tables(self) -> np.ndarray:
        return self._phys(self.tables_compact).astype(np.int32)

    @property
    def slot_mapping(self) -> Optional[np.ndarray]:
        if self.slot_mapping_compact is None:
            return None
        sm = self.slot_mapping_compact
        blk, off = np.divmod(sm, self.block_size)
        phys = np.where(sm >= 0, self.used_blocks[np.maximum(blk, 0)] * self.block_size + off, sm)
        return phys.astype(np.int64)

    @property
    def block_mapping(self) -> Optional[np.ndarray]:
        if self.block_mapping_compact is None:
            return None
        return self.used_blocks[self.block_mapping_compact].astype(np.int32)

    def materialize_pool(self, which: str = "k") -> np.ndarray:
        """The full ``[num_blocks][Hkv][16][D]`` pool on the host (NaN where unused)."""
        src = self.k_pool if which == "k" else self.v_pool
        full = np.full((self.num_blocks,) + src.shape[1:], _nan_value(self.dtype), dtype=src.dtype)
        full[self.used_blocks] = src
        return full

    # -- algorithmic byte counts --------------------------------------------
    def decode_bytes(self) -> int:
        """K and V of every live token (once) plus q read and out written."""
        eb = self.elem_bytes
        kv = int(self.context_lens.astype(np.int64).sum()) * 2 * self.num_kv_heads * self.head_dim * eb
        qo = 2 * self.q.shape[0] * self.num_q_heads * self.head_dim * eb
        return kv + qo

    def unique_decode_bytes(self) -> int:
        """decode_bytes with every physical block counted once however many
        sequences hold it (its live rows: the most any holder uses) -- what a
        decode that reads each shared block once must move."""
        eb = self.elem_bytes
        rows = {}
        for s in range(self.num_seqs):
            n = int(self.context_lens[s])
            for j in range(-(-n // self.block_size)):
                b = int(self.tables_compact[s, j])
                rows[b] = max(rows.get(b, 0), min(self.block_size, n - j * self.block_size))
        kv = sum(rows.values()) * 2 * self.num_kv_heads * self.head_dim * eb
        qo = 2 * self.q.shape[0] * self.num_q_heads * self.head_dim * eb
        return kv + qo

    def attention_flops(self) -> int:
        """2 FLOP per multiply-add of q.K and of p.V, over every attended token."""
        if self.query_start is None:
            attended = int(self.context_lens.astype(np.int64).sum())
        else:
            attended = 0
            for s in range(self.num_seqs):
                n = int(self.context_lens[s])
                Q = int(self.query_start[s + 1] - self.query_start[s])
                attended += Q * (n - Q) + Q * (Q + 1) // 2
        return 4 * attended * self.num_q_heads * self.head_dim

    def reshape_bytes(self) -> int:
        if self.new_key is None:
            return 0
        t = self.new_key.shape[0]
        row = self.num_kv_heads * self.head_dim * self.elem_bytes
        return 4 * t * row + 8 * t   # key+value read, two cache writes, slot ids

    def append_bytes(self) -> int:
        """The slot write when it is fused into decode: the new rows are read
        as part of decode_bytes' live tokens, so only the two cache writes add."""
        if self.new_key is None:
            return 0
        return 2 * self.new_key.shape[0] * self.num_kv_heads * self.head_dim * self.elem_bytes

    def new_rows_per_sequence(self):
        """new_key/new_value as [num_seqs][Hkv][D] (zeros where context_lens
        is 0), the layout of the fused slot write + decode."""
        if self.new_key is None:
            return None, None
        live = np.nonzero(self.context_lens > 0)[0]
        shape = (self.num_seqs, self.num_kv_heads, self.head_dim)
        k = np.zeros(shape, dtype=self.new_key.dtype)
        v = np.zeros(shape, dtype=self.new_value.dtype)
        k[live] = self.new_key
        v[live] = self.new_value
        return k, v

    def copy_bytes(self) -> int:
        if self.block_mapping_compact is None:
            return 0
        m = self.block_mapping_compact.shape[0]
        blk = self.num_kv_heads * self.block_size * self.head_dim * self.elem_bytes
        return 4 * m * blk + 8 * m  # K and V, read and write, plus the pairs


# ---------------------------------------------------------------------------
# builders
# ---------------------------------------------------------------------------
def exp_lengths(rng: np.random.Generator, n: int, mean: float = 400.0,
                base: int = 100, cap: int = 4096) -> np.ndarray:
    """``min(cap, base + floor(Exp(mean)))`` for ``n`` requests."""
    x = rng.exponential(mean, size=n)
    return np.minimum(cap, base + np.floor(x).astype(np.int64)).astype(np.int32)


def make_workload(rng: np.random.Generator, *, name: str, dtype: str,
                  num_q_heads: int, num_kv_heads: int, head_dim: int,
                  context_lens: Sequence[int], num_blocks: int,
                  scale: Optional[float] = None, prefix_tokens: int = 0,
                  cow_count: int = 0, new_token: bool = False,
                  partition_size: int = 0, shuffle: bool = True,
                  max_blocks_per_seq: Optional[int] = None) -> Workload:
    """Lay ``context_lens`` out in a shuffled pool and draw q, K and V.

    ``prefix_tokens`` (a multiple of 16) are shared by every sequence; each
    sequence's own ``context_lens[s]`` counts them.  ``cow_count`` sequences
    then copy-on-write their last prefix block.  With ``new_token`` the last
    token of each sequence is left as NaN in the pool and returned in
    ``new_key``/``new_value`` with its slot, for the slot write to fill.
    """
    if dtype not in ("f32", "bf16"):
        raise ValueError("dtype must be 'f32' or 'bf16'")
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    lens = np.asarray(context_lens, dtype=np.int32)
    S = int(lens.shape[0])
    bs = BLOCK_SIZE
    alloc = BlockAllocator(num_blocks, bs, rng if shuffle else None)

    tables: List[List[int]] = []
    if prefix_tokens:
        if prefix_tokens % bs:
            raise ValueError("prefix_tokens must be a multiple of the block size")
        if (lens < prefix_tokens).any():
            raise ValueError("every sequence must hold the whole prefix")
        if new_token and (lens <= prefix_tokens).any():
            # the new token is written into the sequence's own blocks, never
            # into the shared prefix
            raise ValueError("with new_token every sequence needs a token after the prefix")
        prefix = alloc.allocate(prefix_tokens)
        for s in range(S):
            t = alloc.fork(prefix)
            t += alloc.allocate(int(lens[s]) - prefix_tokens)
            tables.append(t)
        alloc.free(prefix)          # the builder's own reference goes away
    else:
        for s in range(S):
            tables.append(alloc.allocate(int(lens[s])))

    pairs: List[List[int]] = []
    if cow_count:
        if not prefix_tokens:
            raise ValueError("copy-on-write needs a shared prefix")
        last = prefix_tokens // bs - 1
        chosen = np.sort(rng.permutation(S)[:cow_count])
        for s in chosen:
            pair = alloc.cow(tables[int(s)], last)
            if pair is not None:
                pairs.append(list(pair))
    alloc.check_conservation(tables)

    # compact ids in order of first appearance
    order: Dict[int, int] = {}
    for t in tables:
        for b in t:
            order.setdefault(int(b), len(order))
    for src, dst in pairs:
        order.setdefault(int(src), len(order))
        order.setdefault(int(dst), len(order))
    used = np.fromiter(order.keys(), dtype=np.int64, count=len(order))
    U = len(order)

    tmax = max_blocks_per_seq or max(1, max((len(t) for t in tables), default=1))
    tab = np.full((S, tmax), -1, dtype=np.int32)
    for s, t in enumerate(tables):
        tab[s, :len(t)] = [order[int(b)] for b in t]

    # values
    Hkv, D = num_kv_heads, head_dim
    q32 = rng.standard_normal((S, num_q_heads, D), dtype=np.float32)
    k32 = rng.standard_normal((U, Hkv, bs, D), dtype=np.float32)
    v32 = rng.standard_normal((U, Hkv, bs, D), dtype=np.float32)
    q = _cast(q32, dtype)
    k_pool = _cast(k32, dtype)
    v_pool = _cast(v32, dtype)
    del q32, k32, v32
    nanv = _nan_value(dtype)

    # sentinels: slots past each sequence's end in its last block
    for s, t in enumerate(tables):
        n = int(lens[s])
        if n % bs and t:
            c = order[int(t[-1])]
            k_pool[c, :, n % bs:, :] = nanv
            v_pool[c, :, n % bs:, :] = nanv
    # copy-on-write targets hold nothing until the copy
    for _, dst in pairs:
        k_pool[order[dst]] = nanv
        v_pool[order[dst]] = nanv

    new_key = new_value = slot_c = None
    if new_token:
        live = np.nonzero(lens > 0)[0]
        new_key = np.empty((len(live), Hkv, D), dtype=k_pool.dtype)
        new_value = np.empty_like(new_key)
        slot_c = np.empty(len(live), dtype=np.int64)
        for i, s in enumerate(live):
            n = int(lens[s])
            j, off = divmod(n - 1, bs)
            c = int(tab[s, j])
            slot_c[i] = c * bs + off
            new_key[i] = k_pool[c, :, off, :]
            new_value[i] = v_pool[c, :, off, :]
            k_pool[c, :, off, :] = nanv
            v_pool[c, :, off, :] = nanv

    bmap = None
    if pairs:
        bmap = np.array([[order[a], order[b]] for a, b in pairs], dtype=np.int32)

    return Workload(
        name=name, dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=Hkv,
        head_dim=D, num_blocks=num_blocks,
        scale=float(scale if scale is not None else 1.0 / np.sqrt(D)),
        partition_size=partition_size, context_lens=lens, used_blocks=used,
        k_pool=k_pool, v_pool=v_pool, tables_compact=tab, q=q,
        new_key=new_key, new_value=new_value, slot_mapping_compact=slot_c,
        block_mapping_compact=bmap, refcount=alloc.refcount.copy())


def build_workload(name: str, seed: Optional[int] = None,
                   num_blocks: Optional[int] = None) -> Workload:
    """One of the five named workloads (see the module docstring).

    ``num_blocks`` overrides the pool size (the same lengths in a smaller or
    larger shuffled pool; q, K and V are then drawn from a different point of
    the stream), e.g. to keep a profiler's device footprint small."""
    idx = WORKLOAD_NAMES.index(name)
    rng = np.random.default_rng(idx + 1 if seed is None else seed)
    return _build_named(name, rng, num_blocks)


def _build_named(name: str, rng: np.random.Generator, pool: Optional[int]) -> Workload:
    def n(default: int) -> int:
        return default if pool is None else pool

    if name == "tiny":
        return make_workload(rng, name=name, dtype="f32", num_q_heads=4, num_kv_heads=4,
                             head_dim=64, context_lens=[1, 15, 16, 33], num_blocks=n(16),
                             scale=1.0 / 8.0, new_token=True)
    if name == "7b":
        lens = exp_lengths(rng, 64)
        return make_workload(rng, name=name, dtype="bf16", num_q_heads=32, num_kv_heads=32,
                             head_dim=128, context_lens=lens, num_blocks=n(20000), new_token=True)
    if name == "gqa70b":
        lens = exp_lengths(rng, 256)
        return make_workload(rng, name=name, dtype="bf16", num_q_heads=64, num_kv_heads=8,
                             head_dim=128, context_lens=lens, num_blocks=n(40000))
    if name == "prefix_cow":
        suffix = np.floor(rng.exponential(300.0, size=128)).astype(np.int64)
        lens = (2048 + suffix).astype(np.int32)
        return make_workload(rng, name=name, dtype="bf16", num_q_heads=32, num_kv_heads=8,
                             head_dim=128, context_lens=lens, num_blocks=n(4096),
                             prefix_tokens=2048, cow_count=64)
    if name == "prefill":
        prior = exp_lengths(rng, 16)
        return make_prefill_workload(rng, name=name, dtype="bf16", num_q_heads=64,
                                     num_kv_heads=8, head_dim=128, prior_lens=prior, chunk=128,
                                     num_blocks=n(4096))
    if name == "long":
        return make_workload(rng, name=name, dtype="bf16", num_q_heads=32, num_kv_heads=8,
                             head_dim=128, context_lens=[32768] * 8, num_blocks=n(16384),
                             partition_size=512)
    raise KeyError(name)


def make_prefill_workload(rng: np.random.Generator, *, name: str, dtype: str,
                          num_q_heads: int, num_kv_heads: int, head_dim: int,
                          prior_lens: Sequence[int], chunk: int, num_blocks: int) -> Workload:
    """Each sequence holds ``prior_lens[s]`` tokens and takes a chunk of
    ``chunk`` more: the chunk's K/V is returned as new rows with their slots
    (NaN in the pool until the slot write) and its ``chunk`` query rows attend
    causally."""
    prior = np.asarray(prior_lens, dtype=np.int32)
    lens = prior + chunk
    w = make_workload(rng, name=name, dtype=dtype, num_q_heads=num_q_heads,
                      num_kv_heads=num_kv_heads, head_dim=head_dim, context_lens=lens,
                      num_blocks=num_blocks)
    S, T = len(lens), len(lens) * chunk
    qs = (np.arange(S + 1) * chunk).astype(np.int32)
    q32 = rng.standard_normal((T, num_q_heads, head_dim), dtype=np.float32)
    q = _cast(q32, dtype)
    slots = np.empty(T, dtype=np.int64)
    new_key = np.empty((T, num_kv_heads, head_dim), dtype=w.k_pool.dtype)
    new_value = np.empty_like(new_key)
    nanv = _nan_value(dtype)
    for s in range(S):
        for j in range(chunk):
            pos = int(lens[s]) - chunk + j
            b, off = divmod(pos, BLOCK_SIZE)
            c = int(w.tables_compact[s, b])
            r = s * chunk + j
            slots[r] = c * BLOCK_SIZE + off
            new_key[r] = w.k_pool[c, :, off, :]
            new_value[r] = w.v_pool[c, :, off, :]
            w.k_pool[c, :, off, :] = nanv
            w.v_pool[c, :, off, :] = nanv
    return dataclasses.replace(w, q=q, query_start=qs, new_key=new_key, new_value=new_value,
                               slot_mapping_compact=slots)


def random_workload(seed: int, *, dtype: str = "bf16", num_seqs: int = 3,
                    num_q_heads: int = 8, num_kv_heads: int = 2, head_dim: int = 64,
                    max_len: int = 70, lens: Optional[Sequence[int]] = None,
                    spare_blocks: int = 5, new_token: bool = False) -> Workload:
    """A small random case for parity sweeps (lengths uniform in 1..max_len)."""
    rng = np.random.default_rng(seed)
    if lens is None:
        lens = rng.integers(1, max_len + 1, size=num_seqs)
    lens = np.asarray(lens, dtype=np.int32)
    need = int(sum(blocks_for_tokens(int(n)) for n in lens))
    return make_workload(rng, name=f"random{seed}", dtype=dtype, num_q_heads=num_q_heads,
                         num_kv_heads=num_kv_heads, head_dim=head_dim, context_lens=lens,
                         num_blocks=need + spare_blocks, new_token=new_token)


def upload(w: Workload, device="cuda", pool: bool = True):
    """Device tensors for the GPU path: the full NaN-filled pool with the used
    blocks placed at their physical ids, physical tables and slot ids."""
    import torch

    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def elems(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return t.view(torch.bfloat16) if w.dtype == "bf16" else t

    out = {}
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    if pool:
        idx = torch.from_numpy(w.used_blocks).to(device)
        for key, src in (("k_cache", w.k_pool), ("v_cache", w.v_pool)):
            full = torch.full(shape, float("nan"), dtype=tdt, device=device)
            full[idx] = elems(src).to(device)
            out[key] = full
    out["q"] = elems(w.q).to(device)
    if w.query_start is not None:
        out["query_start"] = torch.from_numpy(w.query_start).to(device)
    out["block_tables"] = torch.from_numpy(w.block_tables).to(device)
    out["context_lens"] = torch.from_numpy(w.context_lens).to(device)
    if w.new_key is not None:
        out["key"] = elems(w.new_key).to(device)
        out["value"] = elems(w.new_value).to(device)
        out["slot_mapping"] = torch.from_numpy(w.slot_mapping).to(device)
        if w.query_start is None:
            ks, vs = w.new_rows_per_sequence()
            out["key_seq"] = elems(ks).to(device)
            out["value_seq"] = elems(vs).to(device)
    if w.block_mapping_compact is not None:
        out["block_mapping"] = torch.from_numpy(w.block_mapping).to(device)
    out["out"] = torch.empty((w.q.shape[0], w.num_q_heads, w.head_dim), dtype=tdt, device=device)
    return out
