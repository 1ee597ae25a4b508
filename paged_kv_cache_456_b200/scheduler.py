"""Host-side block manager and continuous-batching step simulator.

The serving loop around the decode path, simulated on the CPU so that the GPU
operations can be driven with real block tables, slot mappings and
copy-on-write pairs:

* Requests arrive over time, wait in a queue, and are admitted while the
  pool has room for them; the batch is decided anew at every step, so a
  finished request leaves at once and a waiting one takes its place
  (day-9 post, section "Idea 2: continuous batching"; "What vLLM Is and Why
  It Exists", section "What grew around it").
* A running request gains one token per step ("What vLLM Is and Why It
  Exists", section "A picture"), taking a new block only when its last one is
  full ("What vLLM Is and Why It Exists", section "The idea vLLM started
  from: pages").
* When the pool runs dry, the most recently admitted request is preempted:
  its blocks are freed and it goes back to the front of the queue, to be
  admitted again later with all of its tokens recomputed ("What vLLM Is and
  Why It Exists", section "Why read its source": a request's blocks taken
  away to serve another).
* Requests may share a system prompt: their tables share its blocks, and a
  shared block that one of them must write into is copied first
  (copy-on-write; day-9 post, "Idea 1", bullets "Sharing" and
  "Copy-on-write").

Two admission policies are simulated on the same arrivals: ``"paged"``
(blocks on demand) and ``"reserve"`` (every request holds blocks for
``max_tokens`` tokens from admission on, the pre-paging baseline), so the
concurrency each reaches can be compared.

The simulator only does bookkeeping.  Each step it returns a ``StepPlan``:
the copy pairs, the prefill slot writes of newly admitted requests, and the
decode batch (tables, lengths, the slot of each request's new token).
"""
from __future__ import annotations

import dataclasses
from collections import deque
from typing import Deque, Dict, Iterable, List, Optional, Tuple

import numpy as np

from .block_allocator import BlockAllocator, OutOfBlocks


@dataclasses.dataclass
class Request:
    rid: int
    arrival: int            # step at which it joins the queue
    prompt_len: int         # tokens of its prompt (the shared prefix included)
    output_len: int         # tokens it will generate
    shared_prefix: bool = False
    # state
    table: List[int] = dataclasses.field(default_factory=list)
    n_tokens: int = 0       # tokens whose K/V is in the cache
    generated: int = 0
    admitted_at: int = -1
    preemptions: int = 0

    @property
    def done(self) -> bool:
        return self.generated >= self.output_len


@dataclasses.dataclass
class StepPlan:
    step: int
    copies: List[Tuple[int, int]]                 # (src, dst) block pairs, applied first
    prefill: List[Tuple[int, List[int], List[int]]]  # (rid, token positions, slots)
    rids: List[int]                               # the decode batch
    context_lens: np.ndarray                      # int32 [B], the new token included
    block_tables: np.ndarray                      # int32 [B][Tmax], -1 padded
    new_slots: np.ndarray                         # int64 [B], slot of each new token
    finished: List[int]                           # rids that finish with this step


@dataclasses.dataclass
class SimStats:
    steps: int = 0
    tokens_generated: int = 0
    finished: int = 0
    preemptions: int = 0
    batch_sizes: List[int] = dataclasses.field(default_factory=list)
    slots_held: List[int] = dataclasses.field(default_factory=list)
    tokens_stored: List[int] = dataclasses.field(default_factory=list)

    @property
    def mean_batch(self) -> float:
        return float(np.mean(self.batch_sizes)) if self.batch_sizes else 0.0

    @property
    def waste_fraction(self) -> float:
        held = float(np.sum(self.slots_held))
        return (held - float(np.sum(self.tokens_stored))) / held if held else 0.0


class ServingSimulator:
    """Continuous batching over one pool of ``num_blocks`` blocks.

    ``arrivals``: ``(step, prompt_len, output_len, shared_prefix)`` tuples.
    ``prefix_len`` tokens of system prompt are shared by every request that
    has ``shared_prefix`` set.  ``max_batch`` bounds the decode batch.
    """

    def __init__(self, num_blocks: int, arrivals: Iterable[Tuple[int, int, int, bool]], *,
                 block_size: int = 16, max_batch: int = 256, max_tokens: int = 4096,
                 policy: str = "paged", prefix_len: int = 0,
                 rng: Optional[np.random.Generator] = None):
        if policy not in ("paged", "reserve"):
            raise ValueError("policy must be 'paged' or 'reserve'")
        self.alloc = BlockAllocator(num_blocks, block_size, rng)
        self.bs = block_size
        self.max_batch = max_batch
        self.max_tokens = max_tokens
        self.policy = policy
        self.step_no = 0
        # a request never holds more than max_tokens tokens (prompt + output)
        reqs = []
        for i, (a, p, o, sh) in enumerate(arrivals):
            p = max(1, min(int(p), max_tokens - 1))
            reqs.append(Request(i, int(a), p, max(1, min(int(o), max_tokens - p)), bool(sh)))
        self.pending: List[Request] = sorted(reqs, key=lambda r: (r.arrival, r.rid))
        self.waiting: Deque[Request] = deque()
        self.running: List[Request] = []          # in admission order
        self.reserved: Dict[int, List[int]] = {}  # "reserve" policy: blocks held beyond the table
        self.stats = SimStats()
        self.prefix_len = prefix_len
        self.prefix_table: List[int] = (self.alloc.allocate(prefix_len) if prefix_len else [])

    # -- helpers -----------------------------------------------------------
    def prefix_slots(self) -> List[int]:
        """Slots of the shared system prompt's tokens, positions 0, 1, ..."""
        return [self.alloc.slot_of(self.prefix_table, i) for i in range(self.prefix_len)]

    def tables(self) -> List[List[int]]:
        t = [r.table for r in self.running] + list(self.reserved.values())
        if self.prefix_table:
            t.append(self.prefix_table)
        return t

    def _release(self, r: Request) -> None:
        self.alloc.free(r.table)
        r.table = []
        if r.rid in self.reserved:
            self.alloc.free(self.reserved.pop(r.rid))

    def _preempt_newest(self) -> bool:
        """Free the most recently admitted request; False if none is left."""
        if not self.running:
            return False
        victim = self.running.pop()
        self._release(victim)
        victim.n_tokens = 0
        victim.generated = 0           # recomputed from scratch when re-admitted
        victim.preemptions += 1
        self.stats.preemptions += 1
        self.waiting.appendleft(victim)
        return True

    def _prefill(self, r: Request, copies: List[Tuple[int, int]]) -> Tuple[List[int], List[int]]:
        """Admit ``r``: place its prompt in the pool (sharing the system prompt
        when it has one).  Returns the positions and slots its prefill writes."""
        shared = r.shared_prefix and self.prefix_len > 0 and r.prompt_len >= self.prefix_len
        start = 0
        if shared:
            r.table = self.alloc.fork(self.prefix_table)
            start = self.prefix_len
        else:
            r.table = []
        positions, slots = [], []
        try:
            for pos in range(start, r.prompt_len):
                slots.append(self.alloc.append_token(r.table, pos))
                positions.append(pos)
        except OutOfBlocks:
            self.alloc.pending_copies.clear()
            self.alloc.free(r.table)
            r.table = []
            raise
        copies.extend(self.alloc.pending_copies)
        self.alloc.pending_copies.clear()
        r.n_tokens = r.prompt_len
        return positions, slots

    def _fits(self, r: Request) -> bool:
        if self.policy == "reserve":
            need = self.alloc.blocks_for(self.max_tokens)
        else:
            own = r.prompt_len - (self.prefix_len if r.shared_prefix and self.prefix_len else 0)
            need = self.alloc.blocks_for(max(own, 0)) + 2   # + its first decode block, + one CoW
        return need <= self.alloc.num_free

    # -- one step ------------------------------------------------------------
    def step(self) -> Optional[StepPlan]:
        """Advance one decode step; None once every request has finished."""
        s = self.step_no
        while self.pending and self.pending[0].arrival <= s:
            self.waiting.append(self.pending.pop(0))
        if not (self.pending or self.waiting or self.running):
            return None

        copies: List[Tuple[int, int]] = []
        # 1. every running request gains a token (oldest first); when the pool
        #    runs dry the newest request gives its blocks back
        grown: Dict[int, int] = {}
        i = 0
        while i < len(self.running):
            r = self.running[i]
            if (self.policy == "reserve" and r.n_tokens % self.bs == 0
                    and self.reserved.get(r.rid)):
                # a reserving request grows into its own reservation
                self.alloc.free([self.reserved[r.rid].pop()])
            try:
                grown[r.rid] = self.alloc.append_token(r.table, r.n_tokens)
                copies.extend(self.alloc.pending_copies)
                self.alloc.pending_copies.clear()
                i += 1
            except OutOfBlocks:
                self.alloc.pending_copies.clear()
                victim = self.running[-1]
                grown.pop(victim.rid, None)
                self._preempt_newest()
                if victim is r:
                    continue            # r itself left; the next request is now at i
        # 2. admit waiting requests while they fit
        prefill = []
        while self.waiting and len(self.running) < self.max_batch and self._fits(self.waiting[0]):
            r = self.waiting[0]
            n_copies = len(copies)
            try:
                positions, slots = self._prefill(r, copies)
                grown[r.rid] = self.alloc.append_token(r.table, r.n_tokens)
                copies.extend(self.alloc.pending_copies)
                self.alloc.pending_copies.clear()
            except OutOfBlocks:
                self.alloc.pending_copies.clear()
                del copies[n_copies:]
                if r.table:
                    self.alloc.free(r.table)
                    r.table = []
                break
            self.waiting.popleft()
            if self.policy == "reserve":
                extra = self.alloc.blocks_for(self.max_tokens) - len(r.table)
                self.reserved[r.rid] = self.alloc.allocate(max(0, extra) * self.bs)
            r.admitted_at = s
            self.running.append(r)
            prefill.append((r.rid, positions, slots))

        # 3. the decode batch: every running request with its new token
        B = len(self.running)
        tmax = max([len(r.table) for r in self.running] + [1])
        tables = np.full((B, tmax), -1, dtype=np.int32)
        lens = np.zeros(B, dtype=np.int32)
        new_slots = np.zeros(B, dtype=np.int64)
        for b, r in enumerate(self.running):
            r.n_tokens += 1
            r.generated += 1
            tables[b, :len(r.table)] = r.table
            lens[b] = r.n_tokens
            new_slots[b] = grown[r.rid]
        finished = [r.rid for r in self.running if r.done]
        # keep the copies whose target a running request still holds (a
        # preempted request's targets went back to the pool), one per target
        live = {b for r in self.running for b in r.table}
        by_dst = {}
        for src, dst in copies:
            if dst in live:
                by_dst[dst] = (src, dst)
        copies = list(by_dst.values())
        plan = StepPlan(step=s, copies=copies, prefill=prefill,
                        rids=[r.rid for r in self.running], context_lens=lens,
                        block_tables=tables, new_slots=new_slots, finished=finished)

        # statistics, then retire the finished requests
        st = self.stats
        st.steps += 1
        st.tokens_generated += B
        st.batch_sizes.append(B)
        held = sum(len(r.table) for r in self.running) * self.bs
        st.slots_held.append(held + sum(len(t) for t in self.reserved.values()) * self.bs)
        st.tokens_stored.append(int(lens.sum()))
        for r in [r for r in self.running if r.done]:
            self._release(r)
            st.finished += 1
        self.running = [r for r in self.running if not r.done]
        self.step_no += 1
        return plan

    def run(self, max_steps: int = 1_000_000) -> SimStats:
        for _ in range(max_steps):
            if self.step() is None:
                break
        return self.stats


def poisson_arrivals(rng: np.random.Generator, count: int, rate: float, *,
                     prompt_mean: float = 400.0, output_mean: float = 100.0,
                     max_tokens: int = 4096, shared_fraction: float = 0.0):
    """``count`` requests arriving at ``rate`` per step (Poisson), with prompt
    lengths ``min(max_tokens - 1, 100 + floor(Exp(prompt_mean)))`` -- the
    skewed mix of the pages' capacity measurement -- and output lengths
    ``1 + floor(Exp(output_mean))``."""
    gaps = rng.exponential(1.0 / rate, size=count)
    steps = np.floor(np.cumsum(gaps)).astype(np.int64)
    prompts = np.minimum(max_tokens - 1, 100 + np.floor(rng.exponential(prompt_mean, count)))
    outputs = 1 + np.floor(rng.exponential(output_mean, count))
    shared = rng.random(count) < shared_fraction
    return [(int(a), int(p), int(o), bool(sh))
            for a, p, o, sh in zip(steps, prompts.astype(np.int64), outputs.astype(np.int64), shared)]
