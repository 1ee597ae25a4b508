"""The continuous-batching step simulator (host bookkeeping, no GPU)."""
import numpy as np
import pytest

from paged_kv_cache_456_b200.block_allocator import blocks_for_tokens
from paged_kv_cache_456_b200.capacity import compare_policies, skewed_lengths
from paged_kv_cache_456_b200.scheduler import ServingSimulator, poisson_arrivals


def check_plan(sim, plan):
    """Invariants of one step's plan and of the pool after it."""
    sim.alloc.check_conservation(sim.tables())
    for r in sim.running:
        assert len(r.table) == blocks_for_tokens(r.n_tokens, sim.bs)
    B = len(plan.rids)
    assert plan.block_tables.shape[0] == B == plan.context_lens.shape[0] == plan.new_slots.shape[0]
    # the new token of each request sits at position n - 1 of its own table
    for b in range(B):
        n = int(plan.context_lens[b])
        j, off = divmod(n - 1, sim.bs)
        assert plan.new_slots[b] == int(plan.block_tables[b, j]) * sim.bs + off
        assert (plan.block_tables[b, blocks_for_tokens(n, sim.bs):] == -1).all()
    writes = list(plan.new_slots) + [x for _, _, slots in plan.prefill for x in slots]
    assert len(writes) == len(set(writes)), "a slot written twice in one step"
    dsts = [d for _, d in plan.copies]
    assert len(dsts) == len(set(dsts))
    assert not set(dsts) & {s for s, _ in plan.copies}


@pytest.mark.parametrize("prefix_len", [0, 40])
def test_every_request_finishes_and_the_pool_is_conserved(prefix_len):
    rng = np.random.default_rng(3)
    arr = poisson_arrivals(rng, 120, 1.5, prompt_mean=150, output_mean=40,
                           max_tokens=1024, shared_fraction=0.5)
    sim = ServingSimulator(1500, arr, max_tokens=1024, prefix_len=prefix_len,
                           rng=np.random.default_rng(4))
    done = set()
    while True:
        plan = sim.step()
        if plan is None:
            break
        check_plan(sim, plan)
        done |= set(plan.finished)
    assert done == set(range(120))
    assert sim.stats.finished == 120
    want = sum(min(o, 1024 - max(1, min(p, 1023))) for _, p, o, _ in arr)
    assert sim.stats.tokens_generated >= want
    # everything but the system prompt went back to the pool
    assert sim.alloc.num_free == sim.alloc.num_blocks - len(sim.prefix_table)


def test_pressure_preempts_and_still_finishes():
    rng = np.random.default_rng(5)
    arr = poisson_arrivals(rng, 60, 4.0, prompt_mean=300, output_mean=150, max_tokens=2048)
    sim = ServingSimulator(260, arr, max_tokens=2048, rng=np.random.default_rng(6))
    while (plan := sim.step()) is not None:
        check_plan(sim, plan)
    assert sim.stats.preemptions > 0
    assert sim.stats.finished == 60


def test_shared_prompt_blocks_are_shared_and_copied_on_write():
    rng = np.random.default_rng(7)
    arr = [(0, 40 + int(x), 5, True) for x in rng.integers(0, 30, size=8)]
    sim = ServingSimulator(200, arr, prefix_len=40, rng=np.random.default_rng(8))
    plan = sim.step()
    check_plan(sim, plan)
    # 40 tokens: blocks 0, 1 full and shared by all; block 2 partly filled and
    # copied by every request that writes past token 40
    shared = sim.prefix_table
    assert all(sim.alloc.refcount[b] == 9 for b in shared[:2])
    writers = [r for r in sim.running if r.prompt_len > 40 or r.n_tokens > 40]
    srcs = [s for s, _ in plan.copies]
    assert srcs == [shared[2]] * len(writers)
    for r in sim.running:
        assert r.table[:2] == shared[:2] and r.table[2] != shared[2]


def test_reserving_the_maximum_admits_fewer_on_the_pages_mix():
    """All requests of the pages' skewed mix (lengths min(4096, 100 +
    floor(Exp(400)))) arrive at once into a 2^20-token pool: the first decode
    batch under paging is about 8 times the one under reserve-the-maximum,
    as the static count says ("What vLLM Is and Why It Exists", section
    "Code")."""
    lens = skewed_lengths(np.random.default_rng(7), count=4000)
    arr = [(0, int(n), 1, False) for n in lens]
    first = {}
    for policy in ("paged", "reserve"):
        sim = ServingSimulator((1 << 20) // 16, arr, max_batch=5000, policy=policy)
        plan = sim.step()
        first[policy] = len(plan.rids)
    static = compare_policies(lens, 1 << 20, 16, 4096)
    assert first["reserve"] == static.reserved_fit == 256
    assert abs(first["paged"] - static.paged_fit) <= 0.02 * static.paged_fit
    assert 7.5 <= first["paged"] / first["reserve"] <= 8.6


def test_paged_policy_reaches_higher_concurrency():
    rng = np.random.default_rng(9)
    arr = poisson_arrivals(rng, 300, 2.0, prompt_mean=200, output_mean=60, max_tokens=2048)
    stats = {p: ServingSimulator(3000, arr, max_tokens=2048, policy=p,
                                 rng=np.random.default_rng(10)).run() for p in ("paged", "reserve")}
    assert stats["paged"].finished == stats["reserve"].finished == 300
    assert stats["paged"].mean_batch > 1.5 * stats["reserve"].mean_batch
    assert stats["paged"].steps < stats["reserve"].steps
    assert stats["paged"].waste_fraction < 0.05 < stats["reserve"].waste_fraction
