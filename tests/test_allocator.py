"""Host block allocator and capacity simulation, pinned to the pages' worked examples."""
import json
import math
import os

import numpy as np
import pytest

from paged_kv_cache_456_b200.block_allocator import (BlockAllocator, ContiguousAllocator,
                                                      OutOfBlocks, blocks_for_tokens)
from paged_kv_cache_456_b200.capacity import compare_policies, skewed_lengths

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_examples.json")


@pytest.fixture(scope="module")
def pages():
    with open(GOLDEN) as f:
        return json.load(f)


def test_blocks_are_ceil_and_waste_at_most_one_block(pages):
    bs = pages["waste_bound"]["block_size"]
    for n in range(0, 4097):
        nb = blocks_for_tokens(n, bs)
        assert nb == math.ceil(n / bs)
        assert 0 <= nb * bs - n <= pages["waste_bound"]["max_wasted_tokens"]


def test_allocate_fork_cow_free_conserve_the_pool():
    rng = np.random.default_rng(0)
    a = BlockAllocator(64, 16, rng)
    t1 = a.allocate(40)                       # 3 blocks
    assert len(t1) == 3 and a.num_free == 61
    t2 = a.fork(t1)
    assert all(a.refcount[b] == 2 for b in t1)
    a.check_conservation([t1, t2])
    pair = a.cow(t2, 2)
    assert pair is not None and pair[0] == t1[2] and pair[1] == t2[2] != t1[2]
    assert a.refcount[t1[2]] == 1 and a.refcount[t2[2]] == 1
    assert a.cow(t2, 2) is None               # already private
    a.check_conservation([t1, t2])
    a.free(t1)
    a.check_conservation([t2])
    a.free(t2)
    assert a.num_free == 64
    with pytest.raises(ValueError):
        a.free(t2)


def test_free_list_is_shuffled_and_blocks_scatter():
    a = BlockAllocator(1000, 16, np.random.default_rng(1))
    t = a.allocate(16 * 50)
    assert len(set(t)) == 50
    assert t != sorted(t)                     # consecutive logical blocks are not adjacent


def test_append_token_takes_a_block_only_when_full_and_cows_shared_tail():
    a = BlockAllocator(8, 16, None)
    t = a.allocate(15)
    slot = a.append_token(t, 15)              # 16th token fits the same block
    assert len(t) == 1 and slot == t[0] * 16 + 15
    slot = a.append_token(t, 16)              # 17th opens a block
    assert len(t) == 2 and slot == t[1] * 16
    u = a.fork(t)
    slot = a.append_token(u, 17)              # shared partial block diverges
    assert a.pending_copies == [(t[1], u[1])] and slot == u[1] * 16 + 1
    a.check_conservation([t, u])


def test_out_of_blocks():
    a = BlockAllocator(2, 16)
    a.allocate(32)
    with pytest.raises(OutOfBlocks):
        a.allocate(1)


def test_fragmentation_example_four_units(pages):
    ex = pages["fragmentation_four_units"]
    cont = ContiguousAllocator(sum(ex["units"].values()))
    for name, size in ex["units"].items():
        cont.allocate(name, size)
    for name in ex["evict"]:
        cont.free(name)
    assert cont.num_free == ex["free_total_after_evict"]
    assert max(s for _, s in cont.free_gaps()) == ex["largest_gap_after_evict"]
    with pytest.raises(OutOfBlocks):
        cont.allocate("new", ex["request"])
    assert not ex["contiguous_fits"]
    # paged: one unit per block, blocks anywhere
    paged = BlockAllocator(sum(ex["units"].values()), 1, None)
    held = {n: paged.allocate(s) for n, s in ex["units"].items()}
    for name in ex["evict"]:
        paged.free(held.pop(name))
    new = paged.allocate(ex["request"])
    assert ex["paged_fits"] and len(new) == ex["request"]
    # the request spans both gaps left by the evicted units
    gap_blocks = [set(range(0, 500)), set(range(1000, 1500))]
    assert all(set(new) & g for g in gap_blocks)


def test_contiguous_slots_example(pages):
    ex = pages["contiguous_slots"]
    cont = ContiguousAllocator(sum(ex["units"].values()))
    paged = BlockAllocator(sum(ex["units"].values()), 1, None)
    held = {}
    for name, size in ex["units"].items():
        cont.allocate(name, size)
        held[name] = paged.allocate(size)
    for name in ex["evict"]:
        cont.free(name)
        paged.free(held.pop(name))
    with pytest.raises(OutOfBlocks):
        cont.allocate("D", ex["request"])
    assert len(paged.allocate(ex["request"])) == ex["request"]


@pytest.mark.parametrize("seed", range(5))
def test_capacity_simulation_matches_the_pages_claims(pages, seed):
    ex = pages["capacity_simulation"]
    lens = skewed_lengths(np.random.default_rng(seed), ex["requests"], cap=ex["max_tokens"])
    r = compare_policies(lens, ex["capacity_tokens"], ex["block_size"], ex["max_tokens"])
    assert r.reserved_fit == ex["reserved_fit_exact"]
    lo, hi = ex["improvement_band"]
    assert lo <= r.improvement <= hi
    lo, hi = ex["waste_band"]
    assert lo <= r.waste_fraction <= hi
    assert r.slots_held <= ex["capacity_tokens"]
    # one more request would not have fit
    nxt = -(-min(int(lens[r.paged_fit]), ex["max_tokens"]) // 16) * 16
    assert r.slots_held + nxt > ex["capacity_tokens"]


def test_try_it_every_request_at_the_maximum(pages):
    ex = pages["try_it_all_max"]
    r = compare_policies([ex["length"]] * 4000, ex["capacity_tokens"], ex["block_size"],
                         ex["max_tokens"])
    assert (r.reserved_fit, r.paged_fit) == (ex["reserved_fit"], ex["paged_fit"])
    assert r.improvement == ex["improvement"] and r.waste_fraction == ex["waste"]


def test_try_it_block_sizes(pages):
    ex = pages["try_it_block_sizes"]
    lens = skewed_lengths(np.random.default_rng(7))
    wastes = [compare_policies(lens, 1 << 20, bs, 4096).waste_fraction for bs in ex["block_sizes"]]
    assert wastes[0] == ex["waste_at_block_size_1"]
    assert all(a < b for a, b in zip(wastes, wastes[1:]))
