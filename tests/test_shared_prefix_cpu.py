"""Prefix-deduplicated decode, host side (no GPU needed).

pa_shared_prefix_plan runs on the host: sequences whose block tables start
with the same physical block form a candidate group, which shares the
longest run of leading blocks every member holds, capped so that each member
keeps at least one token of its own (the blocks before the one holding its
last token).  Checked against a brute force of that rule written from the
header's statement, and by properties that any correct plan has (members
really share the blocks, the run is maximal, nothing is listed twice).
Then the entry point's host-side argument checks.
"""
import ctypes

import numpy as np
import pytest

from paged_kv_cache_456_b200 import ops
from paged_kv_cache_456_b200.workloads import build_workload


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_456_b200 import build
    build.build()
    return ops.library()


def brute_force_plan(tables, lens, min_blocks=1):
    tmax = tables.shape[1]
    by_first = {}
    for s, n in enumerate(lens):
        if n <= 0 or n > 16 * tmax or (n - 1) // 16 < min_blocks:
            continue
        by_first.setdefault(int(tables[s, 0]), []).append(s)
    groups = []
    for members in by_first.values():
        if len(members) < 2:
            continue
        cap = min((int(lens[s]) - 1) // 16 for s in members)
        run = 0
        while run < cap and all(tables[s, run] == tables[members[0], run] for s in members):
            run += 1
        if run >= min_blocks:
            groups.append((members, run))
    groups.sort(key=lambda g: g[0][0])
    return groups


def as_groups(plan):
    return [(plan.seqs[plan.start[g]:plan.start[g + 1]].tolist(), int(plan.blocks[g]))
            for g in range(plan.num_groups)]


def random_forest(seed, S=40, tmax=24, pool=2000):
    """Tables with forks: some sequences copy a prefix of another's table,
    some of those then diverge (copy-on-write) inside it."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 16 * tmax + 1, size=S).astype(np.int32)
    lens[rng.random(S) < 0.1] = 0
    tables = rng.permutation(pool)[: S * tmax].reshape(S, tmax).astype(np.int32)
    for s in range(1, S):
        if rng.random() < 0.6:
            src = int(rng.integers(0, s))
            k = int(rng.integers(1, tmax))
            tables[s, :k] = tables[src, :k]
            if rng.random() < 0.3:
                tables[s, int(rng.integers(0, k))] = pool + s  # a private copy
    return tables, lens


@pytest.mark.parametrize("seed", range(8))
@pytest.mark.parametrize("min_blocks", [1, 3])
def test_plan_matches_brute_force(lib, seed, min_blocks):
    tables, lens = random_forest(seed)
    plan = ops.shared_prefix_plan(tables, lens, min_blocks)
    assert as_groups(plan) == brute_force_plan(tables, lens, min_blocks)


@pytest.mark.parametrize("seed", range(8))
def test_plan_properties(lib, seed):
    tables, lens = random_forest(100 + seed)
    plan = ops.shared_prefix_plan(tables, lens)
    seen = set()
    for members, P in as_groups(plan):
        assert len(members) >= 2 and P >= 1
        assert members == sorted(members) and not (seen & set(members))
        seen |= set(members)
        lead = tables[members[0]]
        for s in members:
            assert (tables[s, :P] == lead[:P]).all()        # they hold the same blocks
            assert 16 * P <= lens[s] - 1                      # and keep a token of their own
        cap = min((int(lens[s]) - 1) // 16 for s in members)
        assert P == cap or any(tables[s, P] != lead[P] for s in members)   # maximal
    # an eligible sequence left out shares its first block with no other one
    firsts = {}
    for s, n in enumerate(lens):
        if 0 < n <= 16 * tables.shape[1] and (n - 1) // 16 >= 1:
            firsts.setdefault(int(tables[s, 0]), []).append(s)
    for s in set(range(len(lens))) - seen:
        if 0 < lens[s] and (lens[s] - 1) // 16 >= 1:
            assert len(firsts[int(tables[s, 0])]) == 1


def test_plan_of_the_named_workloads(lib):
    w = build_workload("prefix_cow")
    plan = ops.shared_prefix_plan(w.block_tables, w.context_lens)
    # 128 sequences fork a 2048-token prompt; 64 copy its last block on write
    assert as_groups(plan) == [(list(range(128)), 127)]
    for name in ("7b", "gqa70b", "long"):
        w = build_workload(name)
        assert ops.shared_prefix_plan(w.block_tables, w.context_lens).num_groups == 0


def test_plan_edge_cases(lib):
    # one token of its own: a 32-token sequence can share 1 block, a 16-token one none
    t = np.array([[5, 6, 7], [5, 6, 8], [5, 9, 9]], dtype=np.int32)
    assert as_groups(ops.shared_prefix_plan(t, np.array([48, 33, 32], np.int32))) == \
        [([0, 1, 2], 1)]
    assert as_groups(ops.shared_prefix_plan(t, np.array([48, 33, 16], np.int32))) == \
        [([0, 1], 2)]
    assert ops.shared_prefix_plan(t, np.array([0, 0, 0], np.int32)).num_groups == 0
    assert ops.shared_prefix_plan(np.zeros((0, 3), np.int32), np.zeros(0, np.int32)).num_groups == 0
    # lengths past the table are not eligible
    assert ops.shared_prefix_plan(t, np.array([49, 33, 32], np.int32)).num_groups == 1


P = ctypes.c_void_p


def shared_call(lib, **kw):
    a = dict(out=P(16), q=P(16), key=None, value=None, k=P(16), v=P(16), tab=P(16), lens=P(16),
             gs=P(16), gst=P(16), gb=P(16), ng=1, nl=4, S=4, Hq=8, Hkv=2, D=128, bs=16, tmax=8,
             N=64, ctx=128, scale=0.1, ps=0, dt=ops.PA_BF16, ws=P(256), wsb=1 << 30, err=None,
             stream=None)
    a.update(kw)
    return lib.pa_decode_shared_prefix(*a.values())


def test_shared_prefix_decode_rejects_bad_arguments_on_the_host(lib):
    assert shared_call(lib, dt=ops.PA_F32) == ops.PA_ERR_UNSUPPORTED
    assert shared_call(lib, ng=-1) == ops.PA_ERR_INVALID_ARG
    assert shared_call(lib, key=P(16)) == ops.PA_ERR_INVALID_ARG        # key without value
    assert shared_call(lib, bs=32) == ops.PA_ERR_UNSUPPORTED
    assert shared_call(lib, D=96) == ops.PA_ERR_UNSUPPORTED
    assert shared_call(lib, Hq=6) == ops.PA_ERR_UNSUPPORTED               # 3 heads per KV head
    assert shared_call(lib, gs=None) == ops.PA_ERR_INVALID_ARG
    assert shared_call(lib, ng=20000) == ops.PA_ERR_UNSUPPORTED
    assert shared_call(lib, ng=5, nl=4) == ops.PA_ERR_INVALID_ARG          # more groups than listed
    assert shared_call(lib, q=P(8)) == ops.PA_ERR_INVALID_ARG            # misaligned
    assert shared_call(lib, scale=float("nan")) == ops.PA_ERR_INVALID_ARG
    assert shared_call(lib, S=0) == ops.PA_OK                             # nothing to do


def test_plan_rejects_bad_arguments(lib):
    n = ctypes.c_int(0)
    assert lib.pa_shared_prefix_plan(P(16), P(16), 2, 4, 32, 1, P(16), P(16), P(16),
                                     ctypes.byref(n), ctypes.byref(n)) == ops.PA_ERR_UNSUPPORTED
    assert lib.pa_shared_prefix_plan(None, P(16), 2, 4, 16, 1, P(16), P(16), P(16),
                                     ctypes.byref(n), ctypes.byref(n)) == ops.PA_ERR_INVALID_ARG
    assert lib.pa_shared_prefix_plan(P(16), P(16), 2, 4, 16, 1, P(16), P(16), P(16),
                                     None, ctypes.byref(n)) == ops.PA_ERR_INVALID_ARG


def test_workspace_size_rejects_fp32(lib):
    out = ctypes.c_size_t(0)
    assert lib.pa_shared_prefix_workspace_size(4, 4, 8, 2, 128, 8, 128, 0, ops.PA_F32,
                                               ctypes.byref(out)) == ops.PA_ERR_UNSUPPORTED


# ---------------------------------------------------------------------------
# the tree planner (pa_shared_prefix_plan_tree)
# ---------------------------------------------------------------------------
def tree_reference(tables, lens, min_blocks=1):
    """The header's rule on an explicit trie (dicts of children by block id),
    resolved recursively: a different construction from the library's
    sort + common-prefix stack."""
    tmax = tables.shape[1]
    root = {"depth": 0, "kids": {}, "here": []}
    for s, n in enumerate(lens):
        if n <= 0 or n > 16 * tmax or (n - 1) // 16 < min_blocks:
            continue
        node = root
        for j in range((n - 1) // 16):
            node = node["kids"].setdefault(int(tables[s, j]),
                                           {"depth": j + 1, "kids": {}, "here": []})
        node["here"].append(s)
    groups = []

    def walk(node, parent_depth):
        free = list(node["here"])
        for kid in node["kids"].values():
            free += walk(kid, node["depth"])
        # (a chain of single children is one node of the compressed trie:
        # only a node that branches or ends paths decides)
        k, d = len(free), node["depth"]
        decides = len(node["kids"]) != 1 or node["here"]
        if decides and k >= 2 and d >= min_blocks and (k - 1) * d >= k * parent_of[id(node)]:
            groups.append((sorted(free), d))
            return []
        return free

    # the parent depth that matters is that of the nearest deciding ancestor
    parent_of = {}

    def mark(node, deciding_depth):
        decides = len(node["kids"]) != 1 or node["here"]
        parent_of[id(node)] = deciding_depth
        for kid in node["kids"].values():
            mark(kid, node["depth"] if decides else deciding_depth)

    mark(root, 0)
    walk(root, 0)
    groups.sort(key=lambda g: g[0][0])
    return groups


def fork_tree(seed, S=60, tmax=40):
    """Sequences that fork earlier ones at random depths (forks of forks)."""
    rng = np.random.default_rng(seed)
    fresh = iter(range(10**6))
    tables = np.zeros((S, tmax), dtype=np.int32)
    lens = rng.integers(1, 16 * tmax + 1, size=S).astype(np.int32)
    for s in range(S):
        tables[s] = [next(fresh) for _ in range(tmax)]
        if s and rng.random() < 0.85:
            src = int(rng.integers(0, s))
            k = int(rng.integers(1, tmax))
            tables[s, :k] = tables[src, :k]
    return tables, lens


def savings(groups):
    return sum((len(m) - 1) * P for m, P in groups)


@pytest.mark.parametrize("seed", range(12))
def test_tree_plan_matches_its_reference(lib, seed):
    tables, lens = fork_tree(seed)
    plan = ops.shared_prefix_plan(tables, lens, tree=True)
    assert as_groups(plan) == tree_reference(tables, lens)


@pytest.mark.parametrize("seed", range(12))
def test_tree_plan_is_valid_and_saves_at_least_as_much(lib, seed):
    tables, lens = fork_tree(100 + seed)
    tree = as_groups(ops.shared_prefix_plan(tables, lens, tree=True))
    flat = as_groups(ops.shared_prefix_plan(tables, lens))
    seen = set()
    for members, P in tree:
        assert len(members) >= 2 and P >= 1 and members == sorted(members)
        assert not (seen & set(members))
        seen |= set(members)
        for s in members:
            assert (tables[s, :P] == tables[members[0], :P]).all() and 16 * P <= lens[s] - 1
    assert savings(tree) >= savings(flat)


def test_tree_plan_examples(lib):
    t = np.arange(10 * 24, dtype=np.int32).reshape(10, 24)
    lens = np.full(10, 16 * 24, dtype=np.int32)
    t[1:, :10] = t[0, :10]          # ten sequences share 10 blocks
    t[1:2, :11] = t[0, :11]         # two of them share 11: not worth a group of their own
    assert as_groups(ops.shared_prefix_plan(t, lens, tree=True)) == [(list(range(10)), 10)]
    t[1:4, :20] = t[0, :20]         # four share 20: (4-1)*20 >= 4*10, a group of their own
    assert as_groups(ops.shared_prefix_plan(t, lens, tree=True)) == \
        [([0, 1, 2, 3], 20), ([4, 5, 6, 7, 8, 9], 10)]
    w = build_workload("prefix_cow")
    assert as_groups(ops.shared_prefix_plan(w.block_tables, w.context_lens, tree=True)) == \
        [(list(range(128)), 127)]
    # different first blocks never share
    u = np.arange(4 * 8, dtype=np.int32).reshape(4, 8)
    assert ops.shared_prefix_plan(u, np.full(4, 100, np.int32), tree=True).num_groups == 0
