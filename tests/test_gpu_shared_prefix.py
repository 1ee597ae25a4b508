"""Prefix-deduplicated decode (pa_decode_shared_prefix) on the GPU against
the oracle.

Its result is defined as ordinary paged attention -- sharing blocks changes
where the bytes are read, not what is computed -- so the reference is the
oracle's paged decode (with the step's copy-on-write copies and slot write
applied first).  Covered: every head group and head size, groups wider than
one CTA's 64 columns, shared prefixes longer than one 32-block range (the
fold of ranges), copy-on-write, the fused slot write, several groups beside
unshared sequences, plans that do not match the tables (the bad entries are
ignored and the output stays exact), a bad block id inside a shared prefix,
repeat calls on one workspace, and the full prefix_cow workload.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_456_b200 import ops
from paged_kv_cache_456_b200.workloads import build_workload, make_workload, upload

from tests.test_gpu_parity import assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_456_b200 import build
    build.build()
    ops.library()


def prefix_workload(seed, *, G, D, S, prefix, suffix_mean=40.0, cow=0, new_token=False, hkv=2):
    rng = np.random.default_rng(seed)
    # (at least one token after the prefix: the new one goes there)
    lens = prefix + 1 + np.floor(rng.exponential(suffix_mean, S)).astype(np.int64)
    blocks = int(sum(-(-lens // 16))) + cow + 4
    return make_workload(rng, name="prefix", dtype="bf16", num_q_heads=hkv * G, num_kv_heads=hkv,
                         head_dim=D, context_lens=lens, num_blocks=blocks, prefix_tokens=prefix,
                         cow_count=cow, new_token=new_token)


def run_shared(w, groups=None, *, fused=False, t=None, ws=None, err=None):
    """The workload's step with deduplicated decode: copies, slot write (or the
    fused one), attention."""
    t = t if t is not None else upload(w)
    err = err if err is not None else torch.zeros(1, dtype=torch.int32, device="cuda")
    if "block_mapping" in t:
        ops.copy_blocks(t["k_cache"], t["v_cache"], t["block_mapping"], err_flag=err)
    if "key" in t and not fused:
        ops.reshape_and_cache(t["key"], t["value"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                              err_flag=err)
    if groups is None:
        groups = ops.shared_prefix_plan(w.block_tables, w.context_lens)
    if ws is None:
        ws = ops.make_shared_prefix_workspace(w.num_seqs, groups.num_listed, w.num_q_heads,
                                              w.num_kv_heads, w.head_dim, w.max_blocks_per_seq,
                                              w.max_context_len, w.partition_size)
    ops.decode_shared_prefix(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                             t["context_lens"], groups.to(), scale=w.scale,
                             max_context_len=w.max_context_len, workspace=ws,
                             key=t["key_seq"] if fused else None,
                             value=t["value_seq"] if fused else None,
                             partition_size=w.partition_size, err_flag=err)
    torch.cuda.synchronize()
    return t, int(err.item()), ws


def reference(w):
    out, k, v, e = oracle.workload_step(w)
    return out, k, v, e


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_matches_oracle(G, D):
    w = prefix_workload(G * 10 + D, G=G, D=D, S=10, prefix=160)
    plan = ops.shared_prefix_plan(w.block_tables, w.context_lens)
    assert plan.num_groups == 1 and plan.num_listed == 10 and plan.blocks[0] >= 9
    t, err, _ = run_shared(w, plan)
    ref, _, _, e = reference(w)
    assert err == 0 and e == 0
    assert_attention_close(t["out"], ref, "bf16", f"G={G} D={D}")


@pytest.mark.parametrize("G,S,prefix", [(1, 70, 1200), (8, 9, 560), (4, 33, 2048), (2, 3, 16)])
def test_wide_groups_and_long_prefixes(G, S, prefix):
    # 70 x 1 and 9 x 8 columns need two CTAs' worth; 1200 and 2048 tokens
    # span several ranges of shared blocks, combined by the fold; a 16-token prefix
    # is one shared block
    w = prefix_workload(7 + G, G=G, D=128, S=S, prefix=prefix, suffix_mean=30.0)
    t, err, _ = run_shared(w)
    ref, _, _, e = reference(w)
    assert err == 0 and e == 0
    assert_attention_close(t["out"], ref, "bf16", f"G={G} S={S}")


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("G", [4, 8])
def test_copy_on_write_and_slot_write(G, fused):
    w = prefix_workload(31 + G, G=G, D=128, S=16, prefix=256, cow=8, new_token=True)
    t, err, _ = run_shared(w, fused=fused)
    ref, k_ref, v_ref, e = reference(w)
    assert err == 0 and e == 0
    assert_attention_close(t["out"], ref, "bf16", f"fused={fused}")
    idx = torch.from_numpy(w.used_blocks).cuda()
    for dev, host in ((t["k_cache"], k_ref), (t["v_cache"], v_ref)):
        assert np.array_equal(dev[idx].view(torch.int16).cpu().numpy(), host.view(np.int16))


def share(w, dst, src, nblocks):
    """Make sequences dst hold the first nblocks blocks of sequence src."""
    for s in dst:
        assert 16 * nblocks < w.context_lens[s]
        w.tables_compact[s, :nblocks] = w.tables_compact[src, :nblocks]


def mixed_workload(seed=5, G=4):
    rng = np.random.default_rng(seed)
    lens = rng.integers(360, 700, size=24)
    w = make_workload(rng, name="mixed", dtype="bf16", num_q_heads=2 * G, num_kv_heads=2,
                      head_dim=128, context_lens=lens, num_blocks=int(sum(-(-lens // 16))) + 8)
    share(w, range(1, 8), 0, 6)          # family A: 8 sequences, 6 blocks
    share(w, range(9, 16), 8, 10)        # family B: 8 sequences, 10 blocks ...
    share(w, range(13, 16), 8, 20)       # ... of which 4 share 20 (the plan takes 10)
    return w                             # 16..23: nothing shared


def test_several_groups_beside_unshared_sequences():
    w = mixed_workload()
    plan = ops.shared_prefix_plan(w.block_tables, w.context_lens)
    assert [(plan.seqs[plan.start[g]:plan.start[g + 1]].tolist(), int(plan.blocks[g]))
            for g in range(plan.num_groups)] == [(list(range(8)), 6), (list(range(8, 16)), 10)]
    t, err, _ = run_shared(w, plan)
    ref, _, _, e = reference(w)
    assert err == 0 and e == 0
    assert_attention_close(t["out"], ref, "bf16", "mixed")
    # the nested sharing as its own group of 4 gives the same attention
    plan2 = ops.SharedPrefixGroups(np.array([13, 14, 15, 8], np.int32), np.array([0, 4], np.int32),
                                   np.array([20], np.int32))
    t2, err2, _ = run_shared(w, plan2)
    assert err2 == 0
    assert_attention_close(t2["out"], ref, "bf16", "nested")


def groups(seqs, starts, blocks):
    return ops.SharedPrefixGroups(np.array(seqs, np.int32), np.array(starts, np.int32),
                                  np.array(blocks, np.int32))


@pytest.mark.parametrize("case", ["foreign_member", "listed_twice", "too_long_for_member",
                                  "past_the_table", "starts_out_of_order", "member_out_of_range"])
def test_plans_that_do_not_match_are_ignored(case):
    w = mixed_workload(9)
    if case == "too_long_for_member":
        w.context_lens[13] = 16 * 20     # holds the 20 blocks but no token after them
    plan = {
        "foreign_member": groups([0, 1, 2, 20], [0, 4], [6]),        # 20 holds other blocks
        "listed_twice": groups([0, 1, 2, 3, 1, 4], [0, 4, 6], [6, 6]),
        "too_long_for_member": groups([8, 13, 14], [0, 3], [20]),
        "past_the_table": groups([0, 1], [0, 2], [w.max_blocks_per_seq + 1]),
        "starts_out_of_order": groups([0, 1, 2, 3], [0, 3, 2], [6, 6]),
        "member_out_of_range": groups([0, 1, 999, 2], [0, 4], [6]),
    }[case]
    t, err, _ = run_shared(w, plan)
    ref, _, _, e = reference(w)
    assert e == 0
    assert err == ops.ERRBIT_GROUP, err
    assert_attention_close(t["out"], ref, "bf16", case)


def test_bad_block_inside_a_shared_prefix():
    w = mixed_workload(11)
    plan = ops.shared_prefix_plan(w.block_tables, w.context_lens)
    for s in range(8):
        w.tables_compact[s, 3] = -7          # every member of family A
    t, err, _ = run_shared(w, plan)
    ref, _, _, e = reference(w)
    assert e == ops.ERRBIT_BLOCK_ID
    assert err == ops.ERRBIT_BLOCK_ID | ops.ERRBIT_GROUP
    got = t["out"].float().cpu().numpy()
    assert (got[:8] == 0).all()
    assert_attention_close(t["out"][8:], ref[8:], "bf16", "others")


def test_repeat_calls_are_bit_identical():
    w = prefix_workload(3, G=8, D=128, S=12, prefix=1024)
    t, err, ws = run_shared(w)
    first = t["out"].clone()
    for _ in range(2):
        t, err2, ws = run_shared(w, t=t, ws=ws)
        assert err == err2 == 0
        assert torch.equal(first.view(torch.int16), t["out"].view(torch.int16))


def test_workspace_aligned_to_16_bytes_only():
    """The pass stores its partial states 32 bytes at a time when the
    workspace allows it; a workspace that is 16-byte aligned only takes the
    16-byte stores, with the same result."""
    w = prefix_workload(4, G=4, D=128, S=10, prefix=512)
    t, err, ws = run_shared(w)
    first = t["out"].clone()
    off = torch.zeros(ws.numel() + 16, dtype=torch.uint8, device="cuda")[16:]
    assert off.data_ptr() % 32 == 16
    t, err2, _ = run_shared(w, t=t, ws=off)
    assert err == err2 == 0
    assert torch.equal(first.view(torch.int16), t["out"].view(torch.int16))


def test_no_groups_is_plain_decode():
    w = mixed_workload(13)
    empty = groups([], [0], [])
    t, err, _ = run_shared(w, empty)
    ref, _, _, e = reference(w)
    assert err == 0 and e == 0
    assert_attention_close(t["out"], ref, "bf16", "no groups")


def test_full_prefix_cow_workload():
    """The benchmark's deduplicated step: every output element against the
    oracle, every used block bit-exact after the copy-on-write copies."""
    w = build_workload("prefix_cow")     # (copy-on-write copies, then attention)
    t, err, _ = run_shared(w)
    assert err == 0
    ref, k_ref, v_ref, e = reference(w)
    assert e == 0
    idx = torch.from_numpy(w.used_blocks).cuda()
    for dev, host in ((t["k_cache"], k_ref), (t["v_cache"], v_ref)):
        assert np.array_equal(dev[idx].view(torch.int16).cpu().numpy(), host.view(np.int16))
    assert_attention_close(t["out"], ref, "bf16", "prefix_cow (deduplicated, all rows)",
                           record=True, strict_abs=True)


def fork_tree_workload(seed=17, G=4, D=128):
    """Sharing that forms a tree: a 20-block root prompt held by 24 sequences;
    two forks of it hold 12 more blocks each (8 sequences each), and one of
    those forks is forked again for 4 sequences (8 blocks more)."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(16 * 44 + 1, 16 * 44 + 300, size=28)
    w = make_workload(rng, name="tree", dtype="bf16", num_q_heads=2 * G, num_kv_heads=2,
                      head_dim=D, context_lens=lens, num_blocks=int(sum(-(-lens // 16))) + 8)
    share(w, range(1, 24), 0, 20)        # root prompt: sequences 0..23
    share(w, range(1, 8), 0, 32)         # fork A: 0..7 share 32 blocks
    share(w, range(9, 16), 8, 32)        # fork B: 8..15 share 32 blocks
    share(w, range(13, 16), 12, 40)      # fork of B: 12..15 share 40 blocks
    return w                             # 24..27 share nothing


@pytest.mark.parametrize("fused", [False, True])
def test_tree_plan_on_the_device(fused):
    """A plan from pa_shared_prefix_plan_tree (groups at different depths,
    members whose blocks past the group's depth are shared with sibling
    groups) through the pass and the decode continuation, against the oracle
    and against plain decode."""
    w = fork_tree_workload()
    if fused:
        rng = np.random.default_rng(99)
        k_new = rng.standard_normal((w.num_seqs, w.num_kv_heads, w.head_dim), dtype=np.float32)
        v_new = rng.standard_normal((w.num_seqs, w.num_kv_heads, w.head_dim), dtype=np.float32)
    plan = ops.shared_prefix_plan(w.block_tables, w.context_lens, tree=True)
    depths = sorted(int(b) for b in plan.blocks[:plan.num_groups])
    assert len(set(depths)) >= 2, depths          # groups at different depths
    t = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = ops.make_shared_prefix_workspace(w.num_seqs, plan.num_listed, w.num_q_heads,
                                          w.num_kv_heads, w.head_dim, w.max_blocks_per_seq,
                                          w.max_context_len, w.partition_size)
    k_ref, v_ref = w.k_pool.copy(), w.v_pool.copy()
    key = value = None
    if fused:
        # the new token of each sequence (its last position, in a private block)
        from paged_kv_cache_456_b200.workloads import f32_to_bf16_bits
        kb, vb = f32_to_bf16_bits(k_new), f32_to_bf16_bits(v_new)
        key = torch.from_numpy(kb).view(torch.bfloat16).cuda()
        value = torch.from_numpy(vb).view(torch.bfloat16).cuda()
        n = w.context_lens.astype(np.int64)
        slots = w.tables_compact[np.arange(w.num_seqs), (n - 1) // 16].astype(np.int64) * 16 + \
            (n - 1) % 16
        assert oracle.reshape_and_cache(k_ref, v_ref, kb, vb, slots) == 0
    ops.decode_shared_prefix(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                             t["context_lens"], plan.to(), scale=w.scale,
                             max_context_len=w.max_context_len, workspace=ws, key=key,
                             value=value, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref, e = oracle.paged_decode(w.q, k_ref, v_ref, w.tables_compact, w.context_lens,
                                 scale=w.scale, dtype=w.dtype)
    assert e == 0
    assert_attention_close(t["out"], ref, "bf16", f"tree plan fused={fused}")
    # plain decode of the same step agrees within the same bound
    dec = torch.empty_like(t["out"])
    ws2 = ops.make_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                             w.max_context_len, 0, torch.bfloat16)
    ops.decode(dec, t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
               scale=w.scale, max_context_len=w.max_context_len, workspace=ws2, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert_attention_close(dec, ref, "bf16", "plain decode after the tree-plan step")


def test_more_groups_than_the_plan_keeps_on_chip():
    """2049 groups of two sequences that share their first block: more groups
    than the plan kernel keeps on chip (2048), so it reads each group's
    members and blocks from the arrays again where it needs them."""
    S = 2 * 2049
    rng = np.random.default_rng(11)
    lens = 17 + rng.integers(0, 40, size=S)
    w = make_workload(rng, name="pairs", dtype="bf16", num_q_heads=16, num_kv_heads=2,
                      head_dim=128, context_lens=lens, num_blocks=int(sum(-(-lens // 16))) + 4)
    w.tables_compact[1::2, 0] = w.tables_compact[0::2, 0]
    plan = groups(np.arange(S), np.arange(0, S + 1, 2), np.ones(S // 2))
    t, err, _ = run_shared(w, plan)
    ref, _, _, e = reference(w)
    assert err == 0 and e == 0
    assert_attention_close(t["out"], ref, "bf16", "2049 groups of two")
