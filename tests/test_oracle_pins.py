"""Pins of the fp64 oracle against things other than itself (CPU only).

* a library special case: torch's scaled_dot_product_attention (fp64, CPU)
  on the same tokens gathered contiguously;
* hand-derived closed forms (``tests/golden/hand_attention.json``) and the
  one-token / constant-V / zero-query cases;
* invariants the pages state: blocks may sit anywhere (any permutation of
  physical blocks gives the same result), shared prefix blocks give the same
  result as private copies, and the split-K merge equals the one-pass result;
* brute force on tiny inputs (pure Python, ``oracle/brute.py``);
* mutation checks: plausible mistakes planted in a copy of the oracle's C
  source are each caught by at least one of the pins above.
"""
import json
import os
import re
import shutil
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from paged_kv_cache_456_b200.workloads import (build_workload, make_workload, random_workload,
                                              to_f64)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_attention.json")


# ---------------------------------------------------------------------------
# helpers independent of the oracle's own indexing
# ---------------------------------------------------------------------------
def contiguous_kv(w, s):
    """Tokens of sequence s gathered into [Hkv][n][D] fp64 by numpy fancy indexing."""
    n = int(w.context_lens[s])
    nb = -(-n // 16)
    blocks = w.tables_compact[s, :nb]
    k = to_f64(w.k_pool[blocks], w.dtype)            # [nb][Hkv][16][D]
    v = to_f64(w.v_pool[blocks], w.dtype)
    k = k.transpose(1, 0, 2, 3).reshape(w.num_kv_heads, nb * 16, w.head_dim)[:, :n]
    v = v.transpose(1, 0, 2, 3).reshape(w.num_kv_heads, nb * 16, w.head_dim)[:, :n]
    return k, v


def sdpa_reference(w):
    """Library special case: torch SDPA in fp64 over contiguous tokens; query
    head h reads KV head h // (Hq / Hkv) (repeat_interleave)."""
    G = w.num_q_heads // w.num_kv_heads
    q = to_f64(w.q, w.dtype)
    out = np.zeros_like(q)
    for s in range(w.num_seqs):
        if w.context_lens[s] == 0:
            continue
        k, v = contiguous_kv(w, s)
        qt = torch.from_numpy(q[s][None, :, None, :])                    # [1,Hq,1,D]
        kt = torch.from_numpy(k).repeat_interleave(G, dim=0)[None]       # [1,Hq,n,D]
        vt = torch.from_numpy(v).repeat_interleave(G, dim=0)[None]
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=w.scale)
        out[s] = o[0, :, 0, :].numpy()
    return out


def run_oracle(w, partition_size=0, lib=None, k=None, v=None, tables=None):
    return oracle.paged_decode(w.q, w.k_pool if k is None else k, w.v_pool if v is None else v,
                               w.tables_compact if tables is None else tables, w.context_lens,
                               scale=w.scale, dtype=w.dtype, partition_size=partition_size, lib=lib)


def filled(w):
    """A workload whose new tokens are already in the pool (slot write applied)."""
    if w.new_key is None:
        return w
    k, v = w.k_pool.copy(), w.v_pool.copy()
    for i, slot in enumerate(w.slot_mapping_compact):
        b, off = divmod(int(slot), 16)
        k[b, :, off] = w.new_key[i]
        v[b, :, off] = w.new_value[i]
    import dataclasses
    return dataclasses.replace(w, k_pool=k, v_pool=v, new_key=None, new_value=None,
                               slot_mapping_compact=None)


SWEEP = [
    dict(dtype="f32", num_q_heads=4, num_kv_heads=4, head_dim=64),
    dict(dtype="bf16", num_q_heads=8, num_kv_heads=1, head_dim=128),
    dict(dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64),
    dict(dtype="f32", num_q_heads=16, num_kv_heads=2, head_dim=128),
    dict(dtype="bf16", num_q_heads=6, num_kv_heads=3, head_dim=64),
]


# ---------------------------------------------------------------------------
# hand-derived values
# ---------------------------------------------------------------------------
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_golden_hand_cases(case):
    Hkv, D, N = case["num_kv_heads"], case["head_dim"], case["num_blocks"]
    k = np.full((N, Hkv, 16, D), np.nan, dtype=np.float32)
    v = np.full_like(k, np.nan)
    tables = np.array(case["block_tables"], dtype=np.int32)
    for i, (kr, vr) in enumerate(zip(case["tokens"]["k"], case["tokens"]["v"])):
        b = tables[0][i // 16]
        k[b, :, i % 16] = kr
        v[b, :, i % 16] = vr
    out, err = oracle.paged_decode(np.array(case["q"], dtype=np.float32), k, v, tables,
                                   case["context_lens"], scale=case["scale"], dtype="f32")
    assert err == 0
    np.testing.assert_allclose(out, np.array(case["expected"]), rtol=0, atol=case["tol"])


# ---------------------------------------------------------------------------
# library special case
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", SWEEP, ids=lambda s: "{dtype}-G{g}-D{head_dim}".format(
    g=s["num_q_heads"] // s["num_kv_heads"], **s))
@pytest.mark.parametrize("seed", [0, 1])
def test_matches_sdpa_on_contiguous_gather(shape, seed):
    w = random_workload(seed, num_seqs=4, max_len=80, lens=None, **shape)
    out, err = run_oracle(w)
    assert err == 0
    np.testing.assert_allclose(out, sdpa_reference(w), rtol=0, atol=1e-12)


def test_block_edges_match_sdpa():
    lens = [1, 15, 16, 17, 31, 32, 33, 47, 48, 49]
    w = random_workload(5, dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=64, lens=lens)
    out, err = run_oracle(w)
    assert err == 0 and np.isfinite(out).all()      # NaN sentinels never read
    np.testing.assert_allclose(out, sdpa_reference(w), rtol=0, atol=1e-12)


def test_tiny_workload_matches_sdpa_and_brute_force():
    w = filled(build_workload("tiny"))
    out, err = run_oracle(w)
    assert err == 0
    np.testing.assert_allclose(out, sdpa_reference(w), rtol=0, atol=1e-12)
    b = brute.paged_decode(to_f64(w.q, w.dtype).tolist(), to_f64(w.k_pool, w.dtype).tolist(),
                           to_f64(w.v_pool, w.dtype).tolist(), w.tables_compact.tolist(),
                           w.context_lens.tolist(), w.scale)
    np.testing.assert_allclose(out, np.array(b), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_random_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    hkv = int(rng.integers(1, 3))
    w = random_workload(seed, dtype="f32", num_seqs=3, num_q_heads=hkv * int(rng.integers(1, 4)),
                        num_kv_heads=hkv, head_dim=8, max_len=40)
    out, err = run_oracle(w)
    b = brute.paged_decode(to_f64(w.q, w.dtype).tolist(), to_f64(w.k_pool, w.dtype).tolist(),
                           to_f64(w.v_pool, w.dtype).tolist(), w.tables_compact.tolist(),
                           w.context_lens.tolist(), w.scale)
    np.testing.assert_allclose(out, np.array(b), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------
def test_single_token_returns_its_value_exactly():
    w = random_workload(3, dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64, lens=[1, 1, 1])
    out, _ = run_oracle(w)
    G = 4
    for s in range(3):
        b = w.tables_compact[s, 0]
        for h in range(8):
            assert np.array_equal(out[s, h], to_f64(w.v_pool[b, h // G, 0], w.dtype))


def test_constant_value_returns_the_constant():
    w = random_workload(4, dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=64, lens=[5, 40, 77])
    v = np.full_like(w.v_pool, 0.375)
    out, _ = run_oracle(w, v=v)
    np.testing.assert_allclose(out, 0.375, rtol=1e-15, atol=0)


def test_zero_query_returns_the_mean_value():
    w = random_workload(6, dtype="bf16", num_q_heads=4, num_kv_heads=4, head_dim=64, lens=[9, 50])
    w.q[...] = 0
    out, _ = run_oracle(w)
    for s in range(2):
        _, v = contiguous_kv(w, s)
        np.testing.assert_allclose(out[s], v.mean(axis=1), rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_physical_block_permutation_is_invisible(seed):
    w = random_workload(seed, dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64, max_len=90)
    base, _ = run_oracle(w)
    perm = np.random.default_rng(50 + seed).permutation(w.k_pool.shape[0])
    k = np.empty_like(w.k_pool)
    v = np.empty_like(w.v_pool)
    k[perm] = w.k_pool                      # block c moves to slot perm[c]
    v[perm] = w.v_pool
    tables = np.where(w.tables_compact >= 0, perm[np.maximum(w.tables_compact, 0)], -1)
    moved, _ = run_oracle(w, k=k, v=v, tables=tables.astype(np.int32))
    assert np.array_equal(base, moved)


def test_shared_prefix_equals_private_copies():
    rng = np.random.default_rng(9)
    lens = 64 + rng.integers(0, 40, size=5)
    w = make_workload(rng, name="share", dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64,
                      context_lens=lens, num_blocks=200, prefix_tokens=64)
    shared, _ = run_oracle(w)
    # give every sequence its own copy of the 4 prefix blocks
    k, v, tab = [w.k_pool], [w.v_pool], w.tables_compact.copy()
    nxt = w.k_pool.shape[0]
    for s in range(1, w.num_seqs):
        for j in range(4):
            k.append(w.k_pool[tab[s, j]][None])
            v.append(w.v_pool[tab[s, j]][None])
            tab[s, j] = nxt
            nxt += 1
    private, _ = run_oracle(w, k=np.concatenate(k), v=np.concatenate(v), tables=tab)
    assert len(set(w.tables_compact[:, 0])) == 1 and len(set(tab[:, 0])) == w.num_seqs
    assert np.array_equal(shared, private)


@pytest.mark.parametrize("psize", [16, 32, 48, 512, 1 << 20])
def test_split_k_merge_equals_one_pass(psize):
    w = random_workload(11, dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=64,
                        lens=[1, 16, 17, 100, 513, 700])
    one, _ = run_oracle(w)
    split, err = run_oracle(w, partition_size=psize)
    assert err == 0
    np.testing.assert_allclose(split, one, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# error contract
# ---------------------------------------------------------------------------
def test_bad_table_entry_and_bad_length_zero_the_row():
    w = random_workload(12, dtype="f32", num_q_heads=2, num_kv_heads=1, head_dim=64, lens=[20, 20, 20])
    tab = w.tables_compact.copy()
    tab[0, 1] = w.k_pool.shape[0] + 7
    out, err = run_oracle(w, tables=tab)
    assert err == 1 and not out[0].any() and out[1].any()
    lens = w.context_lens.copy()
    lens[2] = 10_000
    out2, err2 = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, lens, scale=w.scale,
                                     dtype="f32", max_context_len=20)
    assert err2 == 2 and not out2[2].any() and out2[1].any()


def test_empty_context_gives_zeros():
    w = random_workload(13, dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=64, lens=[5, 3])
    lens = w.context_lens.copy()
    lens[1] = 0
    out, err = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, lens, scale=w.scale,
                                   dtype="bf16")
    assert err == 0 and not out[1].any() and out[0].any()


# ---------------------------------------------------------------------------
# slot write and block copy
# ---------------------------------------------------------------------------
def test_reshape_and_cache_round_trip_and_untouched_slots():
    w = build_workload("tiny")
    k, v = w.k_pool.copy(), w.v_pool.copy()
    err = oracle.reshape_and_cache(k, v, w.new_key, w.new_value, w.slot_mapping_compact)
    assert err == 0
    for i, slot in enumerate(w.slot_mapping_compact):
        b, off = divmod(int(slot), 16)
        assert np.array_equal(k[b, :, off], w.new_key[i])
        assert np.array_equal(v[b, :, off], w.new_value[i])
    changed = np.zeros(k.shape[:3], dtype=bool)
    for slot in w.slot_mapping_compact:
        changed[int(slot) // 16, :, int(slot) % 16] = True
    kb, k0 = k.view(np.uint32), w.k_pool.view(np.uint32)
    assert np.array_equal(kb[~changed], k0[~changed])   # NaN sentinels keep their bits


def test_reshape_and_cache_skips_padding_and_flags_bad_slots():
    w = build_workload("tiny")
    k, v = w.k_pool.copy(), w.v_pool.copy()
    slots = w.slot_mapping_compact.copy()
    slots[0] = -1
    slots[1] = k.shape[0] * 16
    err = oracle.reshape_and_cache(k, v, w.new_key, w.new_value, slots)
    assert err == 4
    b, off = divmod(int(w.slot_mapping_compact[0]), 16)
    assert np.isnan(k[b, :, off]).all()
    b, off = divmod(int(w.slot_mapping_compact[2]), 16)
    assert np.array_equal(k[b, :, off], w.new_key[2])


def test_copy_blocks_copies_whole_blocks_only():
    w = build_workload("tiny")
    k, v = w.k_pool.copy(), w.v_pool.copy()
    pairs = np.array([[0, 3], [2, 5], [1, 1], [0, 99]], dtype=np.int32)
    err = oracle.copy_blocks(k, v, pairs)
    assert err == 8
    for src, dst in pairs[:2]:
        assert np.array_equal(k[dst].view(np.uint32), w.k_pool[src].view(np.uint32))
        assert np.array_equal(v[dst].view(np.uint32), w.v_pool[src].view(np.uint32))
    for b in (0, 1, 2, 4):
        assert np.array_equal(k[b].view(np.uint32), w.k_pool[b].view(np.uint32))


def test_workload_step_on_prefix_cow_shape():
    rng = np.random.default_rng(21)
    lens = 64 + rng.integers(0, 30, size=6)
    w = make_workload(rng, name="cow", dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=64,
                      context_lens=lens, num_blocks=100, prefix_tokens=64, cow_count=3)
    assert w.block_mapping_compact.shape == (3, 2)
    out, k, v, err = oracle.workload_step(w)
    assert err == 0 and np.isfinite(out).all()
    # without the copies the CoW targets are NaN and so are those rows
    bad, _ = run_oracle(w)
    assert np.isnan(bad).any()


def test_write_into_one_copy_moves_only_its_sequence():
    """After copy-on-write, a slot write into one sequence's private copy of
    the last shared block changes that sequence's output alone; the source
    block and every other row stay bit-identical (day-9 post, "Idea 1",
    copy-on-write)."""
    rng = np.random.default_rng(22)
    lens = 64 + rng.integers(1, 30, size=6)
    w = make_workload(rng, name="cow", dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=64,
                      context_lens=lens, num_blocks=100, prefix_tokens=64, cow_count=3)
    out0, k, v, err = oracle.workload_step(w)
    assert err == 0
    src, dst = (int(x) for x in w.block_mapping_compact[0])
    owners = [s for s in range(w.num_seqs) if dst in w.tables_compact[s]]
    sharers = [s for s in range(w.num_seqs) if src in w.tables_compact[s]]
    assert len(owners) == 1 and len(sharers) >= 1
    src_before = (k[src].copy(), v[src].copy())
    key = rng.standard_normal((1, 2, 64)).astype(np.float32)
    assert oracle.reshape_and_cache(k, v, key, -key, np.array([dst * 16 + 15])) == 0
    out1, e = oracle.paged_decode(w.q, k, v, w.tables_compact, w.context_lens, scale=w.scale,
                                  dtype=w.dtype)
    assert e == 0
    changed = [s for s in range(w.num_seqs) if not np.array_equal(out0[s], out1[s])]
    assert changed == owners
    assert np.array_equal(k[src], src_before[0]) and np.array_equal(v[src], src_before[1])


# ---------------------------------------------------------------------------
# mutation checks: each plausible mistake is caught by a pin
# ---------------------------------------------------------------------------
MUTANTS = {
    "kv_head_modulo": ("const int g = h / group;", "const int g = h % num_kv_heads;"),
    "block_index_swapped": ("table[i / block_size]", "table[i % block_size]"),
    "scale_dropped": ("x[i] = scale * dot;", "x[i] = dot;"),
    "last_token_dropped": ("for (int i = 0; i < n; ++i) {\n                size_t ro",
                           "for (int i = 0; i < n - 1; ++i) {\n                size_t ro"),
    "k_for_v": ("o[d] += w * elem(v_cache", "o[d] += w * elem(k_cache"),
    "max_not_subtracted_sign": ("double w = exp(x[i] - m);", "double w = exp(m - x[i]);"),
}


_MUTANT_RUNNER = """
import sys, numpy as np
sys.path.insert(0, {root!r})
import oracle
from tests.test_oracle_pins import SWEEP, random_workload, run_oracle, sdpa_reference
lib = oracle.load({so!r})
caught = False
for shape in SWEEP[1:3]:
    w = random_workload(0, num_seqs=4, max_len=80, **shape)
    out, _ = run_oracle(w, lib=lib)
    if not np.allclose(out, sdpa_reference(w), rtol=0, atol=1e-9):
        caught = True
print("CAUGHT" if caught else "MISSED")
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    """The mutant runs in a child process: a mutant that reads out of bounds
    and crashes counts as caught."""
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, name
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(old, new, 1))
    so = oracle.build(force=True, src=str(mutated), out=str(tmp_path / "mut.so"))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = _MUTANT_RUNNER.format(root=root, so=so)
    r = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 or "CAUGHT" in r.stdout, f"mutant {name} slipped through the pins"
