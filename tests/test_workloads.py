"""Structure of the seeded workloads (CPU only)."""
import numpy as np
import pytest

from paged_kv_cache_456_b200.workloads import (BF16_NAN_BITS, bf16_bits_to_f32, build_workload,
                                              exp_lengths, f32_to_bf16_bits, random_workload)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 1e-3, np.nan], dtype=np.float32)
    b = f32_to_bf16_bits(x)
    y = bf16_bits_to_f32(b)
    assert y[0] == 1.0 and y[1] == 1.0              # tie rounds to even (down)
    assert y[2] == 1.0 + 4 * 2**-8                  # tie rounds to even (up)
    assert y[3] == -2.5 and abs(y[4] - 1e-3) < 1e-5 and np.isnan(y[5])


def test_tiny_layout_and_sentinels():
    w = build_workload("tiny")
    assert list(w.context_lens) == [1, 15, 16, 33]
    assert w.tables_compact.shape == (4, 3)
    assert (w.tables_compact[:3, 1:] == -1).all() and (w.tables_compact[3] >= 0).all()
    assert len(set(w.used_blocks.tolist())) == 6 and w.used_blocks.max() < 16
    # the last token of each sequence waits for the slot write: NaN until then
    for i, slot in enumerate(w.slot_mapping_compact):
        b, off = divmod(int(slot), 16)
        assert np.isnan(w.k_pool[b, :, off]).all() and np.isfinite(w.new_key[i]).all()
    # slots past the end of the last block are NaN for good
    assert np.isnan(w.k_pool[w.tables_compact[3, 2], :, 1:]).all()
    assert np.isnan(w.v_pool[w.tables_compact[1, 0], :, 15:]).all()
    # physical view: the pool the GPU sees
    full = w.materialize_pool("k")
    assert full.shape == (16, 4, 16, 64)
    assert np.array_equal(full[w.block_tables[3, 0]], w.k_pool[w.tables_compact[3, 0]], equal_nan=True)


def test_same_seed_same_inputs():
    a, b = random_workload(3), random_workload(3)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.tables_compact, b.tables_compact)
    assert np.array_equal(a.k_pool.view(np.uint16), b.k_pool.view(np.uint16))


def test_exp_lengths_rule():
    lens = exp_lengths(np.random.default_rng(0), 100000)
    assert lens.min() >= 100 and lens.max() <= 4096
    assert abs(lens.mean() - 499.5) < 5            # 100 + E[floor(Exp(400))], capped
    # the 70B-shaped batch must fit its 40000-block pool
    big = exp_lengths(np.random.default_rng(3), 256)
    assert int(np.sum(-(-big // 16))) < 40000


def test_prefix_cow_structure():
    w = build_workload("prefix_cow")
    assert w.num_seqs == 128 and (w.context_lens >= 2048).all()
    shared = w.block_tables[:, :127]
    assert (shared == shared[0]).all()                      # 127 blocks shared by all
    assert (w.refcount[shared[0]] == 128).all()
    last = w.block_tables[:, 127]
    src = w.block_mapping[:, 0]
    assert w.block_mapping.shape == (64, 2) and len(set(src)) == 1
    assert w.refcount[src[0]] == 64                          # 128 -> 64 after the copies
    assert (last == src[0]).sum() == 64
    assert set(w.block_mapping[:, 1]) == set(last[last != src[0]])
    # copy targets hold NaN until the copy runs
    for c in w.block_mapping_compact[:, 1]:
        assert (w.k_pool[c].view(np.int16) == BF16_NAN_BITS).all()


def test_long_pool_is_exactly_full():
    w = build_workload("long")
    assert w.k_pool.shape[0] == 16384 == w.num_blocks
    assert w.partition_size == 512 and (w.context_lens == 32768).all()
    assert w.decode_bytes() == 8 * 2 * 32768 * 8 * 128 * 2 + 2 * 8 * 32 * 128 * 2


@pytest.mark.parametrize("name", ["7b", "gqa70b"])
def test_lengths_of_the_big_workloads(name):
    # lengths are the first draw of the stream, so they can be checked cheaply
    idx = {"7b": 1, "gqa70b": 2}[name]
    lens = exp_lengths(np.random.default_rng(idx + 1), {"7b": 64, "gqa70b": 256}[name])
    assert lens.min() >= 100 and lens.max() <= 4096


def test_prefill_workload_structure():
    from paged_kv_cache_456_b200.workloads import bf16_bits_to_f32
    w = build_workload("prefill")
    S, T = w.num_seqs, w.q.shape[0]
    assert (np.diff(w.query_start) == 128).all() and w.query_start[-1] == T == 128 * S
    assert w.new_key.shape == (T, w.num_kv_heads, w.head_dim)
    # the chunk's slots are the last 128 positions of each sequence, NaN until written
    for s in (0, S - 1):
        n = int(w.context_lens[s])
        for j in (0, 127):
            r = int(w.query_start[s]) + j
            b, off = divmod(n - 128 + j, 16)
            assert w.slot_mapping_compact[r] == int(w.tables_compact[s, b]) * 16 + off
            assert np.isnan(bf16_bits_to_f32(w.k_pool[int(w.tables_compact[s, b]), :, off])).all()
    assert w.attention_flops() == 4 * w.num_q_heads * w.head_dim * sum(
        128 * (int(n) - 128) + 128 * 129 // 2 for n in w.context_lens)


def test_unique_bytes_count_each_shared_block_once():
    # no sharing: every block has one holder
    for name in ("tiny", "7b"):
        w = build_workload(name)
        assert w.unique_decode_bytes() == w.decode_bytes()
    # prefix_cow: 128 sequences hold the 128 prompt blocks; 64 of them hold
    # a private copy of the last one instead.  Every other holder of a
    # shared block adds 16 rows to the logical count only.
    w = build_workload("prefix_cow")
    row = 2 * w.num_kv_heads * w.head_dim * w.elem_bytes      # K and V of one token
    S, shared, cow = 128, 128, 64
    extra_rows = 16 * ((shared - 1) * (S - 1) + (S - cow - 1))
    assert w.decode_bytes() - w.unique_decode_bytes() == extra_rows * row
