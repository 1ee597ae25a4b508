"""Parity of the CUDA path (called through the C ABI) with the fp64 oracle.

Tolerances: the slot write and block copy must be bit-exact; attention must
satisfy max |gpu - ref| <= 1e-5 for fp32 caches, and
|gpu - ref| <= 1e-2 + 1e-2 |ref| element-wise for bf16 caches (fp32
accumulation, output rounded once to bf16).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_456_b200 import ops
from paged_kv_cache_456_b200.workloads import (build_workload, make_workload, random_workload,
                                              to_f64, upload)

pytestmark = pytest.mark.gpu

F32_ATOL = 1e-5
BF16_ATOL = BF16_RTOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_456_b200 import build
    build.build()
    ops.library()


def assert_attention_close(gpu, ref, dtype, what="", record=False, strict_abs=False):
    """The stated tolerance, element by element.  ``strict_abs`` also holds
    bf16 results to max |gpu - ref| <= 1e-2 (the bound read as purely
    absolute); ``record`` adds the margins to the end-of-run summary."""
    g = gpu.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ref.shape, f"{what}: shape {g.shape} vs {ref.shape}"
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    max_abs = float(err.max()) if err.size else 0.0
    if dtype == "f32":
        worst = max_abs / F32_ATOL
    else:
        worst = float((err / (BF16_ATOL + BF16_RTOL * np.abs(ref))).max()) if err.size else 0.0
    if record:
        from tests.conftest import PARITY_RECORDS
        PARITY_RECORDS.append((what, int(err.size), max_abs, worst))
    if dtype == "f32":
        assert max_abs <= F32_ATOL, f"{what}: max abs err {max_abs:.3e}"
    else:
        assert worst <= 1.0, f"{what}: max abs err {max_abs:.3e}, worst err/bound {worst:.3f}"
        if strict_abs:
            assert max_abs <= BF16_ATOL, f"{what}: max abs err {max_abs:.3e} > {BF16_ATOL}"


def run_gpu(w, partition_size=None, t=None, err=None):
    """copy-on-write copies, slot write, decode: the workload's step on the GPU."""
    t = t if t is not None else upload(w)
    err = err if err is not None else torch.zeros(1, dtype=torch.int32, device="cuda")
    ps = w.partition_size if partition_size is None else partition_size
    if "block_mapping" in t:
        ops.copy_blocks(t["k_cache"], t["v_cache"], t["block_mapping"], err_flag=err)
    if "key" in t:
        ops.reshape_and_cache(t["key"], t["value"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                              err_flag=err)
    tdt = t["q"].dtype
    ws = ops.make_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.max_context_len, ps, tdt)
    ops.decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
               scale=w.scale, max_context_len=w.max_context_len, workspace=ws, partition_size=ps,
               err_flag=err)
    torch.cuda.synchronize()
    return t, int(err.item()), ws


def counters_zero(w, ws):
    n = w.num_seqs * w.num_kv_heads
    return bool((ws[: 4 * n].view(torch.int32) == 0).all())


# ---------------------------------------------------------------------------
# the tiny workload, end to end
# ---------------------------------------------------------------------------
def test_tiny_workload_full_step():
    w = build_workload("tiny")
    ref, k_ref, v_ref, oerr = oracle.workload_step(w)
    t, err, ws = run_gpu(w)
    assert err == 0 and oerr == 0
    assert_attention_close(t["out"], ref, w.dtype, "tiny (pa_decode)", record=True)
    # the slot write is bit-exact and leaves every other slot (NaN sentinels too) alone
    kc = t["k_cache"].cpu().numpy()[w.used_blocks]
    vc = t["v_cache"].cpu().numpy()[w.used_blocks]
    assert np.array_equal(kc.view(np.uint32), k_ref.view(np.uint32))
    assert np.array_equal(vc.view(np.uint32), v_ref.view(np.uint32))
    assert counters_zero(w, ws)


# ---------------------------------------------------------------------------
# sweeps of small shapes
# ---------------------------------------------------------------------------
SHAPES = [(dt, D, G) for dt in ("f32", "bf16") for D in (64, 128) for G in (1, 2, 4, 8)]


@pytest.mark.parametrize("dtype,D,G", SHAPES, ids=lambda x: str(x))
@pytest.mark.parametrize("psize", [0, 16, 48, 512])
def test_shapes_and_partitions(dtype, D, G, psize):
    hkv = 2
    lens = [1, 15, 16, 17, 33, 100, 511, 512, 513, 700]
    w = random_workload(1000 + D + G, dtype=dtype, num_q_heads=hkv * G, num_kv_heads=hkv,
                        head_dim=D, lens=lens, spare_blocks=37)
    ref, _ = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                 scale=w.scale, dtype=w.dtype)
    t, err, ws = run_gpu(w, partition_size=psize)
    assert err == 0
    assert_attention_close(t["out"], ref, dtype, f"{dtype} D{D} G{G} P{psize}")
    assert counters_zero(w, ws)


@pytest.mark.parametrize("seed", range(6))
def test_random_batches(seed):
    rng = np.random.default_rng(seed)
    G = int(rng.choice([1, 2, 4, 8]))
    hkv = int(rng.integers(1, 5))
    S = int(rng.integers(1, 40))
    lens = rng.integers(0, 1500, size=S)
    lens[rng.random(S) < 0.1] = 0
    w = make_workload(rng, name="rand", dtype="bf16", num_q_heads=hkv * G, num_kv_heads=hkv,
                      head_dim=int(rng.choice([64, 128])), context_lens=lens,
                      num_blocks=int(sum(-(-lens // 16))) + 50)
    ref, _ = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                 scale=w.scale, dtype=w.dtype)
    t, err, ws = run_gpu(w, partition_size=int(rng.choice([0, 16, 64, 512])))
    assert err == 0
    assert_attention_close(t["out"], ref, "bf16", f"seed {seed}")
    zero_rows = np.nonzero(lens == 0)[0]
    assert (t["out"][torch.as_tensor(zero_rows, device="cuda")] == 0).all()


def test_many_sequences():
    rng = np.random.default_rng(7)
    lens = rng.integers(1, 60, size=3000)
    w = make_workload(rng, name="many", dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=128,
                      context_lens=lens, num_blocks=int(sum(-(-lens // 16))) + 10)
    ref, _ = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                 scale=w.scale, dtype=w.dtype)
    t, err, _ = run_gpu(w)
    assert err == 0
    assert_attention_close(t["out"], ref, "bf16", "3000 sequences")


def test_very_large_batch():
    """12000 short sequences: the per-sequence arrays take most of an SM's
    shared memory, leaving one CTA per SM."""
    rng = np.random.default_rng(8)
    lens = rng.integers(0, 40, size=12000)
    w = make_workload(rng, name="huge", dtype="bf16", num_q_heads=2, num_kv_heads=2, head_dim=64,
                      context_lens=lens, num_blocks=int(sum(-(-lens // 16))) + 10)
    ref, _ = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                 scale=w.scale, dtype=w.dtype)
    t, err, ws = run_gpu(w)
    assert err == 0
    assert_attention_close(t["out"], ref, "bf16", "12000 sequences")
    assert counters_zero(w, ws)


def test_all_empty_and_single_token():
    w = random_workload(5, dtype="f32", num_q_heads=4, num_kv_heads=4, head_dim=64, lens=[1, 1])
    t, err, _ = run_gpu(w)
    out = t["out"].cpu().numpy()
    for s in range(2):
        b = w.tables_compact[s, 0]
        assert np.array_equal(out[s], w.v_pool[b, :, 0])       # n = 1 returns V exactly
    t["context_lens"].zero_()
    t["out"].fill_(7.0)
    ws = ops.make_workspace(2, 4, 4, 64, 1, 0, torch.float32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
               scale=w.scale, max_context_len=1, workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0 and (t["out"] == 0).all()


# ---------------------------------------------------------------------------
# invariants on the GPU
# ---------------------------------------------------------------------------
def test_physical_placement_and_repeat_are_bit_identical():
    w = random_workload(21, dtype="bf16", num_q_heads=16, num_kv_heads=2, head_dim=128,
                        lens=[300, 17, 900, 45], spare_blocks=200)
    t1, _, _ = run_gpu(w)
    t1b, _, _ = run_gpu(w, t=upload(w))
    perm = np.random.default_rng(3).permutation(w.num_blocks)[: len(w.used_blocks)]
    w2 = dataclasses.replace(w, used_blocks=perm.astype(np.int64))
    t2, _, _ = run_gpu(w2)
    assert torch.equal(t1["out"], t1b["out"])
    assert torch.equal(t1["out"], t2["out"])


def test_split_and_unsplit_agree():
    w = random_workload(22, dtype="f32", num_q_heads=8, num_kv_heads=1, head_dim=128,
                        lens=[2000, 1, 777])
    outs = [run_gpu(w, partition_size=p)[0]["out"] for p in (0, 16, 512)]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 2e-6


def test_shared_memory_need_may_shrink_and_grow_again():
    """The dynamic shared memory a launch needs grows with the batch; calls of
    one kernel with a large, a small and again the large batch all launch."""
    for n in (300, 2, 300, 5, 301):
        w = random_workload(50 + n, dtype="f32", num_q_heads=3, num_kv_heads=3, head_dim=64,
                            num_seqs=n, max_len=40)
        ref, _ = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                     scale=w.scale, dtype=w.dtype)
        t, err, _ = run_gpu(w)
        assert err == 0
        assert_attention_close(t["out"], ref, "f32", f"{n} sequences")


@pytest.mark.parametrize("G", [4, 8])
def test_write_into_one_copy_moves_only_its_sequence(G):
    """Copy-on-write isolation on the GPU: after the copies, a slot write into
    one sequence's private copy of the last shared block changes that
    sequence's output alone, bit for bit everywhere else."""
    rng = np.random.default_rng(23)
    lens = 2048 + rng.integers(1, 300, size=16)
    w = make_workload(rng, name="cow", dtype="bf16", num_q_heads=2 * G, num_kv_heads=2,
                      head_dim=128, context_lens=lens, num_blocks=600, prefix_tokens=2048,
                      cow_count=8)
    t, err, _ = run_gpu(w)
    assert err == 0
    out0 = t["out"].clone()
    src, dst = (int(x) for x in w.block_mapping[0])
    tables = w.block_tables
    owners = [s for s in range(w.num_seqs) if dst in tables[s]]
    assert len(owners) == 1
    src_k = t["k_cache"][src].clone()
    key = torch.randn(1, 2, 128, device="cuda").to(torch.bfloat16)
    slots = torch.tensor([dst * 16 + 15], dtype=torch.int64, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.reshape_and_cache(key, -key, t["k_cache"], t["v_cache"], slots, err_flag=e)
    ws = ops.make_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.max_context_len, 0, torch.bfloat16)
    ops.decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
               scale=w.scale, max_context_len=w.max_context_len, workspace=ws, err_flag=e)
    torch.cuda.synchronize()
    assert e.item() == 0
    same = (t["out"].view(torch.int16) == out0.view(torch.int16)).flatten(1).all(dim=1).cpu()
    assert [s for s in range(w.num_seqs) if not same[s]] == owners
    assert torch.equal(t["k_cache"][src].view(torch.int16), src_k.view(torch.int16))
    # and the moved row is right
    k_ref, v_ref = w.k_pool.copy(), w.v_pool.copy()
    oracle.copy_blocks(k_ref, v_ref, w.block_mapping_compact)
    cdst = int(w.block_mapping_compact[0][1])
    kb = key.view(torch.int16).cpu().numpy()
    oracle.reshape_and_cache(k_ref, v_ref, kb, (-key).view(torch.int16).cpu().numpy(),
                             np.array([cdst * 16 + 15]))
    ref, _ = oracle.paged_decode(w.q, k_ref, v_ref, w.tables_compact, w.context_lens,
                                 scale=w.scale, dtype=w.dtype)
    assert_attention_close(t["out"], ref, "bf16", "after the write into one copy")


# ---------------------------------------------------------------------------
# device-side error contract
# ---------------------------------------------------------------------------
def test_bad_block_id_zeroes_only_that_sequence():
    w = random_workload(30, dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=64,
                        lens=[40, 40, 40])
    t = upload(w)
    t["block_tables"][1, 1] = w.num_blocks + 3
    ref, _ = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                 scale=w.scale, dtype=w.dtype)
    for ps in (0, 16):
        t["out"].fill_(5)
        _, err, ws = run_gpu(w, partition_size=ps, t=t)
        assert err & ops.ERRBIT_BLOCK_ID
        assert (t["out"][1] == 0).all()
        assert_attention_close(t["out"][[0, 2]], ref[[0, 2]], "bf16", "good rows")
        assert counters_zero(w, ws)


def test_bad_context_len_zeroes_the_row():
    w = random_workload(31, dtype="f32", num_q_heads=2, num_kv_heads=1, head_dim=64, lens=[20, 20])
    t = upload(w)
    t["context_lens"][0] = 10_000
    _, err, _ = run_gpu(w, t=t)
    assert err & ops.ERRBIT_CONTEXT_LEN and (t["out"][0] == 0).all() and t["out"][1].abs().sum() > 0


def test_bad_slot_and_bad_pair_are_skipped_and_flagged():
    w = build_workload("tiny")
    t = upload(w)
    good = t["k_cache"].clone()
    slots = t["slot_mapping"].clone()
    slots[0] = -1
    slots[1] = w.num_blocks * 16
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.reshape_and_cache(t["key"], t["value"], t["k_cache"], t["v_cache"], slots, err_flag=err)
    pairs = torch.tensor([[0, 0], [1, w.num_blocks]], dtype=torch.int32, device="cuda")
    ops.copy_blocks(t["k_cache"], t["v_cache"], pairs, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == ops.ERRBIT_SLOT | ops.ERRBIT_PAIR
    changed = (t["k_cache"].view(torch.int32) != good.view(torch.int32)).any(dim=(1, 3))
    b2, o2 = divmod(int(w.slot_mapping[2]), 16)
    assert changed.sum().item() == 2 and changed[b2, o2]       # only tokens 2 and 3 landed


# ---------------------------------------------------------------------------
# the full-size workloads, in the launch configuration the benchmark times
# ---------------------------------------------------------------------------
def full_reference(w):
    """The oracle's whole step (copies, slot write, attention) on every
    sequence of the workload: fp64 output and the caches after the step."""
    out, k_ref, v_ref, err = oracle.workload_step(w)
    assert err == 0
    return out, k_ref, v_ref


def pick_sequences(w, count, seed=0):
    lens = w.context_lens
    rng = np.random.default_rng(seed)
    chosen = {int(np.argmax(lens)), int(np.argmin(lens))}
    chosen |= set(rng.choice(len(lens), size=min(count, len(lens)), replace=False).tolist())
    return np.array(sorted(chosen))


@pytest.mark.parametrize("name", ["7b", "gqa70b", "prefix_cow", "long"])
def test_full_size_workloads(name):
    """The workload's whole step in the benchmark's launch configuration;
    every output element against the oracle, every used block bit-exact."""
    w = build_workload(name)
    ref, k_ref, v_ref = full_reference(w)
    t, err, ws = run_gpu(w)
    assert err == 0
    # slot write and copies: every used block bit-exact
    idx = torch.from_numpy(w.used_blocks).cuda()
    for dev, host in ((t["k_cache"], k_ref), (t["v_cache"], v_ref)):
        got = dev[idx].view(torch.int16).cpu().numpy()
        assert np.array_equal(got, host.view(np.int16)), "cache bytes differ"
    del idx
    assert_attention_close(t["out"], ref, w.dtype, f"{name} (pa_decode, all rows)", record=True,
                           strict_abs=True)
    assert counters_zero(w, ws)
