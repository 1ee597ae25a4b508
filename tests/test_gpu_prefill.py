"""Several query tokens per sequence (pa_prefill) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_456_b200 import ops
from paged_kv_cache_456_b200.workloads import upload

from tests.test_gpu_parity import SHAPES, assert_attention_close
from tests.test_oracle_prefill import prefill_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_456_b200 import build
    build.build()
    ops.library()


def run_prefill(w, q, qs, psize=0, t=None, qs_dev=None):
    t = t if t is not None else upload(w)
    tdt = t["q"].dtype
    qd = torch.from_numpy(np.ascontiguousarray(q))
    qd = (qd.view(torch.bfloat16) if w.dtype == "bf16" else qd).cuda()
    out = torch.full(qd.shape, 7.0, dtype=tdt, device="cuda")
    qs_dev = qs_dev if qs_dev is not None else torch.from_numpy(qs).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = ops.make_prefill_workspace(w.num_seqs, qd.shape[0], w.num_q_heads, w.num_kv_heads,
                                    w.head_dim, w.max_context_len, psize, tdt)
    ops.prefill(out, qd, t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"], qs_dev,
                scale=w.scale, max_context_len=w.max_context_len, workspace=ws,
                partition_size=psize, err_flag=err)
    torch.cuda.synchronize()
    return out, int(err.item()), t


@pytest.mark.parametrize("dtype,D,G", SHAPES, ids=lambda x: str(x))
@pytest.mark.parametrize("psize", [0, 16, 512])
def test_prefill_matches_the_oracle(dtype, D, G, psize):
    hkv = 2
    w, q, qs = prefill_case(300 + D + G, dtype=dtype, num_q_heads=hkv * G, num_kv_heads=hkv,
                            head_dim=D, lens=(40, 17, 1, 700, 33, 16),
                            queries=(5, 17, 1, 40, 0, 16))
    ref, oerr = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                     scale=w.scale, dtype=w.dtype)
    out, err, _ = run_prefill(w, q, qs, psize)
    assert err == 0 and oerr == 0
    assert_attention_close(out, ref, dtype, f"prefill {dtype} D{D} G{G} P{psize}")


@pytest.mark.parametrize("G", [1, 8])
def test_one_query_per_sequence_is_decode(G):
    """One query row per sequence attends like decode.  bf16 prefill runs on
    the tcgen05 tensor cores (softmax weights rounded to bf16 for P.V), so the
    two agree within the bf16 bound rather than bit for bit."""
    w, q, qs = prefill_case(5, dtype="bf16", num_q_heads=2 * G, num_kv_heads=2, head_dim=128,
                            lens=(40, 17, 300, 64), queries=(1, 1, 1, 1))
    out, err, t = run_prefill(w, q, qs)
    assert err == 0
    ws = ops.make_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.max_context_len, 0, torch.bfloat16)
    dec = torch.empty_like(out)
    qd = torch.from_numpy(np.ascontiguousarray(q)).view(torch.bfloat16).cuda()
    ops.decode(dec, qd, t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
               scale=w.scale, max_context_len=w.max_context_len, workspace=ws)
    torch.cuda.synchronize()
    ref = dec.float().cpu().numpy().astype(np.float64)
    assert_attention_close(out, ref, "bf16", "one query row per sequence")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_chunks_spanning_several_tiles(G, D):
    """Chunks longer than one 128-column tile (128 / G query rows per tile)
    over contexts longer than one 128-key tile, with ragged ends: a 300-row
    chunk, a 129-row chunk, single rows and a chunk that is the whole
    sequence."""
    w, q, qs = prefill_case(900 + G + D, dtype="bf16", num_q_heads=2 * G, num_kv_heads=2,
                            head_dim=D, lens=(1000, 129, 257, 1, 300, 700),
                            queries=(300, 129, 1, 1, 300, 65))
    ref, oerr = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                     scale=w.scale, dtype=w.dtype)
    out, err, _ = run_prefill(w, q, qs)
    assert err == 0 and oerr == 0
    assert_attention_close(out, ref, "bf16", f"tiles G{G} D{D}")


def test_repeat_calls_are_bit_identical():
    w, q, qs = prefill_case(77, dtype="bf16", num_q_heads=16, num_kv_heads=2, head_dim=128,
                            lens=(500, 130, 64), queries=(200, 3, 64))
    out1, err1, t = run_prefill(w, q, qs)
    out2, err2, _ = run_prefill(w, q, qs, t=t)
    assert err1 == err2 == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


@pytest.mark.parametrize("D", [64, 128])
def test_output_aligned_to_16_bytes_only(D):
    """The epilogue stores 32 bytes at a time when the output allows it; an
    output that is 16-byte aligned only takes the 16-byte stores, with the
    same result."""
    w, q, qs = prefill_case(79, dtype="bf16", num_q_heads=16, num_kv_heads=2, head_dim=D,
                            lens=(300, 170), queries=(150, 40))
    ref, err, t = run_prefill(w, q, qs)
    qd = torch.from_numpy(np.ascontiguousarray(q)).view(torch.bfloat16).cuda()
    buf = torch.full((qd.numel() + 8,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[8:].view(qd.shape)  # (16 bytes past a 256-byte aligned start)
    assert out.data_ptr() % 32 == 16
    err2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = ops.make_prefill_workspace(w.num_seqs, qd.shape[0], w.num_q_heads, w.num_kv_heads,
                                    w.head_dim, w.max_context_len, 0, torch.bfloat16)
    ops.prefill(out, qd, t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                torch.from_numpy(qs).cuda(), scale=w.scale, max_context_len=w.max_context_len,
                workspace=ws, err_flag=err2)
    torch.cuda.synchronize()
    assert err == err2.item() == 0
    assert torch.equal(ref.view(torch.int16), out.view(torch.int16))


def test_workspace_reused_by_different_calls():
    """Calls with different work on one workspace: each call's unit layout is
    written by its own plan kernel, and no call may see the previous call's
    (a stale layout once dropped whole units here)."""
    cases = [prefill_case(80 + i, dtype="bf16", num_q_heads=32, num_kv_heads=4, head_dim=128,
                          lens=lens, queries=qs)
             for i, (lens, qs) in enumerate([((1500, 900, 1200, 2000), (64, 64, 64, 64)),
                                             ((700, 300, 129), (200, 100, 129)),
                                             ((1500, 900, 1200, 2000), (64, 64, 64, 64))])]
    big = max(ops.make_prefill_workspace(w.num_seqs, q.shape[0], w.num_q_heads, w.num_kv_heads,
                                         w.head_dim, w.max_context_len, 0, torch.bfloat16).numel()
              for w, q, _ in cases)
    ws = torch.zeros(big, dtype=torch.uint8, device="cuda")
    for w, q, qs in cases * 2:
        t = upload(w)
        qd = torch.from_numpy(np.ascontiguousarray(q)).view(torch.bfloat16).cuda()
        out = torch.full(qd.shape, 7.0, dtype=torch.bfloat16, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.prefill(out, qd, t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                    torch.from_numpy(qs).cuda(), scale=w.scale, max_context_len=w.max_context_len,
                    workspace=ws, err_flag=err)
        torch.cuda.synchronize()
        ref, _ = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                      scale=w.scale, dtype=w.dtype)
        assert err.item() == 0
        assert_attention_close(out, ref, "bf16", "reused workspace")


def test_bad_block_zeroes_that_sequence_only():
    w, q, qs = prefill_case(78, dtype="bf16", num_q_heads=8, num_kv_heads=2, head_dim=128,
                            lens=(200, 150, 90), queries=(20, 30, 10))
    ref, _ = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                  scale=w.scale, dtype=w.dtype)
    t = upload(w)
    t["block_tables"][1, 2] = w.num_blocks + 5
    out, err, _ = run_prefill(w, q, qs, t=t)
    assert err == ops.ERRBIT_BLOCK_ID
    r0, r1 = int(qs[1]), int(qs[2])
    assert (out[r0:r1] == 0).all()
    keep = np.r_[0:r0, r1:int(qs[-1])]
    assert_attention_close(out[torch.from_numpy(keep).cuda()], ref[keep], "bf16", "other rows")


def test_long_chunks_of_a_large_batch():
    """8 sequences of ~1-2K tokens, each with a 64-token chunk: 512 query rows."""
    rng = np.random.default_rng(6)
    lens = tuple(int(x) for x in rng.integers(900, 2100, size=8))
    for G in (1, 8):
        w, q, qs = prefill_case(7 + G, dtype="bf16", num_q_heads=4 * G, num_kv_heads=4,
                                head_dim=128, lens=lens, queries=(64,) * 8)
        ref, _ = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                      scale=w.scale, dtype=w.dtype)
        out, err, _ = run_prefill(w, q, qs)
        assert err == 0
        assert_attention_close(out, ref, "bf16", f"chunks of 64, G{G}")


def test_bad_query_rows_zero_that_sequence_only():
    w, q, qs = prefill_case(8, dtype="f32", lens=(40, 17, 30), queries=(5, 9, 3))
    bad = qs.copy()
    bad[2] = bad[1] + 18                # 18 rows for a 17-token sequence
    bad[3] = bad[2] + 3
    q2 = np.resize(q, (int(bad[-1]),) + q.shape[1:])
    ref, oerr = oracle.paged_prefill(q2, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                     bad, scale=w.scale, dtype=w.dtype)
    out, err, _ = run_prefill(w, q2, bad)
    assert err == ops.ERRBIT_QUERY == oerr
    assert (out[5:23] == 0).all()
    assert_attention_close(out, ref, "f32", "rows around the bad sequence")


def test_prefill_workload_step():
    """The benchmark's prefill step: the chunks' slot write, then pa_prefill."""
    from paged_kv_cache_456_b200.workloads import build_workload
    w = build_workload("prefill")
    t = upload(w)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.reshape_and_cache(t["key"], t["value"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                          err_flag=err)
    ws = ops.make_prefill_workspace(w.num_seqs, t["q"].shape[0], w.num_q_heads, w.num_kv_heads,
                                    w.head_dim, w.max_context_len, 0, torch.bfloat16)
    ops.prefill(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                t["context_lens"], t["query_start"], scale=w.scale,
                max_context_len=w.max_context_len, workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    ref, _, _, oerr = oracle.workload_step(w)
    assert err.item() == 0 and oerr == 0
    assert_attention_close(t["out"], ref, "bf16", "prefill (pa_prefill, all rows)", record=True)


@pytest.mark.parametrize("queries", [(1, 1, 1), (3, 5, 7), (2, 64, 33), (128, 1, 0)])
def test_row_pairs_with_odd_and_single_rows(queries):
    """8 heads per KV head, bf16: pairs of query rows share each tile; a
    sequence's last pair may hold one row, and the earlier row of a pair must
    not see the later row's token."""
    w, q, qs = prefill_case(400 + sum(queries), dtype="bf16", num_q_heads=16, num_kv_heads=2,
                            head_dim=128, lens=(200, 65, 140), queries=queries)
    ref, oerr = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                     scale=w.scale, dtype=w.dtype)
    for psize in (0, 16):
        out, err, _ = run_prefill(w, q, qs, psize)
        assert err == 0 and oerr == 0
        assert_attention_close(out, ref, "bf16", f"queries {queries} P{psize}")


@pytest.mark.parametrize("S", [2048, 2049])
def test_more_sequences_than_the_plan_keeps_on_chip(S):
    """The plan kernel keeps each sequence's lengths and unit start on chip
    for up to 2048 sequences and reads them from the arrays past that: both
    sides of the limit, with sequences that have no query rows and one with a
    bad block id near the end."""
    rng = np.random.default_rng(S)
    lens = rng.integers(1, 60, size=S)
    queries = np.minimum(lens, rng.integers(0, 4, size=S))
    w, q, qs = prefill_case(S, dtype="bf16", num_q_heads=16, num_kv_heads=2, head_dim=128,
                            lens=tuple(int(x) for x in lens),
                            queries=tuple(int(x) for x in queries))
    ref, oerr = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                     scale=w.scale, dtype=w.dtype)
    assert oerr == 0
    out, err, t = run_prefill(w, q, qs)
    assert err == 0
    assert_attention_close(out, ref, "bf16", f"{S} sequences")
    bad = int(np.nonzero(queries)[0][-1])
    t["block_tables"][bad, 0] = w.num_blocks + 7
    out, err, _ = run_prefill(w, q, qs, t=t)
    assert err == ops.ERRBIT_BLOCK_ID
    r0, r1 = int(qs[bad]), int(qs[bad + 1])
    assert (out[r0:r1] == 0).all()
    keep = np.r_[0:r0, r1:int(qs[-1])]
    assert_attention_close(out[torch.from_numpy(keep).cuda()], ref[keep], "bf16", "other rows")


def test_many_units_per_cta():
    """256 sequences with chunks of 32 rows, 8 heads per KV head: about 14
    work units per CTA, so each CTA hands over the next unit's Q many times
    (while the previous unit's O goes out), and the plan kernel scans more
    rows than one warp holds."""
    rng = np.random.default_rng(1409)
    S = 256
    lens = tuple(int(x) for x in rng.integers(40, 400, size=S))
    w, q, qs = prefill_case(1409, dtype="bf16", num_q_heads=64, num_kv_heads=8, head_dim=128,
                            lens=lens, queries=(32,) * S)
    ref, oerr = oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                     scale=w.scale, dtype=w.dtype)
    out, err, _ = run_prefill(w, q, qs)
    assert err == 0 and oerr == 0
    assert_attention_close(out, ref, "bf16", "256 chunks of 32 rows")
