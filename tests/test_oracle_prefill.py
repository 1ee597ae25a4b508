"""Pins of the oracle's multi-token (chunked prefill) attention.

Query row j of sequence s sits at position n - Q + j and attends causally
to tokens 0..n-Q+j of its paged cache.  Pinned against torch SDPA with an
explicit mask over the same tokens gathered contiguously (library special
case), against the decode oracle (one query token is decode; any row is
decode over a cut context), and by planted mistakes.
"""
import os
import shutil
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_456_b200.workloads import make_workload, to_f64, f32_to_bf16_bits

from tests.test_oracle_pins import contiguous_kv


def prefill_case(seed, *, dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=64,
                 lens=(40, 17, 1, 64), queries=(5, 17, 1, 0)):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    w = make_workload(rng, name="prefill", dtype=dtype, num_q_heads=num_q_heads,
                      num_kv_heads=num_kv_heads, head_dim=head_dim, context_lens=lens,
                      num_blocks=int(sum(-(-lens // 16))) + 3)
    qs = np.concatenate([[0], np.cumsum(queries)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), num_q_heads, head_dim), dtype=np.float32)
    if dtype == "bf16":
        q = f32_to_bf16_bits(q)
    return w, q, qs


def run(w, q, qs, lib=None):
    return oracle.paged_prefill(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens, qs,
                                scale=w.scale, dtype=w.dtype, lib=lib)


def sdpa_causal(w, q, qs):
    G = w.num_q_heads // w.num_kv_heads
    qf = to_f64(q, w.dtype)
    out = np.zeros_like(qf)
    for s in range(w.num_seqs):
        n, Q = int(w.context_lens[s]), int(qs[s + 1] - qs[s])
        if Q == 0:
            continue
        k, v = contiguous_kv(w, s)
        qt = torch.from_numpy(qf[qs[s]:qs[s + 1]].transpose(1, 0, 2))[None]   # [1,Hq,Q,D]
        kt = torch.from_numpy(k).repeat_interleave(G, dim=0)[None]            # [1,Hq,n,D]
        vt = torch.from_numpy(v).repeat_interleave(G, dim=0)[None]
        keep = torch.arange(n)[None, :] <= (n - Q + torch.arange(Q))[:, None]
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=keep,
                                                             scale=w.scale)
        out[qs[s]:qs[s + 1]] = o[0].numpy().transpose(1, 0, 2)
    return out


SHAPES = [
    dict(dtype="f32", num_q_heads=4, num_kv_heads=2, head_dim=64),
    dict(dtype="bf16", num_q_heads=8, num_kv_heads=1, head_dim=128),
    dict(dtype="bf16", num_q_heads=16, num_kv_heads=2, head_dim=128),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s['dtype']}-{s['num_q_heads']}-{s['num_kv_heads']}")
def test_matches_masked_sdpa(shape):
    w, q, qs = prefill_case(1, lens=(40, 17, 1, 64, 33), queries=(5, 17, 1, 0, 16), **shape)
    out, err = run(w, q, qs)
    assert err == 0
    np.testing.assert_allclose(out, sdpa_causal(w, q, qs), rtol=0, atol=1e-12)


def test_one_query_token_is_decode():
    w, q, qs = prefill_case(2, lens=(40, 17, 1, 64), queries=(1, 1, 1, 1))
    out, err = run(w, q, qs)
    ref, e2 = oracle.paged_decode(q, w.k_pool, w.v_pool, w.tables_compact, w.context_lens,
                                  scale=w.scale, dtype=w.dtype)
    assert err == e2 == 0
    assert np.array_equal(out, ref)


def test_each_row_is_decode_over_its_prefix():
    w, q, qs = prefill_case(3, lens=(40, 33), queries=(7, 33))
    out, err = run(w, q, qs)
    assert err == 0
    for s in range(w.num_seqs):
        n, Q = int(w.context_lens[s]), int(qs[s + 1] - qs[s])
        for j in range(Q):
            r = qs[s] + j
            cut = np.array([n - Q + j + 1], dtype=np.int32)
            ref, e = oracle.paged_decode(q[r:r + 1], w.k_pool, w.v_pool, w.tables_compact[s:s + 1],
                                         cut, scale=w.scale, dtype=w.dtype,
                                         max_context_len=int(w.context_lens.max()))
            assert e == 0 and np.array_equal(out[r], ref[0])


def test_bad_query_rows_zero_that_sequence():
    w, q, qs = prefill_case(4, lens=(40, 17), queries=(5, 9))
    bad = qs.copy()
    bad[1] = 30                      # 30 query rows for a 40-token sequence: fine;
    bad[2] = 30 + 18                 # 18 rows for 17 tokens: too many
    q2 = np.resize(q, (int(bad[-1]),) + q.shape[1:])
    out, err = run(w, q2, bad)
    assert err == 32
    assert (out[30:] == 0).all() and np.abs(out[:30]).sum() > 0


MUTANTS = {
    "causal_off_by_one": ("for (int i = 0; i <= p; ++i) {\n                    size_t ro = row_offset",
                          "for (int i = 0; i < p; ++i) {\n                    size_t ro = row_offset"),
    "position_from_chunk_start": ("const int p = n - Q + j;", "const int p = j;"),
    "rows_of_the_first_sequence": ("qoff = ((size_t)(r0 + j) * num_q_heads + h) * head_dim;",
                                   "qoff = ((size_t)j * num_q_heads + h) * head_dim;"),
}

_RUNNER = """
import sys, numpy as np
sys.path.insert(0, {root!r})
import oracle
from tests.test_oracle_prefill import prefill_case, run, sdpa_causal
lib = oracle.load({so!r})
w, q, qs = prefill_case(1, lens=(40, 17, 1, 64, 33), queries=(5, 17, 1, 0, 16))
out, err = run(w, q, qs, lib=lib)
print("CAUGHT" if not np.allclose(out, sdpa_causal(w, q, qs), rtol=0, atol=1e-9) else "MISSED")
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    so = oracle.build(force=True, src=str(mutated), out=str(tmp_path / "mut.so"))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _RUNNER.format(root=root, so=so)],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 or "CAUGHT" in r.stdout, f"mutant {name} slipped through the pins"
