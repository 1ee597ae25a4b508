"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers may not call cudaMalloc once they are running -- an engine whose
memory pool already owns the device, or a step loop that cannot take the
device synchronisation an allocation may cause.  pa_decode_noalloc takes its
scratch from a fixed array inside the library instead of a caller workspace.
These tests call it through the C ABI twice in a row (different inputs each
time, so the second call starts from whatever the first left in the shared
array), on the CUDA-core path (bf16 and fp32 caches) and on the tensor-core
path (bf16, 8 query heads per KV head).  Each call must give the same bits
as pa_decode with a workspace of its own (same plan, same kernels) and stay
within the oracle's tolerance.

This file is named so pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_456_b200 import ops
from paged_kv_cache_456_b200.workloads import random_workload, upload

pytestmark = pytest.mark.gpu

F32_ATOL = 1e-5
BF16_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_456_b200 import build
    build.build()
    ops.library()


def _within_oracle(gpu, ref, dtype):
    g = gpu.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all()
    err = np.abs(g - ref)
    if dtype == "f32":
        assert err.max() <= F32_ATOL, err.max()
    else:
        assert (err <= BF16_TOL + BF16_TOL * np.abs(ref)).all(), err.max()


SHAPES = [("bf16", 128, 4), ("bf16", 128, 8), ("f32", 64, 4)]


@pytest.mark.parametrize("dtype,D,G", SHAPES, ids=lambda x: str(x))
@pytest.mark.parametrize("partition_size", [0, 64])
def test_noalloc_matches_pa_decode_on_two_calls_in_a_row(dtype, D, G, partition_size):
    lens = [1, 16, 17, 300, 1000, 45, 0, 2049]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    iv = torch.int16 if dtype == "bf16" else torch.int32
    for seed in (1, 2):                     # two calls in a row on the shared scratch
        w = random_workload(seed, dtype=dtype, num_q_heads=2 * G, num_kv_heads=2, head_dim=D,
                            lens=lens, spare_blocks=20)
        need = ops.workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                  w.max_context_len, partition_size, tdt)
        assert need <= ops.NOALLOC_SCRATCH_BYTES
        t = upload(w)
        ws = ops.make_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                w.max_context_len, partition_size, tdt)
        own = torch.empty_like(t["out"])
        err = torch.zeros(2, dtype=torch.int32, device="cuda")
        ops.decode(own, t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
                   scale=w.scale, max_context_len=w.max_context_len, workspace=ws,
                   partition_size=partition_size, err_flag=err[0:1])
        t["out"].fill_(3.0)
        ops.decode_noalloc(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                           t["context_lens"], scale=w.scale, max_context_len=w.max_context_len,
                           partition_size=partition_size, err_flag=err[1:2])
        torch.cuda.synchronize()
        assert err.tolist() == [0, 0]
        assert torch.equal(t["out"].view(iv), own.view(iv))
        ref, oerr = oracle.paged_decode(w.q, w.k_pool, w.v_pool, w.tables_compact,
                                        w.context_lens, scale=w.scale, dtype=w.dtype)
        assert oerr == 0
        _within_oracle(t["out"], ref, dtype)
        assert (t["out"][6] == 0).all()     # the empty sequence


def test_noalloc_rejects_a_request_larger_than_its_scratch():
    w = random_workload(3, dtype="bf16", num_q_heads=8, num_kv_heads=1, head_dim=128, lens=[5])
    t = upload(w)
    # 4096 sequences of up to 32768 tokens cut into 16-token partials need far
    # more than the fixed scratch holds
    need = ops.workspace_size(4096, 8, 1, 128, 32768, 16, torch.bfloat16)
    assert need > ops.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((4096, 8, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    tables = torch.zeros((4096, 2048), dtype=torch.int32, device="cuda")
    lens = torch.zeros(4096, dtype=torch.int32, device="cuda")
    with pytest.raises(ops.PagedAttentionError) as e:
        ops.decode_noalloc(out, q, t["k_cache"], t["v_cache"], tables, lens, scale=0.1,
                           max_context_len=32768, partition_size=16)
    assert e.value.status == ops.PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (out == 0).all()                 # nothing was launched
