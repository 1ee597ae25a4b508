"""Fused slot write + decode (pa_decode_append) on the GPU.

Its result is defined as that of the slot write followed by decode, so the
two are compared bit for bit (output and both caches), and the output is
also held to the oracle's tolerance.  The new token's slot holds NaN in the
uploaded pool: a kernel that read it from the cache instead of from
key/value would show it.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_456_b200 import ops
from paged_kv_cache_456_b200.workloads import build_workload, random_workload, upload

from tests.test_gpu_parity import SHAPES, assert_attention_close, counters_zero

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_456_b200 import build
    build.build()
    ops.library()


def two_calls(w, t, ps):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.reshape_and_cache(t["key"], t["value"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                          err_flag=err)
    ws = ops.make_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.max_context_len, ps, t["q"].dtype)
    ops.decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
               scale=w.scale, max_context_len=w.max_context_len, workspace=ws, partition_size=ps,
               err_flag=err)
    torch.cuda.synchronize()
    return int(err.item())


def fused(w, t, ps, key=None, value=None):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if key is None:
        key, value = t["key_seq"], t["value_seq"]
    ws = ops.make_workspace(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                            w.max_context_len, ps, t["q"].dtype)
    ops.decode_append(t["out"], t["q"], key, value, t["k_cache"], t["v_cache"], t["block_tables"],
                      t["context_lens"], scale=w.scale, max_context_len=w.max_context_len,
                      workspace=ws, partition_size=ps, err_flag=err)
    torch.cuda.synchronize()
    return int(err.item()), ws


def same_bits(a, b):
    iv = torch.int16 if a.dtype == torch.bfloat16 else torch.int32
    return torch.equal(a.view(iv), b.view(iv))


@pytest.mark.parametrize("dtype,D,G", SHAPES, ids=lambda x: str(x))
@pytest.mark.parametrize("psize", [0, 16, 512])
def test_fused_equals_slot_write_then_decode(dtype, D, G, psize):
    hkv = 2
    lens = [1, 15, 16, 17, 0, 33, 100, 511, 512, 513, 700]
    w = random_workload(2000 + D + G, dtype=dtype, num_q_heads=hkv * G, num_kv_heads=hkv,
                        head_dim=D, lens=lens, spare_blocks=23, new_token=True)
    a = upload(w)
    b = upload(w)
    assert two_calls(w, a, psize) == 0
    err, ws = fused(w, b, psize)
    assert err == 0
    assert same_bits(a["out"], b["out"])
    assert same_bits(a["k_cache"], b["k_cache"]) and same_bits(a["v_cache"], b["v_cache"])
    assert counters_zero(w, ws)
    ref, _, _, oerr = oracle.workload_step(w)
    assert oerr == 0
    assert_attention_close(b["out"], ref, dtype, f"fused {dtype} D{D} G{G} P{psize}")
    assert (b["out"][4] == 0).all()


def test_single_token_sequences_return_the_new_value():
    w = random_workload(41, dtype="f32", num_q_heads=8, num_kv_heads=2, head_dim=128,
                        lens=[1, 1, 1], new_token=True)
    t = upload(w)
    key, value = t["key_seq"], t["value_seq"]
    err, _ = fused(w, t, 0, key, value)
    assert err == 0
    # one position: softmax weight 1, out = the new V row, head by head
    want = value.repeat_interleave(4, dim=1)
    assert torch.equal(t["out"], want)


def test_bad_last_block_writes_nothing():
    w = random_workload(42, dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=64,
                        lens=[40, 40, 40], new_token=True)
    t = upload(w)
    t["block_tables"][1, 2] = w.num_blocks + 1           # sequence 1's last block
    t["context_lens"][2] = 10_000                         # sequence 2's length
    k0, v0 = t["k_cache"].clone(), t["v_cache"].clone()
    t["out"].fill_(3)
    err, ws = fused(w, t, 16)
    assert err & ops.ERRBIT_BLOCK_ID and err & ops.ERRBIT_CONTEXT_LEN
    assert (t["out"][1] == 0).all() and (t["out"][2] == 0).all()
    # only sequence 0's new row landed
    changed = (t["k_cache"].view(torch.int16) != k0.view(torch.int16)).any(dim=(1, 3))
    b0, o0 = divmod(int(w.slot_mapping[0]), 16)
    assert changed.sum().item() == 1 and changed[b0, o0]
    assert ((t["v_cache"].view(torch.int16) != v0.view(torch.int16)).any(dim=(1, 3))
            == changed).all()
    assert counters_zero(w, ws)


def test_host_checks():
    w = random_workload(43, dtype="bf16", num_q_heads=4, num_kv_heads=2, head_dim=64,
                        lens=[20], new_token=True)
    t = upload(w)
    key, value = t["key_seq"], t["value_seq"]
    ws = ops.make_workspace(1, 4, 2, 64, w.max_context_len, 0, torch.bfloat16)
    # contiguous but 2 bytes past a 16-byte boundary
    shifted = torch.empty(key.numel() + 1, dtype=key.dtype, device="cuda")[1:].view(key.shape)
    shifted.copy_(key)
    with pytest.raises(ops.PagedAttentionError):
        ops.decode_append(t["out"], t["q"], shifted, value, t["k_cache"], t["v_cache"],
                          t["block_tables"], t["context_lens"], scale=w.scale,
                          max_context_len=w.max_context_len, workspace=ws)


@pytest.mark.parametrize("name", ["tiny", "7b"])
def test_full_size_fused_step(name):
    """The workloads whose step writes a new token, in the benchmark's launch
    configuration: one fused call against the two-call step, bit for bit,
    and every output element against the oracle."""
    w = build_workload(name)
    a = upload(w)
    assert two_calls(w, a, w.partition_size) == 0
    out_a = a["out"].clone()
    k_a, v_a = a["k_cache"], a["v_cache"]
    del a
    b = upload(w)
    err, ws = fused(w, b, w.partition_size)
    assert err == 0 and counters_zero(w, ws)
    assert same_bits(out_a, b["out"])
    assert same_bits(k_a, b["k_cache"]) and same_bits(v_a, b["v_cache"])
    ref, _, _, oerr = oracle.workload_step(w)
    assert oerr == 0
    assert_attention_close(b["out"], ref, w.dtype, f"{name} (pa_decode_append, all rows)",
                           record=True, strict_abs=w.dtype == "bf16")
