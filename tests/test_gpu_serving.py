"""The GPU path driven by the continuous-batching simulator.

Every step applies the simulator's plan on the GPU -- copy-on-write copies
(pa_copy_blocks), the prompt writes of newly admitted requests
(pa_reshape_and_cache), then the fused slot write + decode of the batch
(pa_decode_append, or pa_decode_shared_prefix with the groups the host
planner finds among the requests sharing the system prompt) -- and the same plan on a CPU mirror of the pool with the
oracle.  Each step's attention output is compared with the oracle's; at the
end the two pools must be identical byte for byte.  Blocks are reused after
requests finish or are preempted, so stale rows of earlier owners sit next
to live ones.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_456_b200 import ops
from paged_kv_cache_456_b200.scheduler import ServingSimulator, poisson_arrivals
from paged_kv_cache_456_b200.workloads import f32_to_bf16_bits

from tests.test_gpu_parity import assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_456_b200 import build
    build.build()
    ops.library()


class TokenValues:
    """K and V of token ``pos`` of request ``rid`` (-1: the system prompt),
    fixed by (seed, rid), so a recomputed request writes the same rows."""

    def __init__(self, seed, hkv, d, dtype, max_tokens):
        self.seed, self.shape, self.dtype, self.max_tokens = seed, (hkv, d), dtype, max_tokens
        self.cache = {}

    def rows(self, rid, positions):
        if rid not in self.cache:
            g = np.random.default_rng([self.seed, rid + 1])
            kv = g.standard_normal((2, self.max_tokens) + self.shape, dtype=np.float32)
            if self.dtype == "bf16":
                kv = f32_to_bf16_bits(kv)
            self.cache[rid] = kv
        kv = self.cache[rid]
        p = np.asarray(positions, dtype=np.int64)
        return kv[0][p], kv[1][p]


def to_dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(torch.bfloat16) if dtype == "bf16" else t).cuda()


@pytest.mark.parametrize("dtype,G,D,dedup", [("f32", 2, 64, False), ("bf16", 8, 128, False),
                                             ("bf16", 1, 128, False), ("bf16", 8, 128, True),
                                             ("bf16", 4, 128, True)])
def test_simulated_serving_steps(dtype, G, D, dedup):
    hkv, max_tokens, num_blocks = 2, 1024, 220
    rng = np.random.default_rng(11)
    arr = poisson_arrivals(rng, 40, 1.0, prompt_mean=150, output_mean=40, max_tokens=max_tokens,
                           shared_fraction=0.5)
    sim = ServingSimulator(num_blocks, arr, max_tokens=max_tokens, max_batch=24, prefix_len=40,
                           rng=np.random.default_rng(12))
    vals = TokenValues(13, hkv, D, dtype, max_tokens)
    np_dt = np.int16 if dtype == "bf16" else np.float32
    shape = (num_blocks, hkv, 16, D)
    k_host = np.zeros(shape, dtype=np_dt)
    v_host = np.zeros(shape, dtype=np_dt)
    k_dev, v_dev = to_dev(k_host, dtype), to_dev(v_host, dtype)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(D)

    def write(rid, positions, slots):
        if not slots:
            return
        k, v = vals.rows(rid, positions)
        assert oracle.reshape_and_cache(k_host, v_host, k, v, np.array(slots, np.int64)) == 0
        ops.reshape_and_cache(to_dev(k, dtype), to_dev(v, dtype), k_dev, v_dev,
                              torch.tensor(slots, dtype=torch.int64, device="cuda"), err_flag=err)

    write(-1, range(sim.prefix_len), sim.prefix_slots())
    steps = preempted_seen = grouped_steps = 0
    while (plan := sim.step()) is not None:
        steps += 1
        if plan.copies:
            pairs = np.array(plan.copies, dtype=np.int32)
            assert oracle.copy_blocks(k_host, v_host, pairs) == 0
            ops.copy_blocks(k_dev, v_dev, torch.from_numpy(pairs).cuda(), err_flag=err)
        for rid, positions, slots in plan.prefill:
            write(rid, positions, slots)
        B = len(plan.rids)
        # the decode batch: q, and the new token's K/V per request
        q = np.random.default_rng([14, steps]).standard_normal((B, hkv * G, D), dtype=np.float32)
        if dtype == "bf16":
            q = f32_to_bf16_bits(q)
        key = np.empty((B, hkv, D), dtype=np_dt)
        value = np.empty_like(key)
        for b, rid in enumerate(plan.rids):
            key[b], value[b] = (x[0] for x in vals.rows(rid, [int(plan.context_lens[b]) - 1]))
        assert oracle.reshape_and_cache(k_host, v_host, key, value, plan.new_slots) == 0
        ref, e = oracle.paged_decode(q, k_host, v_host, plan.block_tables, plan.context_lens,
                                     scale=scale, dtype=dtype, max_context_len=max_tokens)
        assert e == 0
        out = torch.empty((B, hkv * G, D), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32,
                          device="cuda")
        tables = torch.from_numpy(plan.block_tables).cuda()
        lens = torch.from_numpy(plan.context_lens).cuda()
        if dedup:
            # the batch's sharers (the system prompt), found by the host planner
            groups = ops.shared_prefix_plan(plan.block_tables, plan.context_lens)
            ws = ops.make_shared_prefix_workspace(B, groups.num_listed, hkv * G, hkv, D,
                                                  plan.block_tables.shape[1], max_tokens)
            ops.decode_shared_prefix(out, to_dev(q, dtype), k_dev, v_dev, tables, lens,
                                     groups.to(), scale=scale, max_context_len=max_tokens,
                                     workspace=ws, key=to_dev(key, dtype),
                                     value=to_dev(value, dtype), err_flag=err)
            grouped_steps += groups.num_groups > 0
        else:
            ws = ops.make_workspace(B, hkv * G, hkv, D, max_tokens, 0, out.dtype)
            ops.decode_append(out, to_dev(q, dtype), to_dev(key, dtype), to_dev(value, dtype),
                              k_dev, v_dev, tables, lens, scale=scale,
                              max_context_len=max_tokens, workspace=ws, err_flag=err)
        torch.cuda.synchronize()
        assert err.item() == 0, f"step {plan.step}: error bits {err.item()}"
        assert_attention_close(out, ref, dtype, f"step {plan.step}")
        preempted_seen = max(preempted_seen, sim.stats.preemptions)
    assert sim.stats.finished == 40 and preempted_seen > 0
    assert grouped_steps > 0 or not dedup
    iv = torch.int16 if dtype == "bf16" else torch.int32
    for dev, host in ((k_dev, k_host), (v_dev, v_host)):
        got = dev.view(iv).cpu().numpy()
        assert np.array_equal(got.view(np.uint8), host.view(np.uint8)), "pools differ"
