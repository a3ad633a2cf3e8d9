"""GPU schedule (binary search) against the CPU oracle (linear scan):
bit-exact on the five workloads and on edge sweeps."""
import numpy as np
import pytest
import torch

import oracle
import paged_mqa_logits_b200 as mq
import workloads

pytestmark = pytest.mark.gpu


def gpu_schedule(ctx, S):
    c = torch.as_tensor(np.asarray(ctx, dtype=np.int32)).cuda()
    s = mq.mqa_logits_schedule(c, S)
    torch.cuda.synchronize()
    return s.cpu().numpy()


@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
@pytest.mark.parametrize("S", [148, 1, 37, 1000])
def test_configs_bit_exact(name, S):
    ctx = workloads.make_config(name).context_lens.numpy()
    assert np.array_equal(gpu_schedule(ctx, S), oracle.schedule(ctx, S))


EDGES = {
    "all_zero": [0] * 100,
    "one_row": [5000],
    "one_token": [1],
    "U_less_than_S": [256, 1, 0, 300],
    "U_equals_S": [256] * 148,
    "U_multiple_of_S": [512] * 148,
    "boundaries": [256 * m + d for m in range(1, 17) for d in (-1, 0, 1)],
    "negatives": [-5, 100, -1, 0, 700],
    "long": [131072, 1, 65536],
    "empty_batch": [],
}


@pytest.mark.parametrize("case", sorted(EDGES))
@pytest.mark.parametrize("S", [148, 7])
def test_edges_bit_exact(case, S):
    ctx = np.array(EDGES[case], dtype=np.int32)
    assert np.array_equal(gpu_schedule(ctx, S), oracle.schedule(ctx, S))


@pytest.mark.parametrize("seed", range(8))
def test_random_bit_exact(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.choice([1, 33, 1024, 1025, 4096, 32768]))
    ctx = rng.integers(0, 20000, B).astype(np.int32)
    ctx[rng.random(B) < 0.2] = 0
    for S in (148, 296):
        assert np.array_equal(gpu_schedule(ctx, S), oracle.schedule(ctx, S))
