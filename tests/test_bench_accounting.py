"""The bench's algorithmic work per step (the numerators of every throughput
and roofline figure), checked against the layer's sizes worked out by hand for
the published workload shapes. CPU only."""
import numpy as np
import pytest

import bench
from sparse_mixture_experts_route_b200 import inputs as moe_inputs


def test_prefill_work_by_hand():
    s = moe_inputs.WORKLOADS["prefill"]          # T=4096 d=7168 E=384 k=8 f=2048
    a = bench.algorithmic(s, np.full(384, 85))   # every expert has rows
    # router 2*4096*7168*384 = 22.55 GFLOP; experts 6*4096*8*7168*2048 = 2886.2 GFLOP
    assert a["F"] == pytest.approx(22_548_578_304 + 2_886_218_022_912)
    # W_router 11.0 MB, x in + out 117.4 MB, 384 experts x 3 bf16 matrices of 7168 x 2048 = 33.82 GB
    assert a["B"] == pytest.approx(11_010_048 + 117_440_512 + 33_822_867_456)
    assert a["n_touched"] == 384
    # gate/up kernel: two weight matrices per touched expert (the step's per-unit
    # figure); the 32768 rows of x it reads and of h it writes are reported apart
    assert a["gu_bytes"] == pytest.approx(22_548_578_304)
    assert a["gu_impl_bytes"] == pytest.approx(469_762_048 + 134_217_728)
    assert a["gu_flops"] == pytest.approx(4 * 4096 * 8 * 7168 * 2048)


def test_untouched_experts_cost_no_bytes_and_bias_counts():
    s = moe_inputs.WORKLOADS["skewed"]           # T=8192 d=7168 E=896 k=16 f=512, biased router
    counts = np.zeros(896, dtype=np.int64)
    counts[:646] = 1
    a = bench.algorithmic(s, counts)
    per_expert = 3 * 7168 * 512 * 2
    assert a["n_touched"] == 646
    assert a["B"] == pytest.approx(4 * 7168 * 896 + 4 * 8192 * 7168 + 646 * per_expert + 4 * 896)
    a2 = bench.algorithmic(s, np.where(np.arange(896) < 10, 5, 0))
    assert a["B"] - a2["B"] == pytest.approx(636 * per_expert)
    assert a["F"] == a2["F"]                     # FLOPs follow the (token, expert) pairs, not the touched set
