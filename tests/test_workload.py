"""The seeded input generator: determinism, shapes and the routing skew it induces."""
import numpy as np
import pytest
import torch

import oracle
from workload import CONFIGS, make_inputs, make_router_logits, shape_of
from workload.gen import make_expert_weights, zipf_bias


def test_deterministic_and_order_independent():
    s = shape_of("tiny")
    a = make_inputs(s, seed=7)
    b = make_inputs(s, seed=7)
    for key in ("x", "W_r", "W1", "W2", "W1s", "W2s"):
        assert torch.equal(a[key], b[key]), key
    c = make_inputs(s, seed=8)
    assert not torch.equal(a["x"], c["x"])
    # one expert regenerated alone equals its slice of the stacked tensor
    assert torch.equal(make_expert_weights(s, "W1", 5, "cpu", 7), a["W1"][5])


def test_tiny_shapes_and_dtypes():
    s = shape_of("tiny")
    t = make_inputs(s)
    assert t["x"].shape == (256, 256) and t["x"].dtype == torch.float32
    assert t["W_r"].dtype == torch.float32
    assert t["W1"].shape == (8, 1024, 256) and t["W1"].dtype == torch.bfloat16
    assert t["W2"].shape == (8, 256, 512)
    assert t["W1s"].shape == (1024, 256) and t["W2s"].shape == (256, 512)
    assert t["bias"] is None
    assert abs(float(t["W1"].float().std()) - 0.02) < 1e-3


def test_zipf_bias_skews_mixtral_routing():
    s = shape_of("mixtral")
    t = make_inputs(s, experts=False)
    r = oracle.route(t["x"], t["W_r"], t["bias"], s.k)
    counts = oracle.expert_counts(r["idx"], s.E)
    assert counts.sum() == s.T * s.k
    ratio = counts.max() / counts.min()
    assert 2.5 <= ratio <= 8.0, counts   # hot experts get several times the cold ones' tokens


def test_zipf_bias_is_a_permuted_power_law():
    b = zipf_bias(8, 1.0, 1234).numpy()
    assert np.allclose(np.sort(-b / 0.7), np.log1p(np.arange(8)), rtol=1e-6, atol=1e-7)


def test_router_micro_logits():
    l = make_router_logits(1024, 128)
    assert l.dtype == torch.float16 and l.shape == (1024, 128)
    assert abs(float(l.float().std()) - 1.0) < 0.02


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_config_divisibility(name):
    s = CONFIGS[name]
    assert s.d % 128 == 0 and s.inter % 128 == 0
    assert s.shared_inter in (0, s.inter)
    assert 1 <= s.k <= s.E
