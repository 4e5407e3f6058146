"""Pins of the oracle's router and permutation against closed forms and brute force.

Pinned facts (from the MoE pages and plain mathematics):
  * softmax rows sum to one and keep the logit order;
  * top-k = the k best experts under (logit descending, index ascending),
    found here by a library sort of all experts -- a different algorithm
    from the oracle's repeated selection;
  * k = E selects every expert in descending order;
  * gate weights are the selected softmax values; with renormalisation at
    k = 1 they are exactly 1 (Dense GEMM -> GroupedGEMM -> TP MoE, §4.3);
  * counts sum to T*k, offsets are their exclusive scan, every expert's
    segment lists its tokens in ascending order, and row_to_token inverts
    token_to_row (same page, §2.2 steps 3-4 and §4.2).
"""
import itertools
import math

import numpy as np
import pytest

import oracle


def _rng(seed=0):
    return np.random.default_rng(seed)


def test_softmax_rows_sum_to_one_and_keep_order():
    l = _rng().normal(size=(64, 37)) * 3
    p = oracle.softmax(l)
    assert np.all(np.abs(p.sum(axis=1) - 1.0) <= 1e-12)
    assert np.all(p > 0)
    assert np.array_equal(np.argsort(-l, axis=1, kind="stable"), np.argsort(-p, axis=1, kind="stable"))
    # brute force on a few rows with math.exp
    for t in range(4):
        z = [math.exp(v) for v in l[t]]
        s = math.fsum(z)
        assert np.allclose(p[t], [v / s for v in z], rtol=1e-13, atol=0)


def _brute_topk(row, k):
    return [e for _, e in sorted(((-v, e) for e, v in enumerate(row)))][:k]


@pytest.mark.parametrize("E,k", [(2, 1), (4, 2), (6, 3), (8, 8), (5, 5)])
def test_topk_matches_library_sort(E, k):
    rng = _rng(E * 10 + k)
    # integer logits in a tiny range: many exact ties
    l = rng.integers(-2, 3, size=(16, E)).astype(np.float64)
    idx = oracle.topk_select(l, k)
    for t in range(16):
        assert list(idx[t]) == _brute_topk(list(l[t]), k)


def test_topk_maximises_selected_sum_exhaustively():
    rng = _rng(7)
    E, k = 6, 3
    l = rng.normal(size=(16, E))
    idx = oracle.topk_select(l, k)
    for t in range(16):
        best = max(itertools.combinations(range(E), k), key=lambda c: sum(l[t, e] for e in c))
        assert sorted(idx[t]) == sorted(best)
        assert all(l[t, idx[t, j]] >= l[t, idx[t, j + 1]] for j in range(k - 1))


def test_topk_k_equals_E_is_descending_order():
    l = _rng(3).normal(size=(10, 7))
    idx = oracle.topk_select(l, 7)
    assert np.array_equal(idx, np.argsort(-l, axis=1, kind="stable"))


def test_tie_goes_to_lower_index():
    l = np.array([[1.0, 3.0, 3.0, 0.0], [2.0, 2.0, 2.0, 2.0]])
    assert oracle.topk_select(l, 2).tolist() == [[1, 2], [0, 1]]
    assert oracle.topk_select(l, 1).tolist() == [[1], [0]]


def test_gate_weights_are_selected_softmax_values():
    l = _rng(4).normal(size=(32, 8))
    p = oracle.softmax(l)
    idx = oracle.topk_select(l, 2)
    w = oracle.gate_weights(p, idx, renormalize=False)
    for t in range(32):
        assert w[t, 0] == p[t, idx[t, 0]] and w[t, 1] == p[t, idx[t, 1]]
    wr = oracle.gate_weights(p, idx, renormalize=True)
    assert np.allclose(wr.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # renormalised top-k weights equal a softmax over the top-k logits
    top = np.take_along_axis(l, idx, axis=1)
    assert np.allclose(wr, oracle.softmax(top), rtol=1e-14, atol=0)


def test_renormalised_top1_weight_is_exactly_one():
    l = _rng(5).normal(size=(50, 8))
    r = oracle.route(l, np.eye(8), None, k=1, renormalize=True)  # x = logits, W_r = I
    assert np.all(r["w"] == 1.0)
    r2 = oracle.route(l, np.eye(8), None, k=1, renormalize=False)
    assert np.all(r2["w"] < 1.0)


def test_router_bias_is_added_before_softmax():
    x = np.zeros((3, 4))
    bias = np.array([0.0, np.log(3.0), 0.0, 0.0])
    r = oracle.route(x, np.ones((4, 4)), bias, k=1)
    assert r["idx"][:, 0].tolist() == [1, 1, 1]
    assert np.allclose(r["w"][:, 0], 3.0 / 6.0, rtol=1e-15)


@pytest.mark.parametrize("T,E,k,shared", [(37, 5, 2, False), (64, 8, 3, True), (1, 4, 4, True), (20, 32, 1, False)])
def test_permutation_invariants(T, E, k, shared):
    rng = _rng(T + E + k)
    l = rng.normal(size=(T, E))
    l[:, 0] += 2.0  # one hot expert
    idx = oracle.topk_select(l, k)
    pm = oracle.permutation(idx, E, shared=shared)
    counts, offsets = pm["counts"], pm["offsets"]
    R = T * k
    assert counts.sum() == R
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert np.array_equal(offsets[:E + 1], np.concatenate([[0], np.cumsum(counts)]))
    if shared:
        assert offsets[E + 1] == R + T and len(offsets) == E + 2
    else:
        assert len(offsets) == E + 1
    r2t, t2r = pm["row_to_token"], pm["token_to_row"]
    assert sorted(t2r.ravel().tolist()) == list(range(R))
    for t in range(T):
        for j in range(k):
            row = t2r[t, j]
            assert r2t[row] == t
            e = idx[t, j]
            assert offsets[e] <= row < offsets[e + 1]
    for e in range(E):
        seg = r2t[offsets[e]:offsets[e + 1]].tolist()
        assert seg == sorted(t for t in range(T) if e in idx[t])
    if shared:
        assert r2t[R:].tolist() == list(range(T))


def test_empty_experts_have_empty_segments():
    idx = np.array([[3, 1], [3, 1], [1, 3]])
    pm = oracle.permutation(idx, 6)
    assert pm["counts"].tolist() == [0, 3, 0, 3, 0, 0]
    assert pm["offsets"].tolist() == [0, 0, 3, 3, 6, 6, 6]
    assert pm["token_to_row"].tolist() == [[3, 0], [4, 1], [2, 5]]


def test_imbalance_diagnostic():
    assert oracle.imbalance([2, 2, 2, 2]) == 1.0
    assert oracle.imbalance([8, 0, 0, 0]) == 4.0


def test_bf16_round_matches_torch():
    import torch
    v = np.concatenate([_rng(9).normal(size=4096).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0, 65504.0],
                                 dtype=np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(oracle.bf16_round(v), ref)
    # ties to even, worked by hand: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7
    assert oracle.bf16_round(np.float32(1.0 + 2 ** -8)) == 1.0
    assert oracle.bf16_round(np.float32(1.0 + 3 * 2 ** -8)) == 1.0 + 2 ** -6
