"""Pins of the oracle's capacity limit (token drop with an overflow path).

"Dense GEMM -> GroupedGEMM -> TP MoE" §5.1 names a capacity factor as an
inference-time remedy for expert imbalance: each expert takes at most a fixed
number of tokens and the tokens over it take a fallback path; "DeepSeek MoE
architecture overview" §3.2 states the capacity factor as an upper bound on
the share of a forward's tokens one expert may take.  The oracle's reading:
an expert keeps its first C (token, slot) pairs in ascending token order, an
overflowing pair gets no row (token_to_row = -1) and adds nothing to its
token's output, which keeps the shared expert and its other experts.

Checked here against a hand-worked case, a brute-force rule written with a
sort, the plan's invariants, and the closed forms of the forward.
"""
import numpy as np
import pytest

import oracle


def test_hand_worked_two_experts_capacity_two():
    # tokens 0..5, top-1: expert 0 gets tokens 0, 2, 3, 5; expert 1 gets 1, 4
    idx = np.array([[0], [1], [0], [0], [1], [0]])
    p = oracle.permutation(idx, 2, shared=True, capacity=2)
    assert p["counts"].tolist() == [2, 2]                 # expert 0 keeps tokens 0 and 2
    assert p["offsets"].tolist() == [0, 2, 4, 10]         # shared rows follow the 4 kept rows
    assert p["token_to_row"].ravel().tolist() == [0, 2, 1, -1, 3, -1]
    assert p["row_to_token"].tolist() == [0, 2, 1, 4, 0, 1, 2, 3, 4, 5, -1, -1]
    assert p["kept"].ravel().tolist() == [True, True, True, False, True, False]


def _brute_kept(idx, E, C):
    """Kept pairs by the rule written with a sort: expert e keeps the C smallest token ids among its pairs."""
    kept = set()
    for e in range(E):
        toks = sorted(t for t in range(idx.shape[0]) for j in range(idx.shape[1]) if idx[t, j] == e)
        kept.update((t, e) for t in toks[:C])
    return kept


@pytest.mark.parametrize("T,E,k,C,shared", [(40, 4, 2, 7, True), (33, 8, 3, 1, False), (100, 16, 4, 20, True)])
def test_plan_follows_the_rule_and_its_invariants(T, E, k, C, shared):
    rng = np.random.default_rng(T + E + C)
    logits = rng.normal(size=(T, E)) - 0.8 * np.log1p(np.arange(E))  # skewed, so some experts overflow
    idx = oracle.topk_select(logits, k)
    p = oracle.permutation(idx, E, shared=shared, capacity=C)
    want = _brute_kept(idx, E, C)
    got = {(t, int(idx[t, j])) for t in range(T) for j in range(k) if p["kept"][t, j]}
    assert got == want
    n = oracle.expert_counts(idx, E)
    assert n.max() > C  # the case really drops something
    assert np.array_equal(p["counts"], np.minimum(n, C))
    assert p["offsets"][0] == 0 and np.array_equal(np.diff(p["offsets"][:E + 1]), p["counts"])
    used = int(p["offsets"][E])
    for t in range(T):
        for j in range(k):
            r = p["token_to_row"][t, j]
            if p["kept"][t, j]:
                assert p["row_to_token"][r] == t
                e = idx[t, j]
                assert p["offsets"][e] <= r < p["offsets"][e + 1]
            else:
                assert r == -1
    if shared:
        assert p["offsets"][E + 1] == used + T
        assert np.array_equal(p["row_to_token"][used:used + T], np.arange(T))
    assert np.all(p["row_to_token"][used + (T if shared else 0):] == -1)


def test_large_capacity_changes_nothing():
    rng = np.random.default_rng(3)
    T, d, E, k, I = 24, 64, 4, 2, 32
    x = rng.normal(size=(T, d))
    Wr = rng.normal(size=(E, d)) * 0.1
    W1 = rng.normal(size=(E, 2 * I, d)) * 0.1
    W2 = rng.normal(size=(E, d, I)) * 0.1
    a = oracle.moe_forward(x, Wr, None, W1, W2, k=k)
    b = oracle.moe_forward(x, Wr, None, W1, W2, k=k, capacity=T)
    assert np.array_equal(a["out"], b["out"])
    pa = oracle.permutation(a["idx"], E, shared=True)
    pb = oracle.permutation(a["idx"], E, shared=True, capacity=T)
    for key in ("counts", "offsets", "row_to_token", "token_to_row"):
        assert np.array_equal(pa[key], pb[key])


def test_identical_experts_closed_form_with_drops():
    # all experts equal: out = shared + (sum of the KEPT slots' p) * FFN(x)
    rng = np.random.default_rng(4)
    T, d, E, k, I, C = 30, 64, 4, 2, 32, 5
    x = oracle.bf16_round(rng.normal(size=(T, d)))
    Wr = rng.normal(size=(E, d)) * 0.3
    W1 = np.repeat(rng.normal(size=(1, 2 * I, d)) * 0.1, E, axis=0)
    W2 = np.repeat(rng.normal(size=(1, d, I)) * 0.1, E, axis=0)
    W1s = rng.normal(size=(2 * I, d)) * 0.1
    W2s = rng.normal(size=(d, I)) * 0.1
    r = oracle.moe_forward(x, Wr, None, W1, W2, W1s, W2s, k=k, capacity=C)
    assert not r["kept"].all()
    l = x @ Wr.T
    pr = np.exp(l - l.max(1, keepdims=True))
    pr /= pr.sum(1, keepdims=True)
    psum = (np.take_along_axis(pr, r["idx"], axis=1) * r["kept"]).sum(axis=1)
    g, u = x @ W1[0, :I].T, x @ W1[0, I:].T
    dense = (g / (1 + np.exp(-g)) * u) @ W2[0].T
    gs, us = x @ W1s[:I].T, x @ W1s[I:].T
    shared = (gs / (1 + np.exp(-gs)) * us) @ W2s.T
    assert np.allclose(r["out"], shared + psum[:, None] * dense, rtol=1e-12, atol=1e-12)
    # a token all of whose slots overflowed gets the shared expert alone
    gone = np.nonzero(~r["kept"].any(axis=1))[0]
    if len(gone):
        assert np.allclose(r["out"][gone], shared[gone], rtol=1e-12, atol=1e-12)


def test_capacity_from_factor():
    assert oracle.capacity_from_factor(1.0, 4096, 2, 8) == 1024
    assert oracle.capacity_from_factor(1.25, 4096, 2, 8) == 1280
    assert oracle.capacity_from_factor(1.0, 5, 1, 8) == 1      # ceil(0.625)
    assert oracle.capacity_from_factor(1e-9, 5, 1, 8) == 1     # at least one row


def test_capacity_rejects_token_subsets():
    with pytest.raises(ValueError):
        oracle.moe_forward(np.zeros((4, 8)), np.zeros((2, 8)), None, np.zeros((2, 4, 8)), np.zeros((2, 8, 2)),
                           k=1, tokens=[0, 1], capacity=1)


def test_fp8_forward_drops_the_same_pairs():
    from oracle import fp8
    rng = np.random.default_rng(8)
    T, d, E, k, I, C = 40, 256, 4, 2, 128, 9
    x = oracle.bf16_round(rng.normal(size=(T, d)))
    Wr = rng.normal(size=(E, d)) * 0.3
    W1 = rng.normal(size=(E, 2 * I, d)) * 0.05
    W2 = rng.normal(size=(E, d, I)) * 0.05
    full = fp8.moe_forward_fp8(x, Wr, None, W1, W2, k=k)
    cap = fp8.moe_forward_fp8(x, Wr, None, W1, W2, k=k, capacity=C)
    kept = oracle.kept_mask(full["idx"], C)
    assert np.array_equal(cap["kept"], kept) and not kept.all()
    # the kept pairs' contributions are those of the full forward: with every pair over capacity
    # given weight 0 instead, the same output results
    zeroed = fp8.moe_forward_fp8(x, Wr, None, W1, W2, k=k, idx=full["idx"], w=full["w"] * kept)
    assert np.allclose(cap["out"], zeroed["out"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(fp8.moe_forward_fp8(x, Wr, None, W1, W2, k=k, capacity=T)["out"], full["out"])
