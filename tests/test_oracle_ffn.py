"""Pins of the oracle's expert FFN and combine.

  * the hand-worked 2-expert / top-1 / 4-token case (tests/golden), whose
    every value was derived on paper (Dense GEMM -> GroupedGEMM -> TP MoE,
    §4.3 asks for exactly this check);
  * E = 1, k = 1 without a shared expert is a dense SiLU-gated FFN, checked
    against a naive triple loop written here;
  * with all experts identical, out = FFN_shared(x) + (sum of selected p)
    * FFN(x); at k = E that is FFN_shared + FFN (MegaMoE walk-through §2.1);
  * W2 = 0 leaves only the shared expert; doubling W2 doubles the routed part;
  * restricting to a token subset gives the same rows as the full forward.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def naive_swiglu(x, W1, W2):
    """Triple loop: h_i = silu(sum_c W1[i,c] x_c) * sum_c W1[I+i,c] x_c; y_o = sum_i W2[o,i] h_i."""
    I = len(W1) // 2
    out = []
    for row in x:
        h = []
        for i in range(I):
            g = math.fsum(W1[i][c] * row[c] for c in range(len(row)))
            u = math.fsum(W1[I + i][c] * row[c] for c in range(len(row)))
            h.append(g / (1.0 + math.exp(-g)) * u)
        out.append([math.fsum(W2[o][i] * h[i] for i in range(I)) for o in range(len(W2))])
    return np.array(out)


def _layer(T=12, d=16, E=4, I=8, shared=True, seed=0):
    rng = np.random.default_rng(seed)
    # x on the bf16 grid so that the experts' bf16 rounding is the identity here
    x = oracle.bf16_round(rng.normal(size=(T, d)))
    Wr = rng.normal(size=(E, d)) * 0.5
    W1 = rng.normal(size=(E, 2 * I, d)) * 0.3
    W2 = rng.normal(size=(E, d, I)) * 0.3
    W1s = rng.normal(size=(2 * I, d)) * 0.3 if shared else None
    W2s = rng.normal(size=(d, I)) * 0.3 if shared else None
    return x, Wr, W1, W2, W1s, W2s


@pytest.mark.parametrize("renorm", [False, True])
def test_hand_worked_two_expert_top1(renorm):
    g = json.load(open(os.path.join(GOLDEN, "hand_2expert_top1.json")))
    L = math.log(3.0)
    x = np.array(g["x"], dtype=np.float64)
    Wr = np.array(g["W_r_over_L"], dtype=np.float64) * L
    W1 = np.array(g["W1_over_L"], dtype=np.float64) * L
    W2 = np.array(g["W2"], dtype=np.float64)
    W1s = np.array(g["W1s_over_L"], dtype=np.float64) * L
    W2s = np.array(g["W2s"], dtype=np.float64)
    ex = g["expected"]
    r = oracle.moe_forward(x, Wr, None, W1, W2, W1s, W2s, k=1, renormalize=renorm)
    assert r["idx"].tolist() == ex["idx"]
    p_sel = np.take_along_axis(r["p"], r["idx"], axis=1)
    assert np.allclose(p_sel, [[a / b] for a, b in ex["p_selected"]], rtol=1e-14)
    key = "out_over_L2_renormalized" if renorm else "out_over_L2_raw"
    want = np.array([[a / b * L * L for a, b in row] for row in ex[key]])
    assert np.allclose(r["out"], want, rtol=1e-13, atol=1e-14)
    pm = oracle.permutation(r["idx"], g["E"], shared=True)
    assert pm["counts"].tolist() == ex["counts"]
    assert pm["offsets"].tolist() == ex["offsets_with_shared"]
    assert pm["token_to_row"].tolist() == ex["token_to_row"]
    assert pm["row_to_token"].tolist() == ex["row_to_token"]


def test_single_expert_is_dense_swiglu():
    x, Wr, W1, W2, _, _ = _layer(T=6, d=8, E=1, I=5, shared=False, seed=1)
    r = oracle.moe_forward(x, Wr, None, W1, W2, k=1)
    assert np.all(r["w"] == 1.0)
    want = naive_swiglu(x.tolist(), W1[0].tolist(), W2[0].tolist())
    assert np.allclose(r["out"], want, rtol=1e-12, atol=1e-13)


def _brute_psum(x, Wr, k):
    out = []
    for row in x:
        l = [math.fsum(Wr[e][c] * row[c] for c in range(len(row))) for e in range(len(Wr))]
        z = [math.exp(v - max(l)) for v in l]
        s = math.fsum(z)
        top = sorted(range(len(l)), key=lambda e: (-l[e], e))[:k]
        out.append(math.fsum(z[e] / s for e in top))
    return np.array(out)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_identical_experts_closed_form(k):
    x, Wr, W1, W2, W1s, W2s = _layer(T=10, d=12, E=4, I=6, seed=2)
    W1[:] = W1[0]
    W2[:] = W2[0]
    r = oracle.moe_forward(x, Wr, None, W1, W2, W1s, W2s, k=k)
    dense = naive_swiglu(x.tolist(), W1[0].tolist(), W2[0].tolist())
    shared = naive_swiglu(x.tolist(), W1s.tolist(), W2s.tolist())
    want = shared + _brute_psum(x.tolist(), Wr.tolist(), k)[:, None] * dense
    assert np.allclose(r["out"], want, rtol=1e-11, atol=1e-12)
    if k == 4:  # k = E: all probability mass
        assert np.allclose(r["out"], shared + dense, rtol=1e-11, atol=1e-12)


def test_zero_down_projection_leaves_shared_expert():
    x, Wr, W1, W2, W1s, W2s = _layer(seed=3)
    r = oracle.moe_forward(x, Wr, None, W1, np.zeros_like(W2), W1s, W2s, k=2)
    shared = naive_swiglu(x.tolist(), W1s.tolist(), W2s.tolist())
    assert np.allclose(r["out"], shared, rtol=1e-12, atol=1e-13)


def test_routed_part_is_linear_in_down_projection():
    x, Wr, W1, W2, W1s, W2s = _layer(seed=4)
    base = oracle.moe_forward(x, Wr, None, W1, W2, W1s, W2s, k=2)["out"]
    dbl = oracle.moe_forward(x, Wr, None, W1, 2 * W2, W1s, W2s, k=2)["out"]
    shared = naive_swiglu(x.tolist(), W1s.tolist(), W2s.tolist())
    assert np.allclose(dbl - shared, 2 * (base - shared), rtol=1e-11, atol=1e-12)


def test_token_subset_matches_full_forward():
    x, Wr, W1, W2, W1s, W2s = _layer(T=16, seed=5)
    full = oracle.moe_forward(x, Wr, None, W1, W2, W1s, W2s, k=2)
    sub = [3, 0, 11]
    part = oracle.moe_forward(x, Wr, None, W1, W2, W1s, W2s, k=2, tokens=sub)
    assert np.array_equal(part["idx"], full["idx"][sub])
    assert np.allclose(part["out"], full["out"][sub], rtol=1e-13, atol=1e-14)


def test_experts_consume_bf16_rounded_activations():
    x, Wr, W1, W2, _, _ = _layer(T=4, d=8, E=1, I=4, shared=False, seed=6)
    xf = x + 1e-3  # off the bf16 grid
    r = oracle.moe_forward(xf, Wr, None, W1, W2, k=1)
    want = naive_swiglu(oracle.bf16_round(xf).tolist(), W1[0].tolist(), W2[0].tolist())
    assert np.allclose(r["out"], want, rtol=1e-12, atol=1e-13)
