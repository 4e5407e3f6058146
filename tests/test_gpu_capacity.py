"""Capacity limit with an overflow path, through the C ABI, against the oracle.

"Dense GEMM -> GroupedGEMM -> TP MoE" §5.1: a capacity factor caps each
expert's tokens at inference and the tokens over it take a fallback path.
The permutation plan with a capacity (which pairs are kept, their rows, the
shared rows after the kept ones, -1 for the overflow) is compared bit for
bit with the oracle's plan from the same top-k indices; the layer forward
with a capacity is compared with the oracle forward that drops the same
pairs (relative Frobenius <= 1e-2, bf16 experts; <= 3e-2, E4M3 experts).
"""
import numpy as np
import pytest
import torch

import grouped_gemm_03_b200 as gg
import oracle
from oracle import fp8 as ofp8
from workload import make_inputs, shape_of

from _util import StreamedExperts, adopt_near_ties, f64, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from grouped_gemm_03_b200.build import build
    build()


def _skewed_idx(T, E, k, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    logits = torch.randn((T, E), generator=g) - 1.2 * torch.log1p(torch.arange(E, dtype=torch.float32))
    return torch.topk(logits, k, dim=1).indices.to(torch.int32)


@pytest.mark.parametrize("T,E,k,d,C,shared,fp8", [
    (300, 8, 2, 256, 40, True, False),
    (1000, 64, 4, 512, 50, False, False),
    (77, 4, 2, 256, 1, True, True),          # capacity 1: one pair per expert survives
    (4096, 256, 8, 1024, 128, True, True),
    (513, 16, 3, 384, 10000, True, False),   # a capacity no expert reaches: nothing dropped
])
def test_permute_with_capacity_matches_the_oracle_plan(T, E, k, d, C, shared, fp8):
    idx = _skewed_idx(T, E, k, seed=T + C)
    x = torch.randn((T, d), generator=torch.Generator(device="cpu").manual_seed(C)).to(torch.bfloat16).to(DEV)
    plan = gg.permute(x, idx.to(DEV).contiguous(), E, append_shared=shared, fp8=fp8, capacity=C)
    assert gg.read_device_status(plan["ws"]) == 0
    want = oracle.permutation(idx.numpy(), E, shared=shared, capacity=C)
    for key in ("counts", "offsets", "row_to_token", "token_to_row"):
        got = plan[key].cpu().numpy().astype(np.int64).reshape(want[key].shape)
        assert np.array_equal(got, want[key]), key
    used = int(want["offsets"][-1])
    r2t = want["row_to_token"][:used]
    if fp8:
        xq, sx = ofp8.quantize_1x128(f64(x).astype(np.float32))
        assert np.array_equal(plan["xp"].cpu().numpy()[:used], xq[r2t])
        assert np.array_equal(plan["xp_scales"].cpu().numpy().T[:used], sx[r2t])
    else:
        assert torch.equal(plan["xp"][:used].cpu(), x.cpu()[torch.from_numpy(r2t)])


def test_combine_plan_skips_overflow_and_finds_the_shared_rows():
    T, E, k, d, C = 200, 8, 2, 512, 20
    idx = _skewed_idx(T, E, k, seed=3)
    plan_want = oracle.permutation(idx.numpy(), E, shared=True, capacity=C)
    x = torch.randn((T, d), device=DEV).to(torch.bfloat16)
    plan = gg.permute(x, idx.to(DEV).contiguous(), E, append_shared=True, capacity=C)
    rows = T * k + T
    Y = torch.randn((rows, d), device=DEV).to(torch.bfloat16)
    w = torch.rand((T, k), device=DEV)
    out = gg.combine(Y, plan["token_to_row"], w, True, out_dtype=torch.float32, offsets=plan["offsets"])
    Yh, wh = f64(Y), f64(w)
    used = int(plan_want["offsets"][E])
    ref = Yh[used:used + T].copy()
    for t in range(T):
        for j in range(k):
            r = plan_want["token_to_row"][t, j]
            if r >= 0:
                ref[t] += wh[t, j] * Yh[r]
    assert rel_fro(f64(out), ref) < 1e-6


def _cfg(s, capacity, fp8=False):
    xdt = gg.MOE_F32 if s.x_dtype == "f32" else gg.MOE_BF16
    rdt = gg.MOE_F32 if s.router_dtype == "f32" else gg.MOE_BF16
    return gg.make_config(s.T, s.d, s.E, s.k, s.inter, s.shared_inter, xdt, rdt,
                          gg.MOE_E4M3 if fp8 else gg.MOE_BF16, xdt, s.renormalize, capacity=capacity)


def _layer(s, inp, capacity, fp8=False):
    cfg = _cfg(s, capacity, fp8)
    ws = torch.empty(gg.workspace_size(cfg), dtype=torch.uint8, device=DEV)
    counts = torch.empty(s.E, dtype=torch.int32, device=DEV)
    if fp8:
        W1q, W1sc = gg.quantize_weights_fp8(inp["W1"])
        W2q, W2sc = gg.quantize_weights_fp8(inp["W2"])
        w = gg.ExpertWeights(W1=W1q, W2=W2q, W1_scales=W1sc, W2_scales=W2sc)
        if s.shared_inter:
            w.W1s, w.W1s_scales = gg.quantize_weights_fp8(inp["W1s"])
            w.W2s, w.W2s_scales = gg.quantize_weights_fp8(inp["W2s"])
    else:
        w = gg.ExpertWeights(W1=inp["W1"], W2=inp["W2"], W1s=inp["W1s"], W2s=inp["W2s"])
    out = gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], w, counts_out=counts, ws=ws)
    torch.cuda.synchronize()
    assert gg.read_device_status(ws) == 0
    return out, counts


def _gpu_idx(s, inp):
    gidx, _ = gg.router_topk(inp["x"], inp["W_r"], s.k, bias=inp["bias"], renormalize=s.renormalize)
    return gidx.cpu().numpy()


@pytest.mark.parametrize("name,over,factor,fp8", [
    ("tiny", dict(), 0.6, False),
    ("tiny", dict(T=500, E=16, k=4, x_dtype="bf16", router_dtype="bf16", zipf_s=1.5), 1.0, False),
    ("tiny", dict(T=300, E=8, k=2, shared_inter=0, inter=256, zipf_s=2.0), 0.5, True),
    ("decode", dict(), 1.0, False),
])
def test_layer_with_capacity_every_element(name, over, factor, fp8):
    s = shape_of(name, **over)
    inp = make_inputs(s, seed=77, device=DEV)
    C = gg.capacity_from_factor(factor, s.T, s.k, s.E)
    out, counts = _layer(s, inp, C, fp8)
    gidx = _gpu_idx(s, inp)
    r = oracle.route(inp["x"], inp["W_r"], inp["bias"], s.k, s.renormalize)
    idx, _, bad = adopt_near_ties(r["logits"], r["idx"], gidx, s.k)
    assert not bad
    plan = oracle.permutation(idx, s.E, shared=bool(s.shared_inter), capacity=C)
    assert np.array_equal(counts.cpu().numpy(), plan["counts"])
    assert not plan["kept"].all(), "the case must overflow some expert"
    W1s = f64(inp["W1s"]) if inp["W1s"] is not None else None
    W2s = f64(inp["W2s"]) if inp["W2s"] is not None else None
    if fp8:
        ref = ofp8.moe_forward_fp8(inp["x"], inp["W_r"], inp["bias"], StreamedExperts(inp["W1"]),
                                   StreamedExperts(inp["W2"]), W1s, W2s, k=s.k, renormalize=s.renormalize,
                                   idx=idx, capacity=C)["out"]
        tol = 3e-2
    else:
        ref = oracle.moe_forward(inp["x"], inp["W_r"], inp["bias"], StreamedExperts(inp["W1"], True),
                                 StreamedExperts(inp["W2"], True), W1s, W2s, k=s.k, renormalize=s.renormalize,
                                 idx=idx, capacity=C)["out"]
        tol = 1e-2
    err = rel_fro(f64(out), ref)
    assert err < tol, err


def test_mixtral_layer_at_capacity_factor_one_every_token():
    s = shape_of("mixtral")
    inp = make_inputs(s, seed=1234, device=DEV)
    C = gg.capacity_from_factor(1.0, s.T, s.k, s.E)   # 1024 rows; the Zipf-hot experts take up to ~2100
    out, counts = _layer(s, inp, C)
    gidx = _gpu_idx(s, inp)
    r = oracle.route(inp["x"], inp["W_r"], inp["bias"], s.k, s.renormalize)
    idx, _, bad = adopt_near_ties(r["logits"], r["idx"], gidx, s.k)
    assert not bad
    plan = oracle.permutation(idx, s.E, capacity=C)
    assert np.array_equal(counts.cpu().numpy(), plan["counts"]) and counts.max().item() == C
    ref = oracle.moe_forward(inp["x"], inp["W_r"], inp["bias"], StreamedExperts(inp["W1"], True),
                             StreamedExperts(inp["W2"], True), None, None, k=s.k, idx=idx, capacity=C)["out"]
    got = f64(out)
    assert rel_fro(got, ref) < 1e-2
    gone = ~plan["kept"].any(axis=1)  # tokens whose every slot overflowed: no expert, no shared -> zero
    assert np.all(got[gone] == 0)
