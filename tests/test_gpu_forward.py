"""End-to-end parity of moe_forward (through the C ABI) against the fp64 oracle.

Small layers are compared on every output element; the full-size layers of the
grouped-GEMM pages' workloads (Mixtral-shaped, fine-grained balanced and
skewed, decode) are run in the same launch configuration bench.py times and
compared on every token, with routing and the permutation plan checked
bit-exact at full size.
Bar: relative Frobenius error <= 1e-2 (bf16 experts); routing is the
oracle's own except at near ties, where the GPU's choice is adopted.
"""
import numpy as np
import pytest
import torch

import grouped_gemm_03_b200 as gg
import oracle
from workload import make_inputs, shape_of

from _util import DeviceExperts, StreamedExperts, adopt_near_ties, check_plan_full_size, f64, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    from grouped_gemm_03_b200.build import build
    build()


def _cfg(s, out_dtype=None):
    xdt = gg.MOE_F32 if s.x_dtype == "f32" else gg.MOE_BF16
    rdt = gg.MOE_F32 if s.router_dtype == "f32" else gg.MOE_BF16
    odt = out_dtype if out_dtype is not None else (gg.MOE_F32 if s.x_dtype == "f32" else gg.MOE_BF16)
    return gg.make_config(s.T, s.d, s.E, s.k, s.inter, s.shared_inter, xdt, rdt,
                          gg.MOE_E4M3 if s.fp8 else gg.MOE_BF16, odt, s.renormalize)


def _weights(inp):
    return gg.ExpertWeights(W1=inp["W1"], W2=inp["W2"], W1s=inp["W1s"], W2s=inp["W2s"])


def _run(s, inp, **kw):
    cfg = _cfg(s, **kw)
    counts = torch.empty(s.E, dtype=torch.int32, device=DEV)
    ws = torch.empty(gg.workspace_size(cfg), dtype=torch.uint8, device=DEV)
    out = gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], _weights(inp), counts_out=counts, ws=ws)
    torch.cuda.synchronize()
    assert gg.read_device_status(ws) == 0
    return out, counts, ws


def _oracle_on(s, inp, tokens):
    """Oracle output rows for `tokens`, adopting the GPU routing at near ties."""
    xs = inp["x"][tokens]
    gidx, _, glog = gg.router_topk(xs.contiguous(), inp["W_r"], s.k, bias=inp["bias"],
                                   renormalize=s.renormalize, want_logits=True)
    r = oracle.route(xs, inp["W_r"], inp["bias"], s.k, s.renormalize)
    idx, adopted, bad = adopt_near_ties(r["logits"], r["idx"], gidx.cpu().numpy(), s.k)
    assert not bad, f"routing differs away from a tie for tokens {bad}"
    W1, W2 = DeviceExperts(inp["W1"]), DeviceExperts(inp["W2"])
    W1s = f64(inp["W1s"]) if inp["W1s"] is not None else None
    W2s = f64(inp["W2s"]) if inp["W2s"] is not None else None
    res = oracle.moe_forward(xs, inp["W_r"], inp["bias"], W1, W2, W1s, W2s, k=s.k,
                             renormalize=s.renormalize, idx=idx)
    return res, adopted


@pytest.mark.parametrize("renorm", [False, True])
def test_tiny_layer_every_element(renorm):
    s = shape_of("tiny", renormalize=renorm)
    inp = make_inputs(s, seed=1234, device=DEV)
    out, counts, _ = _run(s, inp)
    res, adopted = _oracle_on(s, inp, np.arange(s.T))
    err = rel_fro(f64(out), res["out"])
    assert err < TOL_BF16, err
    assert np.max(np.abs(f64(out) - res["out"])) < 3e-2 * np.max(np.abs(res["out"]))
    gidx, _ = gg.router_topk(inp["x"], inp["W_r"], s.k, bias=inp["bias"])
    assert np.array_equal(counts.cpu().numpy(), oracle.expert_counts(gidx.cpu().numpy(), s.E))


@pytest.mark.parametrize("T,E,k,I,shared", [(1, 8, 2, 128, True), (37, 4, 4, 256, False), (500, 16, 1, 384, True),
                                             (64, 64, 2, 128, False),
                                             # the largest layer shape the library takes: 1023 experts + shared, top-32
                                             (40, 1023, 32, 128, True)])
def test_small_ragged_layers(T, E, k, I, shared):
    s = shape_of("tiny", T=T, E=E, k=k, inter=I, shared_inter=I if shared else 0, x_dtype="bf16",
                 router_dtype="bf16")
    inp = make_inputs(s, seed=T * 7 + E, device=DEV)
    out, _, _ = _run(s, inp)
    res, _ = _oracle_on(s, inp, np.arange(T))
    assert rel_fro(f64(out), res["out"]) < TOL_BF16


def test_single_expert_top1_is_dense_ffn():
    s = shape_of("tiny", E=1, k=1, shared_inter=0, x_dtype="bf16", router_dtype="bf16")
    inp = make_inputs(s, seed=9, device=DEV)
    out, _, _ = _run(s, inp)
    ref = oracle.swiglu_ffn(f64(inp["x"]), f64(inp["W1"][0]), f64(inp["W2"][0]))
    assert rel_fro(f64(out), ref) < TOL_BF16


def test_identical_experts_closed_form():
    s = shape_of("tiny", x_dtype="bf16", router_dtype="bf16")
    inp = make_inputs(s, seed=21, device=DEV)
    inp["W1"][:] = inp["W1"][0]
    inp["W2"][:] = inp["W2"][0]
    out, _, _ = _run(s, inp)
    x = f64(inp["x"])
    p = oracle.softmax(oracle.router_logits(x, inp["W_r"], None))
    idx = oracle.topk_select(oracle.router_logits(x, inp["W_r"], None), s.k)
    psum = np.take_along_axis(p, idx, axis=1).sum(axis=1)
    dense = oracle.swiglu_ffn(x, f64(inp["W1"][0]), f64(inp["W2"][0]))
    shared = oracle.swiglu_ffn(x, f64(inp["W1s"]), f64(inp["W2s"]))
    assert rel_fro(f64(out), shared + psum[:, None] * dense) < TOL_BF16


def test_deterministic_and_graph_capturable():
    s = shape_of("tiny", T=512, x_dtype="bf16", router_dtype="bf16")
    inp = make_inputs(s, seed=4, device=DEV)
    cfg = _cfg(s)
    ws = torch.empty(gg.workspace_size(cfg), dtype=torch.uint8, device=DEV)
    w = _weights(inp)
    a = gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], w, ws=ws).clone()
    b = gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], w, ws=ws).clone()
    assert torch.equal(a, b)
    out = torch.empty_like(a)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], w, out=out, ws=ws)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, a)
    del g


def test_host_buffer_entry_matches_device_entry():
    s = shape_of("tiny", T=384, x_dtype="bf16", router_dtype="bf16")
    inp = make_inputs(s, seed=8, device=DEV)
    cfg = _cfg(s)
    dev_out = gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], _weights(inp))
    ws = torch.empty(gg.workspace_size(cfg) + gg.host_staging_size(cfg), dtype=torch.uint8, device=DEV)
    xh = inp["x"].cpu().pin_memory()
    oh = torch.empty((s.T, s.d), dtype=torch.bfloat16).pin_memory()
    gg.moe_forward_host(cfg, xh, inp["W_r"], inp["bias"], _weights(inp), oh, ws)
    torch.cuda.synchronize()
    assert torch.equal(oh, dev_out.cpu())


def test_marked_entry_matches_and_orders_its_events():
    s = shape_of("tiny", T=384, shared_inter=512, x_dtype="bf16", router_dtype="bf16")
    inp = make_inputs(s, seed=9, device=DEV)
    cfg = _cfg(s)
    ws = torch.empty(gg.workspace_size(cfg), dtype=torch.uint8, device=DEV)
    ref = gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], _weights(inp), ws=ws).clone()
    out = torch.empty_like(ref)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    gg.moe_forward_marked(cfg, inp["x"], inp["W_r"], inp["bias"], _weights(inp), evs, out, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    gaps = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
    assert all(g >= 0 for g in gaps) and sum(gaps) > 0


def test_empty_batch():
    s = shape_of("tiny", T=0, x_dtype="bf16", router_dtype="bf16")
    cfg = _cfg(s)
    inp = make_inputs(shape_of("tiny", T=1, x_dtype="bf16", router_dtype="bf16"), device=DEV)
    ws = torch.empty(gg.workspace_size(cfg), dtype=torch.uint8, device=DEV)
    counts = torch.full((s.E,), 9, dtype=torch.int32, device=DEV)
    out = gg.moe_forward(cfg, inp["x"][:0], inp["W_r"], None, _weights(inp), counts_out=counts, ws=ws)
    assert out.shape == (0, s.d)
    assert torch.all(counts == 0)


# ---------------------------------------------------------------- full-size workloads
# The layers bench.py times, in the same launch configuration, compared with
# the oracle on EVERY token; routing and the permutation plan are checked
# bit-exact at full size against the oracle's plan from the GPU's logits.
FULL = ["mixtral", "fine", "fine_skew", "decode"]
TOL_TOKEN = 2e-2  # any single token's relative error (the Frobenius bar is over all tokens)


@pytest.mark.parametrize("name", FULL)
def test_full_size_every_token(name):
    s = shape_of(name)
    inp = make_inputs(s, seed=1234, device=DEV)
    gidx = check_plan_full_size(gg, s, inp)
    out, counts, _ = _run(s, inp)
    assert np.array_equal(counts.cpu().numpy(), oracle.expert_counts(gidx, s.E))
    # oracle routing, adopting the GPU's choice only at near ties
    r = oracle.route(inp["x"], inp["W_r"], inp["bias"], s.k, s.renormalize)
    idx, adopted, bad = adopt_near_ties(r["logits"], r["idx"], gidx, s.k)
    assert not bad, f"routing differs away from a tie for tokens {bad[:10]}"
    keep = s.E * 3 * s.inter * s.d * 8 <= (16 << 30)  # fp64 copies of every expert fit the host
    W1, W2 = StreamedExperts(inp["W1"], keep), StreamedExperts(inp["W2"], keep)
    W1s = f64(inp["W1s"]) if inp["W1s"] is not None else None
    W2s = f64(inp["W2s"]) if inp["W2s"] is not None else None
    ref = oracle.moe_forward(inp["x"], inp["W_r"], inp["bias"], W1, W2, W1s, W2s, k=s.k,
                             renormalize=s.renormalize, idx=idx)["out"]
    got = f64(out)
    err = rel_fro(got, ref)
    assert err < TOL_BF16, (err, len(adopted))
    per_token = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    assert per_token.max() < TOL_TOKEN, (int(per_token.argmax()), per_token.max())
    del inp, W1, W2
    torch.cuda.empty_cache()
