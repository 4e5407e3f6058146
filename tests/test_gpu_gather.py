"""Permute in the load (survey row f1): the grouped GEMM gathers its A rows
through row_to_token (TMA tile::gather4), so the expert-ordered copy of the
tokens is never written.  "Dense GEMM -> GroupedGEMM -> TP MoE" §2.2 names
the prefix sum and scatter (steps 3-4) as hotspots; "MegaMoE ..." §4.3 lays
the tokens of one expert out contiguously, which the gather reproduces in
shared memory instead of HBM.

The gathered GEMM runs the same kernel and tiles as the GEMM on a
materialised copy, so the two must agree bit for bit; that copy is itself
checked against the fp64 oracle elsewhere (test_gpu_kernels / _fp8 / _mx).
The whole layer (which gathers on the fine-grained and tiny shapes) is
compared with the oracle in test_gpu_forward / _fp8 / _mx / _capacity.
"""
import numpy as np
import pytest
import torch

import grouped_gemm_03_b200 as gg
from oracle import fp8 as ofp8

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from grouped_gemm_03_b200.build import build
    build()


def _plan(T, E, k, seed, shared=True):
    g = torch.Generator(device="cpu").manual_seed(seed)
    logits = torch.randn((T, E), generator=g) - 0.7 * torch.log1p(torch.arange(E, dtype=torch.float32))
    idx = torch.topk(logits, k, dim=1).indices.to(torch.int32).to(DEV).contiguous()
    x = torch.randn((T, 8 * 128), generator=g).to(torch.bfloat16).to(DEV)
    return gg.permute(x, idx, E, append_shared=shared)


@pytest.mark.parametrize("T,E,k,N,K,epi,kind", [
    (300, 8, 2, 256, 512, gg.EPI_SILU_GATE, "bf16"),
    (777, 16, 4, 512, 256, gg.EPI_NONE, "bf16"),
    (200, 32, 8, 256, 384, gg.EPI_SILU_GATE, "e4m3"),
    (200, 32, 8, 256, 384, gg.EPI_SILU_GATE, "mx"),
    (513, 8, 2, 512, 256, gg.EPI_NONE, "mx"),
])
def test_gathered_gemm_equals_gemm_on_the_permuted_copy(T, E, k, N, K, epi, kind):
    plan = _plan(T, E, k, seed=T + N)
    r2t = plan["row_to_token"]
    rows = r2t.numel()
    offsets = plan["offsets"]
    G = E + 1  # the routed experts and the shared one, as one set of groups
    Nb = 2 * N if epi == gg.EPI_SILU_GATE else N
    g = torch.Generator(device=DEV).manual_seed(K)
    x = torch.randn((T, K), device=DEV, generator=g)
    B = (torch.randn((G, Nb, K), device=DEV, generator=g) * 0.05).to(torch.bfloat16)
    mx = kind == "mx"
    if kind == "bf16":
        A_src, A_s, Bq, Bs = x.to(torch.bfloat16), None, B, None
        cdt = torch.bfloat16
    else:
        q, sc = ofp8.quantize_1x128(x.cpu().numpy(), pow2=mx)
        A_src = torch.from_numpy(q).to(DEV)
        A_s = torch.from_numpy(np.ascontiguousarray(sc.T)).to(DEV)
        Bq, Bs = (gg.quantize_weights_mx if mx else gg.quantize_weights_fp8)(B)
        cdt = torch.uint8 if epi == gg.EPI_SILU_GATE else torch.bfloat16
    # the materialised copy the gather replaces: A_p[r] = A_src[row_to_token[r]]
    r = r2t.long()
    A_p = A_src[r].contiguous()
    A_ps = A_s[:, r].contiguous() if A_s is not None else None
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    want = gg.grouped_gemm(A_p, Bq, offsets, N, epilogue=epi, c_dtype=cdt, A_scales=A_ps, B_scales=Bs, ws=ws, mx=mx)
    assert gg.read_device_status(ws) == 0
    got = gg.grouped_gemm_gather(A_src, r2t, Bq, offsets, N, epilogue=epi, c_dtype=cdt, A_scales=A_s, B_scales=Bs,
                                 ws=ws, mx=mx)
    assert gg.read_device_status(ws) == 0
    used = int(offsets[-1].item())
    if isinstance(want, tuple):
        assert torch.equal(got[0][:used], want[0][:used]) and torch.equal(got[1][:, :used], want[1][:, :used])
    else:
        assert torch.equal(got[:used], want[:used])


def test_gathered_gemm_with_overflowed_rows_and_fp32_out_rules():
    # capacity leaves rows with row_to_token = -1 past the used ones: they belong to no group
    T, E, k, K, N = 400, 8, 2, 256, 256
    g = torch.Generator(device="cpu").manual_seed(9)
    logits = torch.randn((T, E), generator=g) - 2.0 * torch.log1p(torch.arange(E, dtype=torch.float32))
    idx = torch.topk(logits, k, dim=1).indices.to(torch.int32).to(DEV).contiguous()
    x = torch.randn((T, K), device=DEV).to(torch.bfloat16)
    plan = gg.permute(x, idx, E, append_shared=True, capacity=40)
    r2t = plan["row_to_token"]
    assert (r2t < 0).any()
    B = (torch.randn((E + 1, N, K), device=DEV) * 0.05).to(torch.bfloat16)
    got = gg.grouped_gemm_gather(x, r2t, B, plan["offsets"], N)
    r = r2t.long().clamp(min=0)
    want = gg.grouped_gemm(x[r].contiguous(), B, plan["offsets"], N)
    used = int(plan["offsets"][-1].item())
    assert torch.equal(got[:used], want[:used])
    with pytest.raises(gg.MoEError):  # fp32 C runs on no gathering kernel
        gg.grouped_gemm_gather(x, r2t, B, plan["offsets"], N, c_dtype=torch.float32)


@pytest.mark.parametrize("name,over", [
    ("tiny", dict()),                                                        # fp32 x: cast once per token
    ("tiny", dict(T=700, E=16, k=4, x_dtype="bf16", router_dtype="bf16")),   # bf16 x read as stored
    ("tiny", dict(T=300, E=8, k=2, inter=256, shared_inter=256, fp8=True)),  # E4M3 quantised once per token
    ("tiny", dict(T=300, E=8, k=2, inter=256, shared_inter=256, fp8=True, mx=True, x_dtype="bf16",
                  router_dtype="bf16")),
])
def test_forward_with_gathered_up_gemm_equals_the_default(name, over):
    from workload import make_inputs, shape_of
    s = shape_of(name, **over)
    inp = make_inputs(s, seed=5, device=DEV)
    xdt = gg.MOE_F32 if s.x_dtype == "f32" else gg.MOE_BF16
    rdt = gg.MOE_F32 if s.router_dtype == "f32" else gg.MOE_BF16
    edt = (gg.MOE_MXE4M3 if s.mx else gg.MOE_E4M3) if s.fp8 else gg.MOE_BF16
    if s.fp8:
        q = gg.quantize_weights_mx if s.mx else gg.quantize_weights_fp8
        W1q, W1s = q(inp["W1"])
        W2q, W2s = q(inp["W2"])
        w = gg.ExpertWeights(W1=W1q, W2=W2q, W1_scales=W1s, W2_scales=W2s)
        w.W1s, w.W1s_scales = q(inp["W1s"])
        w.W2s, w.W2s_scales = q(inp["W2s"])
    else:
        w = gg.ExpertWeights(W1=inp["W1"], W2=inp["W2"], W1s=inp["W1s"], W2s=inp["W2s"])
    outs = []
    for flags in (0, gg.MOE_FLAG_GATHER_A):
        cfg = gg.make_config(s.T, s.d, s.E, s.k, s.inter, s.shared_inter, xdt, rdt, edt, xdt, flags=flags)
        ws = torch.empty(gg.workspace_size(cfg), dtype=torch.uint8, device=DEV)
        outs.append(gg.moe_forward(cfg, inp["x"], inp["W_r"], inp["bias"], w, ws=ws).clone())
        assert gg.read_device_status(ws) == 0
    assert torch.equal(outs[0], outs[1])
