"""Per-kernel parity of the CUDA path (through the C ABI) against the oracle.

Bars: routing indices, counts, offsets, the permutation and every quantised
byte / scale are bit-exact; floating-point outputs are within the stated
tolerances (bf16 storage of the results bounds them at a few 2^-9).
"""
import numpy as np
import pytest
import torch

import grouped_gemm_03_b200 as gg
import oracle
from oracle import fp8 as ofp8
from workload import make_inputs, make_router_logits, shape_of

from _util import f64, rel_fro

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from grouped_gemm_03_b200.build import build
    build()
    n, major, minor = gg.device_info()
    assert major == 10, f"needs an sm_100 device, got sm_{major}{minor}"


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- top-k of logits
@pytest.mark.parametrize("N,E,k,dtype", [(4096, 128, 4, torch.float16), (65536, 128, 4, torch.float16),
                                         (777, 64, 2, torch.float32), (300, 256, 8, torch.bfloat16),
                                         (129, 8, 2, torch.float16), (64, 40, 3, torch.float32),
                                         # few experts and many tokens: one or two experts per lane
                                         (2048, 8, 2, torch.float16), (3001, 16, 4, torch.bfloat16),
                                         (1500, 32, 8, torch.float32), (1024, 24, 3, torch.float32),
                                         (4096, 7, 1, torch.float16),
                                         # the largest supported: 1024 experts, top-32
                                         (300, 1024, 32, torch.float32), (129, 1000, 17, torch.bfloat16),
                                         # few tokens, 65..128 experts: 16 lanes of 8 experts per token
                                         (500, 100, 4, torch.float16), (200, 128, 6, torch.bfloat16)])
@pytest.mark.parametrize("renorm", [False, True])
def test_topk_logits(N, E, k, dtype, renorm):
    l = make_router_logits(N, E, seed=5, device=DEV, dtype=dtype)
    idx, w = gg.topk_logits(l, k, renormalize=renorm)
    torch.cuda.synchronize()
    lf = f64(l)
    want_idx = oracle.topk_select(lf, k)
    assert np.array_equal(idx.cpu().numpy(), want_idx)
    want_w = oracle.gate_weights(oracle.softmax(lf), want_idx, renorm)
    np.testing.assert_allclose(w.cpu().numpy(), want_w, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("E,k,dtype", [(8, 1, torch.float16), (24, 3, torch.bfloat16), (56, 8, torch.float16),
                                       (128, 4, torch.float16), (200, 5, torch.bfloat16), (256, 8, torch.float16)])
def test_topk_rows_with_many_ties(E, k, dtype):
    # 16-bit logits, E % 8 == 0, E <= 256, k <= 8 run one thread per token; integer-valued logits tie
    # often, so the order (logit descending, expert ascending) is exercised on every token
    g = torch.Generator(device=DEV).manual_seed(E + k)
    l = torch.randint(-3, 4, (5000, E), device=DEV, generator=g).to(dtype)
    for renorm in (False, True):
        idx, w = gg.topk_logits(l, k, renormalize=renorm)
        torch.cuda.synchronize()
        lf = f64(l)
        want = oracle.topk_select(lf, k)
        assert np.array_equal(idx.cpu().numpy(), want)
        np.testing.assert_allclose(w.cpu().numpy(), oracle.gate_weights(oracle.softmax(lf), want, renorm),
                                   rtol=2e-6, atol=1e-7)


def test_topk_logits_ties_take_lower_index():
    l = torch.zeros((64, 32), dtype=torch.float16, device=DEV)
    l[:, 5] = 1.0
    l[:, 9] = 1.0
    l[:, 20] = 1.0
    idx, w = gg.topk_logits(l, 3)
    assert (idx.cpu() == torch.tensor([5, 9, 20], dtype=torch.int32)).all()
    idx1, _ = gg.topk_logits(torch.zeros((8, 64), dtype=torch.float32, device=DEV), 2)
    assert (idx1.cpu() == torch.tensor([0, 1], dtype=torch.int32)).all()


@pytest.mark.parametrize("dtype,E", [(torch.float16, 64), (torch.bfloat16, 128), (torch.float32, 40)])
def test_topk_signed_zeros_tie(dtype, E):
    # -0 and +0 compare equal, so they tie and the lower expert comes first,
    # whichever sign it carries (rows of -1, -0, +0 and -2: the top picks are zeros)
    g = np.random.default_rng(E)
    vals = np.array([-1.0, -0.0, 0.0, -2.0])
    l = vals[g.integers(0, 4, size=(700, E))]
    l[:, 0] = -0.0  # every row has zeros of both signs
    l[:, 1] = 0.0
    lt = torch.tensor(l, dtype=dtype, device=DEV)
    for k in (1, 3, 6):
        idx, w = gg.topk_logits(lt, k)
        torch.cuda.synchronize()
        want = oracle.topk_select(l, k)
        assert np.array_equal(idx.cpu().numpy(), want)
        np.testing.assert_allclose(w.cpu().numpy(), oracle.gate_weights(oracle.softmax(l), want), rtol=2e-6,
                                   atol=1e-7)


def test_topk_k1_renormalised_is_one():
    l = make_router_logits(1000, 16, seed=2, device=DEV, dtype=torch.float32)
    _, w = gg.topk_logits(l, 1, renormalize=True)
    assert torch.all(w == 1.0)


# ---------------------------------------------------------------- router
@pytest.mark.parametrize("name,T", [("tiny", 256), ("mixtral", 512), ("decode", 128), ("fine", 256), ("fine", 1000),
                                    ("fine", 4096), ("mixtral", 4096), ("tiny", 77)])
@pytest.mark.parametrize("renorm", [False, True])
def test_router_topk(name, T, renorm):
    s = shape_of(name, T=T)
    inp = make_inputs(s, seed=11, device=DEV, experts=False)
    idx, w, logits = gg.router_topk(inp["x"], inp["W_r"], s.k, bias=inp["bias"], renormalize=renorm,
                                    want_logits=True)
    torch.cuda.synchronize()
    gl = f64(logits)
    # logits close to the fp64 definition
    ol = oracle.router_logits(inp["x"], inp["W_r"], inp["bias"])
    np.testing.assert_allclose(gl, ol, rtol=1e-4, atol=2e-5 * np.sqrt(s.d))
    # selection bit-exact given the GPU's logits
    want = oracle.topk_select(gl, s.k)
    assert np.array_equal(idx.cpu().numpy(), want)
    want_w = oracle.gate_weights(oracle.softmax(gl), want, renorm)
    np.testing.assert_allclose(w.cpu().numpy(), want_w, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T,d,E,k,xdt,wdt", [(1000, 264, 5, 2, torch.bfloat16, torch.bfloat16),
                                           (333, 4096, 16, 4, torch.bfloat16, torch.bfloat16),
                                           (70, 1024, 33, 3, torch.bfloat16, torch.bfloat16),
                                           (129, 512, 64, 8, torch.float32, torch.bfloat16),
                                           (513, 256, 8, 2, torch.bfloat16, torch.float32),
                                           (1, 8, 7, 7, torch.float32, torch.float32),
                                           (3, 8, 4, 2, torch.bfloat16, torch.bfloat16),
                                           (200, 2048, 100, 6, torch.bfloat16, torch.bfloat16),
                                           (20000, 512, 256, 8, torch.bfloat16, torch.bfloat16),
                                           (6000, 512, 32, 4, torch.bfloat16, torch.bfloat16),  # 2-CTA clusters
                                           (20000, 256, 8, 2, torch.bfloat16, torch.bfloat16),
                                           # bf16 outside the tensor-core router's range: E > 256 (split-K
                                           # logits + selection kernel), k > 8 with E > 16 (SIMT logits +
                                           # selection), k > 8 with E <= 16 (the SIMT one-launch router)
                                           (600, 1024, 300, 6, torch.bfloat16, torch.bfloat16),
                                           (200, 512, 64, 12, torch.bfloat16, torch.bfloat16),
                                           (300, 512, 16, 10, torch.bfloat16, torch.bfloat16)])
def test_router_ragged_shapes(T, d, E, k, xdt, wdt):
    # ragged d, E not a power of two, mixed operand types; bf16 operands with
    # E <= 256 and k <= 8 run the tensor-core router (one cluster of up to 8
    # CTAs per 128 tokens; a single CTA per tile once 128-token tiles fill the SMs)
    g = torch.Generator(device=DEV).manual_seed(T + d + E)
    x = torch.randn((T, d), device=DEV, generator=g).to(xdt)
    W = (torch.randn((E, d), device=DEV, generator=g) * 0.05).to(wdt)
    bias = torch.randn(E, device=DEV, generator=g)
    idx, w, logits = gg.router_topk(x, W, k, bias=bias, want_logits=True)
    torch.cuda.synchronize()
    gl = f64(logits)
    ol = oracle.router_logits(x, W, bias)
    np.testing.assert_allclose(gl, ol, rtol=1e-4, atol=2e-5 * np.sqrt(d))
    want = oracle.topk_select(gl, k)
    assert np.array_equal(idx.cpu().numpy(), want)
    np.testing.assert_allclose(w.cpu().numpy(), oracle.gate_weights(oracle.softmax(gl), want), rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("E,k", [(8, 2), (32, 5), (64, 8)])
def test_router_ties_go_to_the_lower_index(E, k):
    # every expert row equal: all logits tie, so the selection is experts 0..k-1 in order
    x = torch.randn((300, 512), device=DEV).to(torch.bfloat16)
    W = (torch.randn((1, 512), device=DEV) * 0.05).to(torch.bfloat16).repeat(E, 1).contiguous()
    idx, w = gg.router_topk(x, W, k)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), np.tile(np.arange(k), (300, 1)))
    np.testing.assert_allclose(w.cpu().numpy(), 1.0 / E, rtol=1e-6)


# ---------------------------------------------------------------- permute
def _check_plan(res, idx_np, E, shared):
    plan = oracle.permutation(idx_np, E, shared=shared)
    assert np.array_equal(res["counts"].cpu().numpy(), plan["counts"])
    assert np.array_equal(res["offsets"].cpu().numpy(), plan["offsets"])
    assert np.array_equal(res["row_to_token"].cpu().numpy(), plan["row_to_token"])
    assert np.array_equal(res["token_to_row"].cpu().numpy(), plan["token_to_row"])
    return plan


def _random_routing(T, E, k, seed, skew=0.0):
    l = _rng(seed).normal(size=(T, E)) - skew * np.log1p(np.arange(E))[None, :]
    return oracle.topk_select(l, k)


@pytest.mark.parametrize("T,E,k,shared,xdt", [(256, 8, 2, True, torch.float32), (77, 8, 2, False, torch.bfloat16),
                                              (1000, 256, 8, True, torch.bfloat16), (33, 64, 2, False, torch.float32),
                                              (4096, 8, 2, False, torch.bfloat16), (5, 4, 4, True, torch.bfloat16),
                                              (1, 16, 3, False, torch.bfloat16),
                                              # the largest supported: 1024 experts (1023 with the shared group), top-32
                                              (100, 1024, 32, False, torch.bfloat16), (70, 1023, 32, True, torch.float32)])
def test_permute_bf16(T, E, k, shared, xdt):
    d = 256
    x = torch.randn((T, d), device=DEV).to(xdt)
    idx_np = _random_routing(T, E, k, seed=T + E, skew=1.0)
    idx = torch.from_numpy(idx_np.astype(np.int32)).to(DEV)
    res = gg.permute(x, idx, E, append_shared=shared)
    torch.cuda.synchronize()
    assert gg.read_device_status(res["ws"]) == 0
    plan = _check_plan(res, idx_np, E, shared)
    xb = oracle.bf16_round(f64(x))
    assert np.array_equal(f64(res["xp"]), xb[plan["row_to_token"]])


@pytest.mark.parametrize("T,E,k,shared,xdt", [(256, 8, 2, True, torch.float32), (300, 256, 8, True, torch.bfloat16),
                                              (41, 16, 2, False, torch.bfloat16)])
def test_permute_fp8_bytes_and_scales_bit_exact(T, E, k, shared, xdt):
    d = 512
    x = (torch.randn((T, d), device=DEV) * torch.rand((T, 1), device=DEV) * 10).to(xdt)
    x[0, :128] = 0  # an all-zero group (scale 1)
    idx_np = _random_routing(T, E, k, seed=3)
    idx = torch.from_numpy(idx_np.astype(np.int32)).to(DEV)
    res = gg.permute(x, idx, E, append_shared=shared, fp8=True)
    torch.cuda.synchronize()
    plan = _check_plan(res, idx_np, E, shared)
    q, s = ofp8.quantize_1x128(oracle.bf16_round(f64(x)).astype(np.float32))
    r2t = plan["row_to_token"]
    assert np.array_equal(res["xp"].cpu().numpy(), q[r2t])
    assert np.array_equal(res["xp_scales"].cpu().numpy().T, s[r2t])


def test_permute_flags_bad_expert_ids():
    x = torch.randn((64, 256), device=DEV, dtype=torch.bfloat16)
    idx = torch.zeros((64, 2), dtype=torch.int32, device=DEV)
    idx[:, 1] = 1
    idx[7, 1] = 9  # out of range for E = 8
    res = gg.permute(x, idx, 8)
    assert gg.read_device_status(res["ws"]) == -1
    idx[7, 1] = 0  # repeated within token 7
    res = gg.permute(x, idx, 8)
    assert gg.read_device_status(res["ws"]) == -1


# ---------------------------------------------------------------- grouped GEMM
def _offsets(sizes):
    return torch.tensor(np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32), device=DEV)


def _gemm_ref(A, B, sizes, epi, N):
    Af, out = f64(A), []
    o = 0
    for g, m in enumerate(sizes):
        Bg = f64(B[g])
        if epi == gg.EPI_SILU_GATE:
            gt = Af[o:o + m] @ Bg[:N].T
            up = Af[o:o + m] @ Bg[N:].T
            out.append(gt / (1 + np.exp(-gt)) * up)
        else:
            out.append(Af[o:o + m] @ Bg.T)
        o += m
    return np.concatenate(out, axis=0)


GEMM_CASES = [
    # sizes, N, K, epilogue, out dtype
    ([128], 256, 64, gg.EPI_NONE, torch.float32),
    ([128], 256, 128, gg.EPI_NONE, torch.bfloat16),
    ([300, 0, 1, 127, 129, 128], 256, 512, gg.EPI_NONE, torch.bfloat16),
    ([5, 200, 0, 64], 128, 256, gg.EPI_NONE, torch.float32),
    ([77, 3], 64, 192, gg.EPI_NONE, torch.bfloat16),
    ([128], 128, 64, gg.EPI_SILU_GATE, torch.bfloat16),
    ([0, 250, 1, 128, 513], 256, 384, gg.EPI_SILU_GATE, torch.bfloat16),
    ([1000, 24, 0, 0, 333], 512, 1024, gg.EPI_NONE, torch.bfloat16),
    # groups of >= 512 rows on average run on CTA pairs (256-row tiles split over two SMs)
    ([1024, 700, 513], 256, 256, gg.EPI_NONE, torch.bfloat16),
    ([2000, 0, 129], 512, 128, gg.EPI_NONE, torch.float32),
    ([257, 1600, 0, 255], 128, 320, gg.EPI_SILU_GATE, torch.bfloat16),
    ([1536, 1], 256, 512, gg.EPI_SILU_GATE, torch.bfloat16),
    # last tiles of 128, 129, 128, 232, 129 and 1 rows: those of at most 128 rows run as 128-row pair MMAs
    ([640, 641, 384, 0, 1000, 1153, 257], 384, 256, gg.EPI_SILU_GATE, torch.bfloat16),
    # fp32 output on CTA pairs, last tiles of 76 and 30 rows (128-row pair MMAs)
    ([1100, 30], 256, 128, gg.EPI_NONE, torch.float32),
    # 320..512 rows per group on average: the single-CTA 128x256 kernel (64-row MMA for short tails)
    ([400, 350, 0, 700, 333], 256, 512, gg.EPI_NONE, torch.bfloat16),
    ([340, 512, 330], 256, 384, gg.EPI_SILU_GATE, torch.bfloat16),
    # fine-grained groups: 128-row tiles and 64-row MMAs for short last tiles (1..64 rows)
    ([144, 150, 139, 0, 256, 257, 511, 300], 256, 256, gg.EPI_SILU_GATE, torch.bfloat16),
    ([1, 2, 300, 40], 128, 128, gg.EPI_NONE, torch.bfloat16),
    ([17, 33, 49, 65, 81, 97, 113, 129, 145], 128, 1024, gg.EPI_NONE, torch.bfloat16),
    # a few tokens per group (fewer than 32 rows per group on average): the weights take the
    # MMA's 128-row side (swap-AB), tokens the 32-wide side
    ([1, 0, 3, 2, 5, 33, 0, 1, 0, 7, 64, 1], 256, 128, gg.EPI_NONE, torch.bfloat16),
    ([2, 0, 1, 40, 3, 0, 0, 9], 192, 320, gg.EPI_SILU_GATE, torch.bfloat16),
    ([31, 32, 33, 0, 1], 128, 64, gg.EPI_NONE, torch.bfloat16),
    ([65, 0, 2, 0, 0, 0], 64, 256, gg.EPI_SILU_GATE, torch.bfloat16),
    # the largest group count one launch takes (1024): a few rows each (swap-AB), and up to 300 rows each
    ([int(v) for v in np.random.default_rng(1).integers(0, 4, 1024)], 128, 64, gg.EPI_NONE, torch.bfloat16),
    ([int(v) for v in np.random.default_rng(2).integers(0, 300, 1024)], 128, 64, gg.EPI_SILU_GATE, torch.bfloat16),
]


@pytest.mark.parametrize("sizes,N,K,epi,cdt", GEMM_CASES)
def test_grouped_gemm_bf16(sizes, N, K, epi, cdt):
    torch.manual_seed(sum(sizes) + N + K)
    rows = int(sum(sizes)) + 7  # trailing rows that belong to no group
    G = len(sizes)
    Nb = 2 * N if epi == gg.EPI_SILU_GATE else N
    A = torch.randn((rows, K), device=DEV).to(torch.bfloat16)
    B = (torch.randn((G, Nb, K), device=DEV) * 0.05).to(torch.bfloat16)
    C = torch.full((rows, N), 7.0, dtype=cdt, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    gg.grouped_gemm(A, B, _offsets(sizes), N, epilogue=epi, c_dtype=cdt, out=C, ws=ws)
    assert gg.read_device_status(ws) == 0
    ref = _gemm_ref(A, B, sizes, epi, N)
    got = f64(C)
    used = int(sum(sizes))
    assert np.all(got[used:] == 7.0), "rows outside every group must be untouched"
    err = rel_fro(got[:used], ref)
    assert err < (2e-3 if cdt == torch.bfloat16 else 1e-5), err
    scale = np.sqrt(np.mean(ref ** 2)) + 1e-30
    assert np.max(np.abs(got[:used] - ref)) < 2e-2 * scale + 1e-2 * np.max(np.abs(ref))


def test_grouped_gemm_rejects_bad_offsets_without_writing():
    A = torch.randn((256, 128), device=DEV).to(torch.bfloat16)
    B = torch.randn((2, 256, 128), device=DEV).to(torch.bfloat16)
    C = torch.full((256, 256), 3.0, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    for bad in ([0, 200, 100], [5, 100, 200], [0, 100, 300]):  # decreasing / not from 0 / past rows
        gg.grouped_gemm(A, B, torch.tensor(bad, dtype=torch.int32, device=DEV), 256, out=C, ws=ws)
        assert gg.read_device_status(ws) == -5
        assert torch.all(C == 3.0)


def test_grouped_gemm_all_groups_empty():
    A = torch.randn((64, 128), device=DEV).to(torch.bfloat16)
    B = torch.randn((3, 256, 128), device=DEV).to(torch.bfloat16)
    C = torch.full((64, 256), 3.0, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    gg.grouped_gemm(A, B, _offsets([0, 0, 0]), 256, out=C, ws=ws)
    assert gg.read_device_status(ws) == 0
    assert torch.all(C == 3.0)


# ---------------------------------------------------------------- combine
@pytest.mark.parametrize("T,d,k,shared,odt", [(256, 256, 2, True, torch.float32), (1000, 7168, 8, True, torch.bfloat16),
                                              (33, 4096, 2, False, torch.bfloat16)])
def test_combine(T, d, k, shared, odt):
    rng = _rng(T)
    R = T * k
    rows = R + (T if shared else 0)
    Y = torch.randn((rows, d), device=DEV).to(torch.bfloat16)
    perm = rng.permutation(R).reshape(T, k).astype(np.int32)
    w = rng.uniform(0, 1, size=(T, k)).astype(np.float32)
    out = gg.combine(Y, torch.from_numpy(perm).to(DEV), torch.from_numpy(w).to(DEV), shared, out_dtype=odt)
    Yf = f64(Y)
    ref = (Yf[R:] if shared else 0) + np.einsum("tk,tkd->td", w.astype(np.float64), Yf[perm])
    err = rel_fro(f64(out), ref)
    assert err < (1e-6 if odt == torch.float32 else 4e-3), err


# ---------------------------------------------------------------- FP8 weight quantisation
@pytest.mark.parametrize("G,N,K", [(2, 256, 384), (1, 128, 128), (3, 512, 256)])
def test_quantize_weights_bit_exact(G, N, K):
    W = (torch.randn((G, N, K), device=DEV) * 0.02).to(torch.bfloat16)
    W[0, :128, :128] = 0  # zero block -> scale 1
    W[-1, -1, -1] = 5.0   # one outlier dominates its block
    q, s = gg.quantize_weights_fp8(W)
    torch.cuda.synchronize()
    for g in range(G):
        wq, ws_ = ofp8.quantize_128x128(f64(W[g]).astype(np.float32))
        assert np.array_equal(q[g].cpu().numpy(), wq)
        assert np.array_equal(s[g].cpu().numpy(), ws_)


# ---------------------------------------------------------------- failure detection
def test_stalled_pipeline_times_out_and_context_survives():
    import time
    L = gg.lib()
    ws = torch.zeros(L.moe_selftest_workspace_size(), dtype=torch.uint8, device=DEV)
    t0 = time.perf_counter()
    st = L.moe_selftest_stalled_pipeline(gg._ptr(ws), ws.numel(), 50_000_000, gg._stream())
    assert st == 0
    assert gg.read_device_status(ws) == -6  # MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 10.0
    # the context is intact: a normal grouped GEMM still computes the right thing
    sizes = [200, 57]
    A = torch.randn((257, 128), device=DEV).to(torch.bfloat16)
    B = (torch.randn((2, 256, 128), device=DEV) * 0.05).to(torch.bfloat16)
    gws = torch.empty(256, dtype=torch.uint8, device=DEV)
    C = gg.grouped_gemm(A, B, _offsets(sizes), 256, ws=gws)
    assert gg.read_device_status(gws) == 0
    assert rel_fro(f64(C), _gemm_ref(A, B, sizes, gg.EPI_NONE, 256)) < 2e-3


def test_selftest_rejects_bad_arguments():
    L = gg.lib()
    ws = torch.zeros(L.moe_selftest_workspace_size(), dtype=torch.uint8, device=DEV)
    assert L.moe_selftest_stalled_pipeline(gg._ptr(ws), 100, 50_000_000, gg._stream()) == -3
    assert L.moe_selftest_stalled_pipeline(gg._ptr(ws), ws.numel(), 10, gg._stream()) == -1


# ---------------------------------------------------------------- the full-size layers' GEMM shapes
# The Mixtral-shaped layer's two GEMMs at their real sizes (CTA pairs, K = 4096
# and K = 14336 main loops, Zipf-skewed groups summing to T*k = 8192 rows),
# compared on sampled rows that cover every 128-row block of every group.
MIXTRAL_SIZES = [561, 2121, 1280, 700, 950, 1105, 620, 855]


@pytest.mark.parametrize("N,K,epi", [(14336, 4096, gg.EPI_SILU_GATE), (4096, 14336, gg.EPI_NONE)])
def test_grouped_gemm_bf16_mixtral_shapes(N, K, epi):
    from _util import rows_in_every_block
    sizes = MIXTRAL_SIZES
    assert "cta-pair" in gg.grouped_gemm_plan(len(sizes), sum(sizes), N, K, epilogue=epi)
    torch.manual_seed(N + K)
    rows = sum(sizes) + 3
    G = len(sizes)
    Nb = 2 * N if epi == gg.EPI_SILU_GATE else N
    A = torch.randn((rows, K), device=DEV).to(torch.bfloat16)
    B = (torch.randn((G, Nb, K), device=DEV) * 0.02).to(torch.bfloat16)
    C = torch.full((rows, N), 7.0, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    gg.grouped_gemm(A, B, _offsets(sizes), N, epilogue=epi, out=C, ws=ws)
    assert gg.read_device_status(ws) == 0
    sample = rows_in_every_block(sizes, np.random.default_rng(N), per_block=2)
    bounds = np.concatenate([[0], np.cumsum(sizes)])
    got, ref = [], []
    for g in range(G):
        r = sample[(sample >= bounds[g]) & (sample < bounds[g + 1])]
        if not len(r):
            continue
        Ar = f64(A[torch.from_numpy(r).to(DEV)])
        Bg = B[g].to(torch.float64).cpu().numpy()  # exact widening
        if epi == gg.EPI_SILU_GATE:
            gt, up = Ar @ Bg[:N].T, Ar @ Bg[N:].T
            ref.append(gt / (1 + np.exp(-gt)) * up)
        else:
            ref.append(Ar @ Bg.T)
        got.append(f64(C[torch.from_numpy(r).to(DEV)]))
    got, ref = np.concatenate(got), np.concatenate(ref)
    err = rel_fro(got, ref)
    assert err < 2e-3, err
    assert torch.all(C[sum(sizes):] == 7.0)
