"""The allocation-free permute entry point (moe_permute_noalloc).

It exists for callers that cannot give the library device memory of its own
-- a plugin whose host runtime owns every allocation, a serving loop with a
memory plan fixed at start-up -- so its scratch lives in static device memory
of the library instead of a caller workspace.  These tests call it through
the C ABI and check that calls in a row (different shapes: the second covers
more scratch than the first, the third runs inside what the second left
behind) give exactly what moe_permute gives;
the permutation plan and the permuted bytes are compared bit for bit, the
tolerance every permute test uses.  This file is collected last so a run
that stops at the first failure has run everything else already.
"""
import ctypes

import numpy as np
import pytest
import torch

import grouped_gemm_03_b200 as gg

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from grouped_gemm_03_b200.build import build
    build()


def _inputs(T, E, k, d, xdt, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(xdt).to(DEV)
    logits = torch.randn((T, E), generator=g) - torch.log1p(torch.arange(E, dtype=torch.float32))
    idx = torch.topk(logits, k, dim=1).indices.to(torch.int32).to(DEV)  # distinct experts per token
    return x, idx.contiguous()


def _noalloc(x, idx, E, shared, fp8):
    """Caller-owned outputs, no workspace: the entry point's contract."""
    T, d = x.shape
    k = idx.shape[1]
    rows = T * k + (T if shared else 0)
    out = dict(
        xp=torch.empty((rows, d), dtype=torch.uint8 if fp8 else torch.bfloat16, device=DEV),
        xp_scales=torch.empty((d // 128, rows), dtype=torch.float32, device=DEV) if fp8 else None,
        counts=torch.empty(E, dtype=torch.int32, device=DEV),
        offsets=torch.empty(E + 1 + (1 if shared else 0), dtype=torch.int32, device=DEV),
        row_to_token=torch.empty(rows, dtype=torch.int32, device=DEV),
        token_to_row=torch.empty((T, k), dtype=torch.int32, device=DEV),
    )
    P = gg._ptr
    st = gg.lib().moe_permute_noalloc(P(x), gg._dt(x), P(idx), T, d, E, k, int(shared),
                                      gg.MOE_E4M3 if fp8 else gg.MOE_BF16, P(out["xp"]), P(out["xp_scales"]),
                                      P(out["counts"]), P(out["offsets"]), P(out["row_to_token"]),
                                      P(out["token_to_row"]), gg._stream())
    assert st == 0, gg.status_string(st)
    return out


CALLS = [  # T, E, k, d, x dtype, shared, fp8
    (300, 8, 2, 256, torch.float32, False, False),     # 10 blocks x 8 experts of count words
    (1000, 256, 8, 512, torch.bfloat16, True, True),   # 32 x 256: beyond what the first call wrote
    (200, 64, 4, 384, torch.bfloat16, True, False),    # 7 x 64: over the second call's leftovers
]


def test_calls_in_a_row_match_moe_permute():
    results = []
    for n, (T, E, k, d, xdt, shared, fp8) in enumerate(CALLS):
        x, idx = _inputs(T, E, k, d, xdt, seed=17 + n)
        results.append((_noalloc(x, idx, E, shared, fp8), gg.permute(x, idx, E, append_shared=shared, fp8=fp8)))
    torch.cuda.synchronize()
    for got, want in results:
        for key in ("counts", "offsets", "row_to_token", "token_to_row", "xp", "xp_scales"):
            if want[key] is None:
                assert got[key] is None
                continue
            assert torch.equal(got[key], want[key]), key
        assert gg.read_device_status(want["ws"]) == 0


def test_rejects_sizes_beyond_the_static_scratch():
    fake = ctypes.c_void_p(0x10000)
    # ceil(65537 / 32) * 256 > 262144 count words
    st = gg.lib().moe_permute_noalloc(fake, gg.MOE_BF16, fake, 65537, 256, 256, 8, 0, gg.MOE_BF16, fake, None,
                                      fake, fake, fake, fake, None)
    assert st == -2
    # permuted rows are int32 indices: T * (k + 1) > 2^30 is refused before anything runs
    st = gg.lib().moe_permute_noalloc(fake, gg.MOE_BF16, fake, 1 << 27, 256, 1, 1, 0, gg.MOE_BF16, fake, None,
                                      fake, fake, fake, fake, None)
    assert st == -2
