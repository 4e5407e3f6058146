"""The C-ABI library: it builds, loads, exports every function include/moe.h
declares, and rejects bad arguments on the host (no GPU needed: each call
below returns before any CUDA call is made)."""
import ctypes
import os
import re
import subprocess

import pytest

import grouped_gemm_03_b200 as gg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    from grouped_gemm_03_b200.build import build
    build()
    return gg.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_surface():
    assert header_functions() == gg.exported_symbols()


def test_binding_signatures_match_the_header():
    # parameter count of every declaration against the ctypes argument list of the binding
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"\b(moe_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S)
    assert len(decls) == len(gg.exported_symbols())
    for name, params in decls:
        p = params.strip()
        n = 0 if p in ("", "void") else len(p.split(","))
        assert len(gg._SIGS[name][1]) == n, name


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", gg.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (moe_[a-z0-9_]+)$", out, flags=re.M))
    missing = [f for f in header_functions() if f not in exported]
    assert not missing, missing
    for f in header_functions():
        assert hasattr(L, f)


def test_build_targets_sm100a_only():
    from grouped_gemm_03_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings(L):
    for code in range(0, -7, -1):
        s = gg.status_string(code)
        assert s.startswith("MOE_")
    assert "BAD_OFFSETS" in gg.status_string(-5)


def test_workspace_sizes_are_host_arithmetic(L):
    cfg = gg.make_config(T=4096, d=4096, E=8, k=2, inter=14336)
    n = gg.workspace_size(cfg)
    # at least Xp, H and Y (bf16) for R = 8192 rows
    assert n >= 8192 * (4096 + 14336 + 4096) * 2
    cfg_s = gg.make_config(T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048)
    assert gg.workspace_size(cfg_s) >= (4096 * 9) * (7168 * 2 + 2048) * 2
    assert L.moe_grouped_gemm_workspace_size() >= 4
    assert L.moe_permute_workspace_size(4096, 256) >= 128 * 256 * 4
    bad = gg.make_config(T=16, d=256, E=4, k=5, inter=128)
    assert L.moe_workspace_size(ctypes.byref(bad)) == 0


def test_host_validation_rejects_bad_arguments(L):
    fake = ctypes.c_void_p(0x10000)
    null = None
    # k > E
    assert L.moe_router_topk(fake, 2, fake, 2, null, 16, 256, 4, 5, 0, null, fake, fake, fake, 1 << 20, null) == -1
    # workspace too small
    assert L.moe_router_topk(fake, 2, fake, 2, null, 16, 256, 4, 2, 0, null, fake, fake, fake, 8, null) == -3
    # misaligned workspace
    assert L.moe_permute(fake, 2, fake, 16, 256, 4, 2, 0, 2, fake, null, fake, fake, fake, fake,
                         ctypes.c_void_p(0x10010), 1 << 20, null) == -3
    # E4M3 permute needs d % 128 == 0
    assert L.moe_permute(fake, 2, fake, 16, 200, 4, 2, 0, 3, fake, fake, fake, fake, fake, fake,
                         fake, 1 << 20, null) == -2
    # permuted rows are int32 indices: T * (k + 1) > 2^30 is refused before any launch
    assert L.moe_permute(fake, 2, fake, 1 << 27, 256, 16, 8, 0, 2, fake, null, fake, fake, fake, fake,
                         fake, 1 << 40, null) == -2
    assert L.moe_permute(fake, 2, fake, (1 << 29) - 1, 256, 16, 1, 0, 2, fake, null, fake, fake, fake, fake,
                         fake, 8, null) == -3   # within the bound: the short workspace is what fails
    # grouped GEMM: K not a multiple of 64 / null offsets
    assert L.moe_grouped_gemm(fake, null, fake, null, fake, 4, 64, 256, 100, 2, 0, fake, 2, null,
                              fake, 256, null) == -2
    assert L.moe_grouped_gemm(fake, null, fake, null, null, 4, 64, 256, 128, 2, 0, fake, 2, null,
                              fake, 256, null) == -1
    # FP8 weights need 128-multiples
    assert L.moe_quantize_weights_fp8(fake, 2, 100, 128, fake, fake, null) == -2
    # whole layer: short workspace, shared size != inter
    cfg = gg.make_config(T=256, d=256, E=8, k=2, inter=512, shared_inter=512)
    args = [fake, fake, null, fake, null, fake, null, fake, null, fake, null, fake, null]
    assert L.moe_forward(ctypes.byref(cfg), *args, fake, 1024, null) == -3
    cfg2 = gg.make_config(T=256, d=256, E=8, k=2, inter=512, shared_inter=256)
    assert L.moe_forward(ctypes.byref(cfg2), *args, fake, 1 << 30, null) == -2
    # marked forward: the six event handles are required
    assert L.moe_forward_marked(ctypes.byref(cfg), *args, fake, 1 << 30, null, null) == -1
    events = (ctypes.c_void_p * 6)(*([0x20000] * 5 + [0]))
    assert L.moe_forward_marked(ctypes.byref(cfg), *args, fake, 1 << 30, events, null) == -1


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(gg, "LIB_PATH", str(tmp_path / "libmoe.so"))
    monkeypatch.setattr(gg, "_LIB", None)
    with pytest.raises(RuntimeError, match="missing"):
        gg.lib()


def _layer_plans(name):
    from workload import shape_of
    s = shape_of(name)
    extra = 1 if s.shared_inter else 0
    rows = s.T * s.k + (s.T if extra else 0)
    ab = gg.MOE_E4M3 if s.fp8 else gg.MOE_BF16
    up = gg.grouped_gemm_plan(s.E, rows, s.inter, s.d, ab, gg.EPI_SILU_GATE, ab, extra)
    down = gg.grouped_gemm_plan(s.E, rows, s.d, s.inter, ab, gg.EPI_NONE, gg.MOE_BF16, extra)
    return up, down


# The kernel each benchmarked layer runs on. A heuristic change that moves a
# workload to another kernel shows up here before it shows up as a slowdown.
@pytest.mark.parametrize("name,up,down", [
    ("mixtral", "bf16 cta-pair 256x256 silu-gate", "bf16 cta-pair 256x256"),
    ("fine", "bf16 128x256 silu-gate", "bf16 128x256"),
    ("fine_skew", "bf16 128x256 silu-gate", "bf16 128x256"),
    ("decode", "bf16 swap-ab 128x32 silu-gate", "bf16 swap-ab 128x32"),
    ("tiny", "bf16 128x128 silu-gate (64 out cols)", "bf16 128x256"),
    ("fine_fp8", "e4m3 128x256 silu-gate e4m3-out", "e4m3 128x256"),
])
def test_grouped_gemm_plan_per_workload(L, name, up, down):
    assert _layer_plans(name) == (up, down)


def test_grouped_gemm_plan_edges(L):
    P = gg.grouped_gemm_plan
    assert P(8, 0, 256, 128) == "empty"
    assert P(0, 1024, 256, 128) == "empty"
    # widths the kernels do not tile
    assert P(4, 1024, 96, 128, epilogue=gg.EPI_SILU_GATE) == "unsupported"
    assert P(4, 4096, 100, 128) == "unsupported"
    assert P(4, 4096, 384, 256, ab_dtype=gg.MOE_E4M3) == "unsupported"
    # a gate width that is a multiple of 64 only takes the 64-column tiles
    assert P(4, 100000, 192, 256, epilogue=gg.EPI_SILU_GATE) == "bf16 128x128 silu-gate (64 out cols)"
    # few rows per group -> weights on the 128-row side; many -> CTA pairs
    assert P(64, 64 * 31, 1024, 1024).startswith("bf16 swap-ab")
    assert P(64, 64 * 32, 1024, 1024) == "bf16 128x256"
    assert P(8, 8 * 512, 1024, 1024) == "bf16 cta-pair 256x256"
    # narrow gate tiles only while 128-column tiles fill under two waves of the SMs
    assert P(8, 8 * 256, 1024, 1024, epilogue=gg.EPI_SILU_GATE, num_sms=148) == \
        "bf16 128x128 silu-gate (64 out cols)"
    assert P(8, 8 * 256, 4096, 1024, epilogue=gg.EPI_SILU_GATE, num_sms=148) == "bf16 128x256 silu-gate"


def test_forward_launch_count():
    L = gg.lib()
    import ctypes
    mixtral = gg.make_config(T=4096, d=4096, E=8, k=2, inter=14336)
    fine = gg.make_config(T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048)
    decode = gg.make_config(T=128, d=2048, E=64, k=2, inter=1408)
    # one-launch router (bf16, E <= 256, k <= 8) and the scan folded into the
    # scatter (ceil(T/32) * E <= 8192)
    assert L.moe_forward_launches(ctypes.byref(mixtral)) == 6
    assert L.moe_forward_launches(ctypes.byref(decode)) == 6
    assert L.moe_forward_launches(ctypes.byref(fine)) == 7      # histogram + scan + scatter
    # fp32 x with 64 experts: logits + selection
    decode32 = gg.make_config(T=128, d=2048, E=64, k=2, inter=1408, x_dtype=gg.MOE_F32)
    assert L.moe_forward_launches(ctypes.byref(decode32)) == 7
    assert L.moe_forward_launches(ctypes.byref(gg.make_config(T=0, d=256, E=8, k=2, inter=512))) == 0
    assert L.moe_forward_launches(ctypes.byref(gg.make_config(T=4, d=100, E=8, k=2, inter=512))) == -1
