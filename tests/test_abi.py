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


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(gg, "LIB_PATH", str(tmp_path / "libmoe.so"))
    monkeypatch.setattr(gg, "_LIB", None)
    with pytest.raises(RuntimeError, match="missing"):
        gg.lib()
