"""bench.py's host arithmetic, checked on the CPU: the algorithmic work each
kernel is credited with, the choice of roofline bound from arithmetic
intensity, and the rule that committed DRAM-traffic figures are only used
while the kernel sources still hash to what was profiled."""
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workload import shape_of  # noqa: E402

PEAKS = {"hbm_gbs": 6545.3, "bf16_tflops": 1618.5, "bf16_tflops_sustained": 1374.0}


def test_algorithmic_work_of_the_mixtral_layer():
    s = shape_of("mixtral")
    a = bench.algorithmic(s, counts=np.full(8, 1024))
    # up: 2 * R * (2I) * d with R = T k = 8192 rows, I = 14336, d = 4096
    assert a["up_gemm"]["flops"] == 2.0 * 8192 * 28672 * 4096
    assert a["down_gemm"]["flops"] == 2.0 * 8192 * 4096 * 14336
    # up bytes: the 8 experts' W1 once, A (Xp) once, H written once
    assert a["up_gemm"]["bytes"] == 8 * 28672 * 4096 * 2 + 8192 * 4096 * 2 + 8192 * 14336 * 2
    # combine reads k rows per token and writes the token
    assert a["combine"]["bytes"] == 8192 * 4096 * 2 + 4096 * 4096 * 2 + 4096 * 2 * 8
    assert a["up_gemm"]["flops"] + a["down_gemm"]["flops"] == s.gemm_flops()


def test_algorithmic_counts_only_experts_that_received_tokens():
    s = shape_of("decode")
    counts = np.zeros(64, dtype=int)
    counts[:5] = [100, 80, 40, 20, 16]
    a = bench.algorithmic(s, counts=counts)
    w1 = 2 * s.inter * s.d * 2
    assert a["up_gemm"]["bytes"] == 5 * w1 + 256 * s.d * 2 + 256 * s.inter * 2


def test_fp8_weights_count_one_byte():
    bf, f8 = bench.algorithmic(shape_of("fine")), bench.algorithmic(shape_of("fine_fp8"))
    assert f8["up_gemm"]["flops"] == bf["up_gemm"]["flops"]
    assert f8["up_gemm"]["bytes"] < 0.55 * bf["up_gemm"]["bytes"]


def _kernels(up_us, down_us=1.0, rest_us=1.0):
    return {"router": {"us": rest_us}, "permute": {"us": rest_us}, "up_gemm": {"us": up_us},
            "down_gemm": {"us": down_us}, "combine": {"us": rest_us}}


def test_roofline_bound_follows_arithmetic_intensity():
    # Mixtral: ~880 FLOP per algorithmic byte, above the ridge (1618.5e12 / 6545.3e9 = 247): tensor
    s = shape_of("mixtral")
    alg = bench.algorithmic(s, counts=np.full(8, 1024))
    r = bench.roofline(s, alg, _kernels(1400.0), PEAKS, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["kernel"].startswith("up-projection")
    assert r["achieved"] == pytest.approx(alg["up_gemm"]["flops"] / 1400e-6 / 1e12, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / 1618.5, abs=1e-4)
    # fine: ~130 FLOP per byte, below the ridge: HBM, in GB/s of algorithmic bytes
    s = shape_of("fine")
    alg = bench.algorithmic(s)
    r = bench.roofline(s, alg, _kernels(2800.0), PEAKS, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6545.3
    assert r["achieved"] == pytest.approx(alg["up_gemm"]["bytes"] / 2800e-6 / 1e9, rel=1e-3)


def test_roofline_reports_the_largest_stage_and_fp8_peak():
    s = shape_of("fine_fp8")
    alg = bench.algorithmic(s)
    r = bench.roofline(s, alg, _kernels(100.0, down_us=900.0), PEAKS, "measured")
    assert r["kernel"].startswith("down-projection")
    # an E4M3 contraction is held against twice the bf16 tensor peak; here it is HBM-bound anyway
    assert r["bound"] == "hbm"
    tiny = shape_of("tiny")
    r = bench.roofline(tiny, bench.algorithmic(tiny), _kernels(1.0, rest_us=5.0), PEAKS, "measured")
    assert r["bound"] == "hbm" and r["kernel"].startswith("router")


def test_traffic_is_used_only_for_the_profiled_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.kernel_source_hash("up_gemm")
    now = bench.kernel_source_hash("down_gemm")
    (prof / "traffic.json").write_text(json.dumps({"mixtral": {
        "up_gemm": {"bytes_per_launch": 123, "source_sha256": good},
        "down_gemm": {"bytes_per_launch": 456, "source_sha256": "0" * 64}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile("mixtral", "up_gemm", good) == 123
    assert bench.traffic_from_profile("mixtral", "down_gemm", now) is None  # profiled on other sources
    assert bench.traffic_from_profile("fine", "up_gemm", good) is None


def test_committed_traffic_figures_are_consistent():
    # (whether they still match the sources is bench.py's business: it reports null when not)
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for stage, e in d["mixtral"].items():
        assert stage in bench.STAGE_SOURCES
        assert e["bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"]
        assert len(e["source_sha256"]) == 64 and e["command"].startswith("ncu ")


def test_reference_arm_times_the_oracle_on_the_cpu_baseline_batches():
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "2", "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["host_cores"] >= 1 and cb["cpu_model"]
    # the same batches as the cpu_baseline leg: oracle_batch_tokens of the workload
    assert f"batch(es) of {bench.oracle_batch_tokens(shape_of('tiny'))} random tokens" in cb["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_oracle_batches_are_bounded():
    assert bench.oracle_batch_tokens(shape_of("mixtral")) == 512
    assert bench.oracle_batch_tokens(shape_of("decode")) == 128
    # fine-grained experts do not fit the host cache as fp64: converted one at a time
    assert 256 * 3 * 2048 * 7168 * 8 > bench.HOST_CACHE_BYTES
    assert 8 * 3 * 14336 * 4096 * 8 <= bench.HOST_CACHE_BYTES
