"""Named MoE-layer workloads and their seeded input tensors.

Every tensor is drawn by torch's Philox-based generator from a seed derived
from (seed, tensor id, expert id), so a tensor does not depend on the order in
which others are drawn and one expert's weights can be regenerated alone.
The draws are made on the requested device; CPU and CUDA streams differ, so a
test that compares two implementations feeds both from the SAME tensors.

Value recipe (the workloads of the grouped-GEMM / MoE pages):
  * x ~ N(0, 1): fp32 for the tiny layer, bf16 (round-to-nearest-even of the
    fp32 draw) otherwise;
  * router W_r, expert W1 / W2 and shared-expert weights ~ N(0, 0.02^2),
    stored bf16 (the tiny layer's router is fp32);
  * skewed workloads add a per-expert logit offset
        bias[e] = -gamma * s * ln(1 + pi(e)),   gamma = 0.7,
    pi a seeded permutation of 0..E-1, so the routing probability of expert e
    falls off like a Zipf law of exponent ~gamma*s in its popularity rank and
    the hot experts are not always the low indices;
  * W1[e] is [2*I, d]: rows 0..I-1 are the gate projection, rows I..2I-1 the
    up projection; W2[e] is [d, I] (both K-major, i.e. row-major with the
    contraction dimension contiguous).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

ZIPF_GAMMA = 0.7
WEIGHT_STD = 0.02

# tensor ids mixed into the per-tensor seed
_TID_X, _TID_WR, _TID_W1, _TID_W2, _TID_W1S, _TID_W2S, _TID_PERM, _TID_LOGITS = range(8)


@dataclass(frozen=True)
class MoEShape:
    name: str
    T: int                  # tokens
    d: int                  # hidden size
    E: int                  # routed experts
    k: int                  # experts per token
    inter: int              # routed-expert intermediate size I
    shared_inter: int = 0   # shared-expert intermediate size (0 = no shared expert)
    x_dtype: str = "bf16"   # "f32" | "bf16"
    router_dtype: str = "bf16"
    fp8: bool = False       # expert GEMMs in E4M3 with 1x128 / 128x128 scales
    mx: bool = False        # with fp8: power-of-two (MX) scales the tensor core applies
    gather: bool = False    # the up GEMM gathers its A rows in the load (no expert-ordered copy of x)
    zipf_s: float = 0.0     # 0 = balanced router
    renormalize: bool = False

    @property
    def R(self) -> int:           # routed rows
        return self.T * self.k

    @property
    def rows(self) -> int:        # routed + shared rows of the permuted buffer
        return self.T * self.k + (self.T if self.shared_inter else 0)

    def gemm_flops(self) -> float:
        """Algorithmic GEMM FLOPs of one forward (routed k rows/token + shared)."""
        f = 2.0 * self.R * (2 * self.inter) * self.d + 2.0 * self.R * self.d * self.inter
        if self.shared_inter:
            f += 2.0 * self.T * (2 * self.shared_inter) * self.d + 2.0 * self.T * self.d * self.shared_inter
        return f


CONFIGS: dict[str, MoEShape] = {
    "tiny": MoEShape("tiny", T=256, d=256, E=8, k=2, inter=512, shared_inter=512,
                     x_dtype="f32", router_dtype="f32"),
    "mixtral": MoEShape("mixtral", T=4096, d=4096, E=8, k=2, inter=14336, zipf_s=1.0),
    "fine": MoEShape("fine", T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048),
    "fine_skew": MoEShape("fine_skew", T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048,
                          zipf_s=1.2),
    "fine_fp8": MoEShape("fine_fp8", T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048,
                         fp8=True),
    "fine_fp8_skew": MoEShape("fine_fp8_skew", T=4096, d=7168, E=256, k=8, inter=2048,
                              shared_inter=2048, fp8=True, zipf_s=1.2),
    # the same FP8 layers with power-of-two (MX) scales
    "fine_mx": MoEShape("fine_mx", T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048,
                        fp8=True, mx=True),
    "fine_mx_skew": MoEShape("fine_mx_skew", T=4096, d=7168, E=256, k=8, inter=2048,
                             shared_inter=2048, fp8=True, mx=True, zipf_s=1.2),
    # the fine-grained layer with the up GEMM gathering its rows in the load
    "fine_gather": MoEShape("fine_gather", T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048,
                            gather=True),
    "decode": MoEShape("decode", T=128, d=2048, E=64, k=2, inter=1408, zipf_s=1.5),
}

# router-only microbenchmark: N tokens of fp16 logits over E experts, top-k
ROUTER_MICRO = dict(N=65536, E=128, k=4)


def shape_of(name: str, **overrides) -> MoEShape:
    s = CONFIGS[name]
    return replace(s, **overrides) if overrides else s


def _seed(seed: int, tid: int, sub: int = 0) -> int:
    # splitmix64 finaliser of the packed (seed, tensor, sub) key -> 63-bit seed
    z = (seed * 0x9E3779B97F4A7C15 + tid * 0xBF58476D1CE4E5B9 + sub * 0x94D049BB133111EB) & (2**64 - 1)
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & (2**64 - 1)
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & (2**64 - 1)
    return (z ^ (z >> 31)) & (2**63 - 1)


def _gen(device, seed: int, tid: int, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, tid, sub))
    return g


def _normal(shape, std, dtype, device, seed, tid, sub=0) -> torch.Tensor:
    g = _gen(device, seed, tid, sub)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def zipf_bias(E: int, s: float, seed: int) -> torch.Tensor:
    """Per-expert logit offset -gamma*s*ln(1+pi(e)) (fp32, CPU)."""
    g = _gen("cpu", seed, _TID_PERM)
    pi = torch.randperm(E, generator=g)
    return torch.tensor([-ZIPF_GAMMA * s * math.log1p(float(pi[e])) for e in range(E)],
                        dtype=torch.float32)


def make_expert_weights(shape: MoEShape, which: str, e: int, device, seed: int) -> torch.Tensor:
    """One expert's weight matrix: which in {"W1", "W2", "W1s", "W2s"}."""
    I = shape.shared_inter if which in ("W1s", "W2s") else shape.inter
    rows, cols = (2 * I, shape.d) if which in ("W1", "W1s") else (shape.d, I)
    tid = {"W1": _TID_W1, "W2": _TID_W2, "W1s": _TID_W1S, "W2s": _TID_W2S}[which]
    return _normal((rows, cols), WEIGHT_STD, torch.bfloat16, device, seed, tid, e)


def make_inputs(shape: MoEShape | str, seed: int = 1234, device="cpu",
                experts: bool = True) -> dict:
    """All inputs of one layer forward, on `device`.

    Returns dict(x, W_r, bias, W1, W2, W1s, W2s) where bias / W1s / W2s may be
    None.  With experts=False the (large) expert weights are omitted.
    """
    if isinstance(shape, str):
        shape = CONFIGS[shape]
    out = {}
    out["x"] = _normal((shape.T, shape.d), 1.0, _DT[shape.x_dtype], device, seed, _TID_X)
    out["W_r"] = _normal((shape.E, shape.d), WEIGHT_STD, _DT[shape.router_dtype], device, seed, _TID_WR)
    out["bias"] = zipf_bias(shape.E, shape.zipf_s, seed).to(device) if shape.zipf_s else None
    out["W1"] = out["W2"] = out["W1s"] = out["W2s"] = None
    if experts:
        I, d, E = shape.inter, shape.d, shape.E
        W1 = torch.empty((E, 2 * I, d), dtype=torch.bfloat16, device=device)
        W2 = torch.empty((E, d, I), dtype=torch.bfloat16, device=device)
        for e in range(E):
            W1[e] = make_expert_weights(shape, "W1", e, device, seed)
            W2[e] = make_expert_weights(shape, "W2", e, device, seed)
        out["W1"], out["W2"] = W1, W2
        if shape.shared_inter:
            out["W1s"] = make_expert_weights(shape, "W1s", 0, device, seed)
            out["W2s"] = make_expert_weights(shape, "W2s", 0, device, seed)
    return out


def make_router_logits(N: int, E: int, seed: int = 1234, device="cpu",
                       dtype=torch.float16) -> torch.Tensor:
    """Router-only microbenchmark input: logits ~ N(0,1) stored in `dtype`."""
    return _normal((N, E), 1.0, dtype, device, seed, _TID_LOGITS)
