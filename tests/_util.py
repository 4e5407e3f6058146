"""Shared helpers of the GPU parity tests (comparison metrics, oracle adapters)."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def rel_fro(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def f64(t: torch.Tensor) -> np.ndarray:
    return oracle.as_f64(t)


class DeviceExperts:
    """Indexable view of a stacked device weight tensor: [e] -> host fp64 copy.

    The weights come from the seeded input generator (drawn on the GPU); the
    oracle reads one expert at a time.
    """

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            self.cache[e] = f64(self.t[e])
        return self.cache[e]


def adopt_near_ties(oracle_logits: np.ndarray, oracle_idx: np.ndarray, gpu_idx: np.ndarray, k: int,
                    rel_gap: float = 1e-4):
    """Routing to give the oracle's forward: its own, except at near ties.

    Where the oracle's fp64 top-k differs from the GPU's and the oracle's gap
    between the k-th and (k+1)-th logit is below rel_gap * max(1, |l_k|), both
    choices are correct and the oracle adopts the GPU's.  Any other mismatch
    is returned in `bad`.
    """
    idx = oracle_idx.copy()
    adopted, bad = [], []
    for t in range(idx.shape[0]):
        if set(oracle_idx[t]) == set(gpu_idx[t]) and np.array_equal(oracle_idx[t], gpu_idx[t]):
            continue
        srt = np.sort(oracle_logits[t])[::-1]
        gap = srt[k - 1] - srt[k] if k < len(srt) else np.inf
        # ordering differences inside the top-k also come from near-equal logits
        inner = np.min(np.abs(np.diff(srt[:k]))) if k > 1 else np.inf
        if min(gap, inner) < rel_gap * max(1.0, abs(srt[k - 1])):
            idx[t] = gpu_idx[t]
            adopted.append(t)
        else:
            bad.append(t)
    return idx, adopted, bad


class StreamedExperts:
    """Indexable view of a stacked device bf16 weight tensor: [e] -> host fp64.

    bf16 -> fp64 is an exact widening; it is done on the device by torch and
    the fp64 values are copied to the host, which is far faster than widening
    on the host for the full-size layers.  With keep=False nothing is cached,
    so host memory holds one expert at a time (the fine-grained layers' 256
    experts are ~90 GB as fp64).
    """

    def __init__(self, t: torch.Tensor, keep: bool = False):
        self.t, self.keep, self.cache = t, keep, {}

    def __getitem__(self, e):
        e = int(e)
        if e in self.cache:
            return self.cache[e]
        v = self.t[e].to(torch.float64).cpu().numpy()
        if self.keep:
            self.cache[e] = v
        return v


def check_plan_full_size(gg, s, inp):
    """Routing and permutation at full size, through the C ABI, bit-exact against
    the oracle's selection and plan computed from the GPU's own logits.

    Returns the GPU's top-k indices.
    """
    gidx, gw, glog = gg.router_topk(inp["x"], inp["W_r"], s.k, bias=inp["bias"], renormalize=s.renormalize,
                                    want_logits=True)
    l = f64(glog)
    oidx = oracle.topk_select(l, s.k)
    gi = gidx.cpu().numpy()
    assert np.array_equal(gi, oidx), "top-k differs from the oracle's selection on the same logits"
    ow = oracle.gate_weights(oracle.softmax(l), oidx, s.renormalize)
    assert np.max(np.abs(gw.cpu().numpy() - ow) / np.maximum(ow, 1e-30)) < 2e-6
    shared = bool(s.shared_inter)
    plan = gg.permute(inp["x"], gidx, s.E, append_shared=shared, fp8=s.fp8)
    want = oracle.permutation(oidx, s.E, shared=shared)
    for key in ("counts", "offsets", "row_to_token", "token_to_row"):
        got = plan[key].cpu().numpy().astype(np.int64).reshape(want[key].shape)
        assert np.array_equal(got, want[key]), key
    if not s.fp8:  # the permuted rows are the tokens' bf16 rows, in the oracle's row order
        xb = inp["x"].to(torch.bfloat16).view(torch.int16).cpu().numpy()
        assert np.array_equal(plan["xp"].view(torch.int16).cpu().numpy(), xb[want["row_to_token"]])
    else:  # E4M3 codes and 1x128 scales of each token, quantised once, in the oracle's row order
        from oracle import fp8 as ofp8
        xq, sx = ofp8.quantize_1x128(oracle.bf16_round(f64(inp["x"])).astype(np.float32))
        r2t = want["row_to_token"]
        assert np.array_equal(plan["xp"].cpu().numpy(), xq[r2t])
        assert np.array_equal(plan["xp_scales"].cpu().numpy().T, sx[r2t])
    return gi


def tokens_covering_every_group(gidx: np.ndarray, E: int, n: int, seed: int = 5) -> np.ndarray:
    """At least n token ids such that every expert some token selects is selected
    by one of them: one token per expert, then random tokens up to n."""
    rng = np.random.default_rng(seed)
    T = gidx.shape[0]
    pick = set()
    for e in range(E):
        t = np.nonzero((gidx == e).any(axis=1))[0]
        if len(t):
            pick.add(int(rng.choice(t)))
    rest = [t for t in rng.permutation(T) if t not in pick]
    pick.update(int(t) for t in rest[: max(0, n - len(pick))])
    return np.array(sorted(pick))


def rows_in_every_block(sizes, rng, per_block: int = 2, block: int = 128) -> np.ndarray:
    """Sampled row ids of a grouped operand: per_block random rows from every
    `block`-row tile of every group, plus each group's last row."""
    out, o = [], 0
    for m in sizes:
        for b0 in range(0, m, block):
            n = min(block, m - b0)
            out.extend(int(o + b0 + r) for r in rng.choice(n, size=min(per_block, n), replace=False))
        if m:
            out.append(o + m - 1)
        o += m
    return np.unique(np.array(out, dtype=np.int64))


def host_threads() -> int:
    import os
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)
