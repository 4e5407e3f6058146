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
