"""Plain fp64 reference of one MoE-layer forward -- TEST INFRASTRUCTURE ONLY.

Used by tests/, the smoke check and bench.py's CPU-baseline leg; never by the
library.  Every step is the plain definition the source pages give, written
out with numpy in float64 (matrix products use numpy's matmul as a library
primitive; nothing is blocked, fused or reordered).

Sources (web pages on grouped GEMM for MoE):
  [MegaMoE]   "MegaMoE math model -> DeepGEMM source walk-through"
              (2kiu.com news 6052262), §2.1 routing / combine formula,
              §2.3 FP8 scaled GEMM, §4.3 expert-contiguous layout.
  [GroupedTP] "Dense GEMM -> GroupedGEMM -> TP MoE" (2kiu.com news 6174947),
              §2.2 six-step data flow, §4.2 route_tokens /
              compute_expert_offsets, §4.3 hand-check and gate-normalisation
              trap, §5.1 imbalance diagnostic.
  [DSMoE]     "DeepSeek MoE architecture overview" (agent.csdn.net), §2.2
              top-k gating.

Readings taken where the pages are silent (each is also pinned by a test):
  * top-k compares logits (softmax is monotone), ties go to the lower expert
    index, slots are ordered by descending logit;
  * the combine weight is the selected softmax value p_i itself ([MegaMoE]
    §2.1); `renormalize=True` divides by the sum over the selected experts
    ([GroupedTP] §4.2), which equals a softmax over the top-k logits
    ([DSMoE] §2.2);
  * inside an expert's segment of the permuted buffer rows are in ascending
    token order; the shared expert, when present, owns rows R..R+T-1 in token
    order (R = T*k);
  * the expert FFN is SiLU-gated: rows 0..I-1 of W1[e] are the gate, rows
    I..2I-1 the up projection, h = silu(gate) * up, y = W2[e] h;
  * the experts consume x rounded to bf16 (round to nearest even); the
    router consumes x as stored.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "as_f64", "bf16_round", "router_logits", "softmax", "topk_select", "gate_weights",
    "route", "expert_counts", "expert_offsets", "permutation", "swiglu_ffn",
    "moe_forward", "imbalance", "capacity_from_factor", "kept_mask",
]


def as_f64(t) -> np.ndarray:
    """Exact float64 copy of a torch tensor (any float dtype) or array."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().to("cpu")
            if t.dtype in (torch.bfloat16, torch.float16):
                t = t.float()
            return t.numpy().astype(np.float64)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def bf16_round(a) -> np.ndarray:
    """Round to the nearest bfloat16, ties to even; returns float64.

    bfloat16 keeps the upper 16 bits of an IEEE float32, so the value is
    first rounded to float32 and then to 8 significant bits by adding half an
    ulp of the kept part (plus the kept LSB for ties-to-even) and truncating.
    Inputs must be finite.
    """
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Router: [MegaMoE] §2.1  p = Softmax(W_r x_t);  [GroupedTP] §4.2 F.linear
# --------------------------------------------------------------------------
def router_logits(x, W_r, bias=None) -> np.ndarray:
    """l[t, e] = sum_c x[t, c] * W_r[e, c] (+ bias[e]); W_r is [E, d]."""
    l = as_f64(x) @ as_f64(W_r).T
    if bias is not None:
        l = l + as_f64(bias)[None, :]
    return l


def softmax(l) -> np.ndarray:
    """p[t, e] = exp(l[t, e] - max_e l) / sum_e' exp(l[t, e'] - max_e l)."""
    l = as_f64(l)
    z = np.exp(l - l.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def topk_select(l, k: int) -> np.ndarray:
    """k experts per token by repeated selection of the largest logit.

    Ties go to the lower expert index (numpy's argmax returns the first
    maximum); the result is ordered by descending logit.  [MegaMoE] §2.1,
    [DSMoE] §2.2.
    """
    l = as_f64(l)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    idx = np.empty((T, k), dtype=np.int64)
    taken = np.zeros((T, E), dtype=bool)
    rows = np.arange(T)
    for j in range(k):
        pick = np.argmax(np.where(taken, -np.inf, l), axis=1)
        idx[:, j] = pick
        taken[rows, pick] = True
    return idx


def gate_weights(p, idx, renormalize: bool = False) -> np.ndarray:
    """w[t, j] = p[t, idx[t, j]], optionally divided by sum_j of those."""
    p = as_f64(p)
    w = np.take_along_axis(p, np.asarray(idx), axis=1)
    if renormalize:
        w = w / w.sum(axis=1, keepdims=True)
    return w


def route(x, W_r, bias, k: int, renormalize: bool = False) -> dict:
    """Steps 1-2 of [GroupedTP] §2.2: logits, softmax, top-k, gate weights."""
    l = router_logits(x, W_r, bias)
    p = softmax(l)
    idx = topk_select(l, k)
    return dict(logits=l, p=p, idx=idx, w=gate_weights(p, idx, renormalize))


# --------------------------------------------------------------------------
# Permutation: [GroupedTP] §2.2 steps 3-4, §4.2 compute_expert_offsets
# --------------------------------------------------------------------------
def expert_counts(idx, E: int) -> np.ndarray:
    """counts[e] = number of (token, slot) pairs routed to expert e."""
    counts = np.zeros(E, dtype=np.int64)
    for e in np.asarray(idx).ravel():
        counts[e] += 1
    return counts


def expert_offsets(counts, shared_rows: int = 0) -> np.ndarray:
    """Exclusive prefix sum: offsets[e] = sum_{e' < e} counts[e'].

    offsets has E+1 entries (offsets[E] = total routed rows); with a shared
    expert one more entry closes its segment (offsets[E+1] = R + shared_rows).
    """
    counts = np.asarray(counts)
    n = len(counts) + 1 + (1 if shared_rows else 0)
    offsets = np.zeros(n, dtype=np.int64)
    running = 0
    for e, c in enumerate(counts):
        offsets[e] = running
        running += int(c)
    offsets[len(counts)] = running
    if shared_rows:
        offsets[len(counts) + 1] = running + shared_rows
    return offsets


def capacity_from_factor(factor: float, T: int, k: int, E: int) -> int:
    """Rows one expert may take: ceil(factor * T * k / E), the factor times an
    even share of the T*k routed rows ([GroupedTP] §5.1 caps each expert's
    tokens at inference by a capacity factor; [DSMoE] §3.2 bounds the share
    of a forward's tokens one expert may take)."""
    import math
    return max(1, math.ceil(factor * T * k / E))


def kept_mask(idx, capacity: int = 0) -> np.ndarray:
    """kept[t, j]: whether pair (t, j) is within its expert's capacity.

    An expert keeps its first `capacity` pairs in ascending token order (the
    order of its segment); the rest overflow.  capacity <= 0 keeps all.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    kept = np.ones((T, k), dtype=bool)
    if capacity <= 0:
        return kept
    seen = {}
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            seen[e] = seen.get(e, 0) + 1
            kept[t, j] = seen[e] <= capacity
    return kept


def permutation(idx, E: int, shared: bool = False, capacity: int = 0) -> dict:
    """Scatter plan of the expert-contiguous buffer.

    Within expert e's segment rows follow ascending token id, so the rank of
    token t in expert e is #{t' < t : e in sel(t')}.  Returns counts, offsets,
    row_to_token [R(+T)] and token_to_row [T, k].

    With capacity > 0 an expert keeps only its first `capacity` rows (pairs
    of rank >= capacity overflow: token_to_row = -1, no row); counts are the
    kept rows, offsets their exclusive scan, and the shared expert's rows
    follow the kept rows (offsets[E] .. offsets[E] + T - 1).  Rows past the
    last used one are unused (row_to_token = -1).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    kept = kept_mask(idx, capacity)
    counts = expert_counts(idx[kept], E)
    offsets = expert_offsets(counts, T if shared else 0)
    R = T * k
    used = int(offsets[E])
    row_to_token = np.full(R + (T if shared else 0), -1, dtype=np.int64)
    token_to_row = np.full((T, k), -1, dtype=np.int64)
    filled = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            if not kept[t, j]:
                continue
            e = idx[t, j]
            row = offsets[e] + filled[e]
            filled[e] += 1
            token_to_row[t, j] = row
            row_to_token[row] = t
    if shared:
        row_to_token[used:used + T] = np.arange(T)
    return dict(counts=counts, offsets=offsets, row_to_token=row_to_token,
                token_to_row=token_to_row, kept=kept)


def imbalance(counts) -> float:
    """max/mean of the per-expert token counts ([GroupedTP] §5.1: > 3 is severe)."""
    c = np.asarray(counts, dtype=np.float64)
    return float(c.max() / c.mean())


# --------------------------------------------------------------------------
# Expert FFN and combine: [MegaMoE] §2.1  y = E_shared(x) + sum p_i E_i(x)
# --------------------------------------------------------------------------
def swiglu_ffn(xrows, W1e, W2e) -> np.ndarray:
    """y = W2e (silu(W1e[:I] x) * (W1e[I:] x)) for each row x; fp64."""
    xrows = as_f64(xrows)
    W1e = as_f64(W1e)
    W2e = as_f64(W2e)
    I = W1e.shape[0] // 2
    g = xrows @ W1e[:I].T
    u = xrows @ W1e[I:].T
    h = g / (1.0 + np.exp(-g)) * u
    return h @ W2e.T


def moe_forward(x, W_r, bias, W1, W2, W1s=None, W2s=None, k: int = 2,
                renormalize: bool = False, tokens=None, idx=None, w=None, capacity: int = 0) -> dict:
    """out[t] = E_shared(x_t) + sum_{j<k, kept} w[t, j] * E_{idx[t, j]}(x_t).

    W1 / W2 may be any object indexable by expert id (W1[e] -> [2I, d],
    W2[e] -> [d, I]); only the experts some token selects are touched.
    `tokens` restricts the computation to those token ids (routing included).
    `idx` / `w`, when given (shape [len(tokens), k]), replace this oracle's
    own routing (used where the caller adopts another router's choice at a
    near tie).  With capacity > 0 each expert takes only its first
    `capacity` pairs in token order (kept_mask); an overflowing pair adds
    nothing: its token keeps the shared expert and its other experts, with
    their gate weights unchanged (the pages' "fallback path" for tokens over
    capacity is the shared expert / residual the layer already has).
    Capacity applies to the whole batch, so it must not be combined with
    `tokens` (a subset would see other ranks).
    """
    if capacity > 0 and tokens is not None:
        raise ValueError("capacity is a whole-batch limit: pass the batch itself, not a token subset")
    xs = x if tokens is None else x[tokens]
    r = route(xs, W_r, bias, k, renormalize)
    if idx is not None:
        r["idx"] = np.asarray(idx)
        r["w"] = as_f64(w) if w is not None else gate_weights(r["p"], r["idx"], renormalize)
    sel, wts = r["idx"], r["w"]
    kept = kept_mask(sel, capacity)
    r["kept"] = kept
    xe = bf16_round(as_f64(xs))
    out = np.zeros((xe.shape[0], xe.shape[1]), dtype=np.float64)
    if W1s is not None:
        out += swiglu_ffn(xe, W1s, W2s)
    for e in np.unique(sel[kept]):
        t_rows, slots = np.nonzero((sel == e) & kept)
        y = swiglu_ffn(xe[t_rows], W1[int(e)], W2[int(e)])
        out[t_rows] += wts[t_rows, slots][:, None] * y
    r["out"] = out
    return r
