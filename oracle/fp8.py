"""FP8 (E4M3) quantisation and the FP8 MoE forward -- TEST INFRASTRUCTURE ONLY.

Follows [MegaMoE] ("MegaMoE math model -> DeepGEMM source walk-through",
2kiu.com news 6052262) §2.3 and §5.1: E4M3 for the forward pass, one scale
per token per 128-element group of activations (1x128) and one per 128x128
block of weights, fp32 accumulation, and the scaled product
C ~ (A_q / scale_A)(B_q / scale_B) scale_C.

Readings (the pages leave these open):
  * a scale s is stored as the DEQUANTISING multiplier (a ~ q * s), i.e. the
    page's scale_A is 1/s and scale_C = 1;
  * s = fp32(amax / 448) with IEEE float32 division (s = 1 when amax = 0),
    q = E4M3(fp32(a / s)) with IEEE float32 division, E4M3 rounding to
    nearest even with saturation to +-448 (OCP 8-bit floating point:
    bias 7, no infinities, code 0x7F/0xFF = NaN, subnormals down to 2^-9);
  * the scales vary along K, so the product is promoted per 128-wide K
    block: C = sum_kb (sum_{k in kb} qa qb) * sa[m, kb] * sb[n/128, kb];
  * the intermediate h = silu(gate) * up is rounded to fp32 and quantised per
    row per 128 columns before the down projection;
  * the router stays in bf16; the shared expert runs in FP8 like the others.

MX variant (pow2=True): the same groups (1x128 per token, 128x128 per weight
block), but each scale is the smallest power of two s = 2^p with
448 * s >= amax (s = 1 when amax = 0; 2^-127 <= s <= 2^127, the range of an
8-bit exponent), so that the tensor core can apply it as a UE8M0 block
scale ([MegaMoE] §5.1 folds the scales into the GEMM; with power-of-two
scales the MMA does it in hardware).  q = E4M3(fp32(a / s)) as before; a / s
is exact in fp32.  The GEMM is the same blockwise sum, with these scales.
"""
from __future__ import annotations

import numpy as np

from .moe_oracle import as_f64, bf16_round, route

__all__ = [
    "E4M3_MAX", "e4m3_magnitudes", "e4m3_decode", "e4m3_encode", "pow2_scale_of", "quantize_1x128",
    "quantize_128x128", "dequantize_1x128", "dequantize_128x128", "fp8_gemm",
    "swiglu_ffn_fp8", "quantize_expert", "moe_forward_fp8",
]

E4M3_MAX = 448.0


def e4m3_magnitudes() -> np.ndarray:
    """Values of the non-negative finite codes 0x00..0x7E, ascending with the code."""
    vals = np.empty(127, dtype=np.float64)
    for code in range(127):
        e, m = code >> 3, code & 7
        vals[code] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_MAGS = e4m3_magnitudes()


def e4m3_decode(codes) -> np.ndarray:
    """uint8 E4M3 codes -> float64 (0x7F / 0xFF decode to NaN)."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = c & 0x7F
    v = np.where(mag == 0x7F, np.nan, _MAGS[np.minimum(mag, 126)])
    return np.where(c & 0x80, -v, v)


def e4m3_encode(v) -> np.ndarray:
    """float32 values -> E4M3 codes, round to nearest (ties to even code), saturating.

    The sign bit is kept, so a negative value that rounds to zero gives 0x80.
    Inputs must be finite.
    """
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v).astype(np.float64)
    hi = np.clip(np.searchsorted(_MAGS, a, side="left"), 1, 126)
    lo = hi - 1
    dlo = a - _MAGS[lo]
    dhi = _MAGS[hi] - a
    code = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    code = np.where(a >= E4M3_MAX, 126, code).astype(np.uint8)
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)


def _scale_of(amax32: np.ndarray) -> np.ndarray:
    s = (amax32.astype(np.float32) / np.float32(E4M3_MAX)).astype(np.float32)
    return np.where(amax32 == 0, np.float32(1.0), s).astype(np.float32)


def pow2_scale_of(amax32) -> np.ndarray:
    """Smallest power of two s = 2^p with 448 * s >= amax (exact comparisons in
    fp64), p clamped to the UE8M0 exponent range [-127, 127]; s = 1 for amax = 0."""
    amax = np.asarray(amax32, dtype=np.float32).astype(np.float64)
    safe = np.where(amax > 0, amax, E4M3_MAX)
    p = np.ceil(np.log2(safe / E4M3_MAX)).astype(np.int64)
    # log2 is rounded: settle p by exact comparisons against 448 * 2^p
    p = np.where(np.ldexp(E4M3_MAX, p) < safe, p + 1, p)
    p = np.where(np.ldexp(E4M3_MAX, p - 1) >= safe, p - 1, p)
    p = np.clip(np.where(amax > 0, p, 0), -127, 127)
    return np.ldexp(np.float64(1.0), p).astype(np.float32)


def quantize_1x128(a, pow2: bool = False) -> tuple[np.ndarray, np.ndarray]:
    """Per row, per 128-column group: (codes [M, K], scales [M, K/128] fp32).

    pow2: power-of-two (MX) scales instead of amax/448."""
    a = np.asarray(a, dtype=np.float32)
    M, K = a.shape
    if K % 128:
        raise ValueError("K must be a multiple of 128")
    g = a.reshape(M, K // 128, 128)
    amax = np.abs(g).max(axis=2)
    s = pow2_scale_of(amax) if pow2 else _scale_of(amax)
    q = e4m3_encode((g / s[:, :, None]).astype(np.float32))
    return q.reshape(M, K), s


def quantize_128x128(W, pow2: bool = False) -> tuple[np.ndarray, np.ndarray]:
    """Per 128x128 block: (codes [N, K], scales [N/128, K/128] fp32).

    pow2: power-of-two (MX) scales instead of amax/448."""
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    if N % 128 or K % 128:
        raise ValueError("N and K must be multiples of 128")
    b = W.reshape(N // 128, 128, K // 128, 128)
    amax = np.abs(b).max(axis=(1, 3))
    s = pow2_scale_of(amax) if pow2 else _scale_of(amax)
    q = e4m3_encode((b / s[:, None, :, None]).astype(np.float32))
    return q.reshape(N, K), s


def dequantize_1x128(q, s) -> np.ndarray:
    M, K = q.shape
    return (e4m3_decode(q).reshape(M, K // 128, 128) * as_f64(s)[:, :, None]).reshape(M, K)


def dequantize_128x128(q, s) -> np.ndarray:
    N, K = q.shape
    d = e4m3_decode(q).reshape(N // 128, 128, K // 128, 128) * as_f64(s)[:, None, :, None]
    return d.reshape(N, K)


def fp8_gemm(qa, sa, qb, sb) -> np.ndarray:
    """C[m, n] = sum_kb (sum_{k in kb} qa[m,k] qb[n,k]) * sa[m,kb] * sb[n//128, kb] (fp64)."""
    A = e4m3_decode(qa)
    B = e4m3_decode(qb)
    sa = as_f64(sa)
    sb = as_f64(sb)
    M, K = A.shape
    N = B.shape[0]
    C = np.zeros((M, N), dtype=np.float64)
    for kb in range(K // 128):
        ks = slice(128 * kb, 128 * kb + 128)
        partial = A[:, ks] @ B[:, ks].T
        C += partial * sa[:, kb][:, None] * np.repeat(sb[:, kb], 128)[None, :]
    return C


def swiglu_ffn_fp8(xq, sx, W1q, s1, W2q, s2, pow2: bool = False) -> dict:
    """SiLU-gated FFN on quantised operands; h is re-quantised 1x128 (power-of-two scales with pow2)."""
    I = W1q.shape[0] // 2
    gu = fp8_gemm(xq, sx, W1q, s1)
    g, u = gu[:, :I], gu[:, I:]
    h = g / (1.0 + np.exp(-g)) * u
    hq, sh = quantize_1x128(h.astype(np.float32), pow2)
    return dict(h=h, hq=hq, sh=sh, y=fp8_gemm(hq, sh, W2q, s2))


def quantize_expert(W1e, W2e, pow2: bool = False) -> tuple:
    """One expert's weights (bf16 values) quantised per 128x128 block: (W1q, s1, W2q, s2)."""
    W1q, s1 = quantize_128x128(as_f64(W1e), pow2)
    W2q, s2 = quantize_128x128(as_f64(W2e), pow2)
    return W1q, s1, W2q, s2


def moe_forward_fp8(x, W_r, bias, W1, W2, W1s=None, W2s=None, k: int = 2,
                    renormalize: bool = False, tokens=None, idx=None, w=None,
                    quantized=None, workers: int = 1, capacity: int = 0, pow2: bool = False) -> dict:
    """FP8 variant of oracle.moe_forward: same routing, quantised expert GEMMs.

    Each expert's W1[e] / W2[e] (bf16 values) is quantised per 128x128 block;
    x (as bf16) per token per 128 columns.  `quantized`, when given, maps an
    expert id to its quantize_expert() result (computed once, e.g. for two
    workloads with the same weights).  With workers > 1 the experts are
    evaluated on that many threads; each expert's rows are computed exactly as
    with one thread and the weighted outputs are still added in ascending
    expert order, so the result does not depend on `workers`.  `capacity`
    drops the pairs over an expert's capacity exactly as oracle.moe_forward
    does (kept_mask).  pow2 selects the MX variant: every scale (x, the
    weights, h) is a power of two (pow2_scale_of).
    """
    from .moe_oracle import kept_mask
    if capacity > 0 and tokens is not None:
        raise ValueError("capacity is a whole-batch limit: pass the batch itself, not a token subset")
    xs = x if tokens is None else x[tokens]
    r = route(xs, W_r, bias, k, renormalize)
    if idx is not None:
        from .moe_oracle import gate_weights
        r["idx"] = np.asarray(idx)
        r["w"] = as_f64(w) if w is not None else gate_weights(r["p"], r["idx"], renormalize)
    sel, wts = r["idx"], r["w"]
    kept = kept_mask(sel, capacity)
    r["kept"] = kept
    xe = bf16_round(as_f64(xs)).astype(np.float32)
    xq, sx = quantize_1x128(xe, pow2)
    out = np.zeros(xe.shape, dtype=np.float64)
    if W1s is not None:
        W1q, s1, W2q, s2 = quantize_expert(W1s, W2s, pow2)
        out += swiglu_ffn_fp8(xq, sx, W1q, s1, W2q, s2, pow2)["y"]

    def expert_rows(e):
        t_rows, slots = np.nonzero((sel == e) & kept)
        q = quantized[int(e)] if quantized is not None else quantize_expert(W1[int(e)], W2[int(e)], pow2)
        y = swiglu_ffn_fp8(xq[t_rows], sx[t_rows], *q, pow2=pow2)["y"]
        return t_rows, wts[t_rows, slots][:, None] * y

    experts = np.unique(sel[kept])
    if workers > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(workers) as ex:
            parts = list(ex.map(expert_rows, experts))
    else:
        parts = [expert_rows(e) for e in experts]
    for t_rows, contrib in parts:   # ascending expert order
        out[t_rows] += contrib
    r.update(out=out, xq=xq, sx=sx)
    return r
