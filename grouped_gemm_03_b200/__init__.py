"""Python binding of libmoe.so, the B200 (sm_100a) MoE-layer forward library.

Argument marshalling only: every function here checks dtypes, allocates the
output tensors with torch (device memory is PyTorch's job) and calls the C
entry point of the same name on the current CUDA stream.  All computation
happens in the library's CUDA kernels; there is no fallback path, and a
missing or unloadable library raises immediately.

Build the library with ``python -m grouped_gemm_03_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

__all__ = [
    "LIB_PATH", "MoEError", "MoEConfig", "lib", "exported_symbols", "status_string", "device_info",
    "router_topk", "topk_logits", "permute", "grouped_gemm", "combine", "quantize_weights_fp8",
    "capacity_from_factor", "forward_launches", "grouped_gemm_gather",
    "workspace_size", "moe_forward", "moe_forward_marked", "moe_forward_host", "host_staging_size", "read_device_status",
    "MOE_F32", "MOE_F16", "MOE_BF16", "MOE_E4M3", "MOE_MXE4M3", "MOE_FLAG_GATHER_A", "EPI_NONE", "EPI_SILU_GATE",
    "quantize_weights_mx",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_F32, MOE_F16, MOE_BF16, MOE_E4M3, MOE_MXE4M3 = 0, 1, 2, 3, 4
MOE_FLAG_GATHER_A = 1
EPI_NONE, EPI_SILU_GATE = 0, 1
_STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_WORKSPACE",
           -4: "MOE_ERR_CUDA", -5: "MOE_ERR_BAD_OFFSETS", -6: "MOE_ERR_TIMEOUT"}

_TORCH_DT = {torch.float32: MOE_F32, torch.float16: MOE_F16, torch.bfloat16: MOE_BF16,
             torch.float8_e4m3fn: MOE_E4M3, torch.uint8: MOE_E4M3}


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class MoEConfig(ctypes.Structure):
    """Mirror of `moe_config` in include/moe.h."""
    _fields_ = [(n, ctypes.c_int) for n in ("T", "d", "E", "k", "inter", "shared_inter", "x_dtype",
                                            "router_dtype", "expert_dtype", "out_dtype", "renormalize",
                                            "capacity", "flags")]


_vp, _i, _sz, _fp, _ip = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
_CFG = ctypes.POINTER(MoEConfig)

# name -> (restype, argtypes); the full C ABI of include/moe.h
_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [_i]),
    "moe_last_error_string": (ctypes.c_char_p, []),
    "moe_device_info": (_i, [ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "moe_read_device_status": (_i, [_vp, _vp, ctypes.POINTER(_i)]),
    "moe_router_workspace_size": (_sz, [_i, _i]),
    "moe_router_topk": (_i, [_vp, _i, _vp, _i, _fp, _i, _i, _i, _i, _i, _fp, _ip, _fp, _vp, _sz, _vp]),
    "moe_topk_logits": (_i, [_vp, _i, _i, _i, _i, _i, _ip, _fp, _vp]),
    "moe_permute_workspace_size": (_sz, [_i, _i]),
    "moe_permute": (_i, [_vp, _i, _ip, _i, _i, _i, _i, _i, _i, _vp, _fp, _ip, _ip, _ip, _ip, _vp, _sz, _vp]),
    "moe_permute_capacity": (_i, [_vp, _i, _ip, _i, _i, _i, _i, _i, _i, _i, _vp, _fp, _ip, _ip, _ip, _ip, _vp, _sz,
                                  _vp]),
    "moe_permute_noalloc": (_i, [_vp, _i, _ip, _i, _i, _i, _i, _i, _i, _vp, _fp, _ip, _ip, _ip, _ip, _vp]),
    "moe_grouped_gemm_workspace_size": (_sz, []),
    "moe_grouped_gemm_plan": (ctypes.c_char_p, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "moe_grouped_gemm": (_i, [_vp, _fp, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, _vp, _i, _fp, _vp, _sz, _vp]),
    "moe_grouped_gemm_gather": (_i, [_vp, _fp, _i, _ip, _vp, _fp, _ip, _i, _i, _i, _i, _i, _i, _vp, _i, _fp, _vp, _sz,
                                     _vp]),
    "moe_combine": (_i, [_vp, _ip, _fp, _i, _i, _i, _i, _vp, _i, _vp]),
    "moe_combine_plan": (_i, [_vp, _ip, _fp, _ip, _i, _i, _i, _i, _i, _vp, _i, _vp]),
    "moe_selftest_workspace_size": (_sz, []),
    "moe_selftest_stalled_pipeline": (_i, [_vp, _sz, ctypes.c_ulonglong, _vp]),
    "moe_quantize_weights_fp8": (_i, [_vp, _i, _i, _i, _vp, _fp, _vp]),
    "moe_quantize_weights_mx": (_i, [_vp, _i, _i, _i, _vp, _fp, _vp]),
    "moe_workspace_size": (_sz, [_CFG]),
    "moe_forward": (_i, [_CFG, _vp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _ip, _vp, _sz, _vp]),
    "moe_forward_marked": (_i, [_CFG, _vp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _ip, _vp, _sz,
                                ctypes.POINTER(ctypes.c_void_p), _vp]),
    "moe_host_staging_size": (_sz, [_CFG]),
    "moe_forward_launches": (_i, [_CFG]),
    "moe_forward_host": (_i, [_CFG, _vp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _fp, _vp, _vp, _sz, _vp]),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m grouped_gemm_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def exported_symbols() -> list[str]:
    return sorted(_SIGS)


def status_string(status: int) -> str:
    try:
        return lib().moe_status_string(int(status)).decode()
    except Exception:  # pragma: no cover - library missing
        return _STATUS.get(int(status), "unknown")


def _check(status: int, what: str) -> None:
    if status != 0:
        if status == -4:
            what = f"{what} [{lib().moe_last_error_string().decode()}]"
        raise MoEError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    try:
        return _TORCH_DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _scratch(nbytes: int, device) -> torch.Tensor:
    # 256-byte aligned (torch's caching allocator hands out 512-byte aligned blocks)
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def device_info() -> tuple[int, int, int]:
    n, a, b = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    st = lib().moe_device_info(ctypes.byref(n), ctypes.byref(a), ctypes.byref(b))
    if st not in (0, -2):
        _check(st, "moe_device_info")
    return n.value, a.value, b.value


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return the status word at the start of `ws`."""
    v = ctypes.c_int()
    _check(lib().moe_read_device_status(_ptr(ws), _stream(stream), ctypes.byref(v)), "moe_read_device_status")
    return v.value


# ---------------------------------------------------------------- router
def router_topk(x, W_r, k: int, bias=None, renormalize: bool = False, want_logits: bool = False, ws=None,
                stream=None):
    """(topk_idx [T,k] int32, topk_w [T,k] fp32[, logits [T,E] fp32])."""
    _cuda(x, W_r, bias)
    T, d = x.shape
    E = W_r.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    logits = torch.empty((T, E), dtype=torch.float32, device=x.device) if want_logits else None
    L = lib()
    if ws is None:
        ws = _scratch(L.moe_router_workspace_size(T, E), x.device)
    _check(L.moe_router_topk(_ptr(x), _dt(x), _ptr(W_r), _dt(W_r), _ptr(bias), T, d, E, k, int(renormalize),
                             _ptr(logits), _ptr(idx), _ptr(w), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_router_topk")
    return (idx, w, logits) if want_logits else (idx, w)


def topk_logits(logits, k: int, renormalize: bool = False, out_idx=None, out_w=None, stream=None):
    _cuda(logits)
    N, E = logits.shape
    idx = out_idx if out_idx is not None else torch.empty((N, k), dtype=torch.int32, device=logits.device)
    w = out_w if out_w is not None else torch.empty((N, k), dtype=torch.float32, device=logits.device)
    _check(lib().moe_topk_logits(_ptr(logits), _dt(logits), N, E, k, int(renormalize), _ptr(idx), _ptr(w),
                                 _stream(stream)), "moe_topk_logits")
    return idx, w


# ---------------------------------------------------------------- permute
def permute(x, topk_idx, E: int, append_shared: bool = False, fp8: bool = False, ws=None, stream=None,
            capacity: int = 0, mx: bool = False) -> dict:
    """Histogram, scan and scatter (moe_permute; moe_permute_capacity when capacity > 0).
    fp8: E4M3 rows with 1x128 scales (mx: power-of-two scales)."""
    _cuda(x, topk_idx)
    T, d = x.shape
    k = topk_idx.shape[1]
    rows = T * k + (T if append_shared else 0)
    dev = x.device
    xp = torch.empty((rows, d), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    xps = torch.empty((d // 128, rows), dtype=torch.float32, device=dev) if fp8 else None
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1 + (1 if append_shared else 0), dtype=torch.int32, device=dev)
    r2t = torch.empty(rows, dtype=torch.int32, device=dev)
    t2r = torch.empty((T, k), dtype=torch.int32, device=dev)
    L = lib()
    if ws is None:
        ws = _scratch(L.moe_permute_workspace_size(T, E), dev)
    if capacity:
        _check(L.moe_permute_capacity(_ptr(x), _dt(x), _ptr(topk_idx), T, d, E, k, int(append_shared), int(capacity),
                                      (MOE_MXE4M3 if mx else MOE_E4M3) if fp8 else MOE_BF16, _ptr(xp), _ptr(xps),
                                      _ptr(counts),
                                      _ptr(offsets), _ptr(r2t), _ptr(t2r), _ptr(ws), ws.numel(), _stream(stream)),
               "moe_permute_capacity")
    else:
        _check(L.moe_permute(_ptr(x), _dt(x), _ptr(topk_idx), T, d, E, k, int(append_shared),
                             (MOE_MXE4M3 if mx else MOE_E4M3) if fp8 else MOE_BF16, _ptr(xp), _ptr(xps),
                             _ptr(counts), _ptr(offsets),
                             _ptr(r2t), _ptr(t2r), _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
    return dict(xp=xp, xp_scales=xps, counts=counts, offsets=offsets, row_to_token=r2t, token_to_row=t2r, ws=ws)


# ---------------------------------------------------------------- grouped GEMM
def grouped_gemm(A, B, offsets, N: int, epilogue: int = EPI_NONE, c_dtype=torch.bfloat16, A_scales=None,
                 B_scales=None, out=None, out_scales=None, ws=None, stream=None, mx: bool = False):
    """C [rows, N] for groups offsets[g]..offsets[g+1] of A against B[g] ([G, Nb, K]).

    E4M3 operands are uint8 codes with fp32 scales; mx=True says the scales are
    powers of two (MOE_MXE4M3: applied by the tensor core), and an E4M3 C then
    gets power-of-two scales too."""
    _cuda(A, B, offsets, A_scales, B_scales)
    rows, K = A.shape
    G = B.shape[0]
    fp8 = A.dtype in (torch.uint8, torch.float8_e4m3fn)
    q8 = MOE_MXE4M3 if mx else MOE_E4M3
    cdt = {torch.bfloat16: MOE_BF16, torch.float32: MOE_F32, torch.uint8: q8}[c_dtype]
    C = out if out is not None else torch.empty((rows, N), dtype=c_dtype, device=A.device)
    Cs = out_scales
    if cdt == q8 and Cs is None:
        Cs = torch.empty((N // 128, rows), dtype=torch.float32, device=A.device)
    L = lib()
    if ws is None:
        ws = _scratch(L.moe_grouped_gemm_workspace_size(), A.device)
    _check(L.moe_grouped_gemm(_ptr(A), _ptr(A_scales), _ptr(B), _ptr(B_scales), _ptr(offsets), G, rows, N, K,
                              q8 if fp8 else MOE_BF16, epilogue, _ptr(C), cdt, _ptr(Cs), _ptr(ws), ws.numel(),
                              _stream(stream)), "moe_grouped_gemm")
    return (C, Cs) if cdt == q8 else C


def grouped_gemm_gather(A, A_rows, B, offsets, N: int, epilogue: int = EPI_NONE, c_dtype=torch.bfloat16,
                        A_scales=None, B_scales=None, out=None, out_scales=None, ws=None, stream=None,
                        mx: bool = False):
    """grouped_gemm whose A row r is row A_rows[r] of A (moe_grouped_gemm_gather); C has len(A_rows) rows."""
    _cuda(A, A_rows, B, offsets, A_scales, B_scales)
    src_rows, K = A.shape
    rows = A_rows.numel()
    G = B.shape[0]
    fp8 = A.dtype in (torch.uint8, torch.float8_e4m3fn)
    q8 = MOE_MXE4M3 if mx else MOE_E4M3
    cdt = {torch.bfloat16: MOE_BF16, torch.float32: MOE_F32, torch.uint8: q8}[c_dtype]
    C = out if out is not None else torch.empty((rows, N), dtype=c_dtype, device=A.device)
    Cs = out_scales
    if cdt == q8 and Cs is None:
        Cs = torch.empty((N // 128, rows), dtype=torch.float32, device=A.device)
    L = lib()
    if ws is None:
        ws = _scratch(L.moe_grouped_gemm_workspace_size(), A.device)
    _check(L.moe_grouped_gemm_gather(_ptr(A), _ptr(A_scales), src_rows, _ptr(A_rows), _ptr(B), _ptr(B_scales),
                                     _ptr(offsets), G, rows, N, K, q8 if fp8 else MOE_BF16, epilogue, _ptr(C), cdt,
                                     _ptr(Cs), _ptr(ws), ws.numel(), _stream(stream)), "moe_grouped_gemm_gather")
    return (C, Cs) if cdt == q8 else C


# ---------------------------------------------------------------- combine
def grouped_gemm_plan(G: int, rows: int, N: int, K: int, ab_dtype: int = MOE_BF16, epilogue: int = EPI_NONE,
                      c_dtype: int = MOE_BF16, extra_groups: int = 0, num_sms: int = 0) -> str:
    """Which kernel a grouped GEMM of this shape runs on (host arithmetic only)."""
    return lib().moe_grouped_gemm_plan(G, extra_groups, rows, N, K, ab_dtype, epilogue, c_dtype,
                                       num_sms).decode()


def combine(Y, token_to_row, topk_w, has_shared: bool, out_dtype=torch.bfloat16, out=None, stream=None,
            offsets=None):
    """Gather, weight and sum (moe_combine; with the permute's `offsets`, moe_combine_plan:
    shared rows from offsets[E], overflowed slots skipped)."""
    _cuda(Y, token_to_row, topk_w, offsets)
    T, k = token_to_row.shape
    d = Y.shape[1]
    o = out if out is not None else torch.empty((T, d), dtype=out_dtype, device=Y.device)
    if offsets is not None:
        E = offsets.numel() - 1 - (1 if has_shared else 0)
        _check(lib().moe_combine_plan(_ptr(Y), _ptr(token_to_row), _ptr(topk_w), _ptr(offsets), E, int(has_shared),
                                      T, d, k, _ptr(o), _dt(o), _stream(stream)), "moe_combine_plan")
        return o
    _check(lib().moe_combine(_ptr(Y), _ptr(token_to_row), _ptr(topk_w), int(has_shared), T, d, k, _ptr(o),
                             _dt(o), _stream(stream)), "moe_combine")
    return o


# ---------------------------------------------------------------- FP8 weights
def quantize_weights_fp8(W, stream=None):
    """W [G, N, K] bf16 -> (codes uint8 [G, N, K], scales fp32 [G, N/128, K/128])."""
    _cuda(W)
    squeeze = W.dim() == 2
    W3 = W.unsqueeze(0) if squeeze else W
    G, N, K = W3.shape
    q = torch.empty((G, N, K), dtype=torch.uint8, device=W.device)
    s = torch.empty((G, N // 128, K // 128), dtype=torch.float32, device=W.device)
    _check(lib().moe_quantize_weights_fp8(_ptr(W3), G, N, K, _ptr(q), _ptr(s), _stream(stream)),
           "moe_quantize_weights_fp8")
    return (q[0], s[0]) if squeeze else (q, s)


def quantize_weights_mx(W, stream=None):
    """As quantize_weights_fp8, with power-of-two block scales (MOE_MXE4M3)."""
    _cuda(W)
    squeeze = W.dim() == 2
    W3 = W.unsqueeze(0) if squeeze else W
    G, N, K = W3.shape
    q = torch.empty((G, N, K), dtype=torch.uint8, device=W.device)
    s = torch.empty((G, N // 128, K // 128), dtype=torch.float32, device=W.device)
    _check(lib().moe_quantize_weights_mx(_ptr(W3), G, N, K, _ptr(q), _ptr(s), _stream(stream)),
           "moe_quantize_weights_mx")
    return (q[0], s[0]) if squeeze else (q, s)


# ---------------------------------------------------------------- whole layer
def make_config(T, d, E, k, inter, shared_inter=0, x_dtype=MOE_BF16, router_dtype=MOE_BF16,
                expert_dtype=MOE_BF16, out_dtype=MOE_BF16, renormalize=False, capacity=0, flags=0) -> MoEConfig:
    return MoEConfig(T, d, E, k, inter, shared_inter, x_dtype, router_dtype, expert_dtype, out_dtype,
                     int(renormalize), int(capacity), int(flags))


def capacity_from_factor(factor: float, T: int, k: int, E: int) -> int:
    """Per-expert row limit for a capacity factor: ceil(factor * T * k / E), at least 1."""
    import math
    return max(1, math.ceil(factor * T * k / E))


def workspace_size(cfg: MoEConfig) -> int:
    n = lib().moe_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise MoEError(-1, "moe_workspace_size")
    return n


def host_staging_size(cfg: MoEConfig) -> int:
    return lib().moe_host_staging_size(ctypes.byref(cfg))


def forward_launches(cfg: MoEConfig) -> int:
    """Kernels one moe_forward of this shape launches (host arithmetic)."""
    return lib().moe_forward_launches(ctypes.byref(cfg))


@dataclass
class ExpertWeights:
    """Expert weights as the library consumes them (bf16, or E4M3 codes + scales)."""
    W1: torch.Tensor
    W2: torch.Tensor
    W1s: torch.Tensor | None = None
    W2s: torch.Tensor | None = None
    W1_scales: torch.Tensor | None = None
    W2_scales: torch.Tensor | None = None
    W1s_scales: torch.Tensor | None = None
    W2s_scales: torch.Tensor | None = None


def moe_forward(cfg: MoEConfig, x, W_r, bias, w: ExpertWeights, out=None, counts_out=None, ws=None, stream=None):
    _cuda(x, W_r, bias, w.W1, w.W2, w.W1s, w.W2s)
    dt = torch.float32 if cfg.out_dtype == MOE_F32 else torch.bfloat16
    o = out if out is not None else torch.empty((cfg.T, cfg.d), dtype=dt, device=x.device)
    if ws is None:
        ws = _scratch(workspace_size(cfg), x.device)
    _check(lib().moe_forward(ctypes.byref(cfg), _ptr(x), _ptr(W_r), _ptr(bias), _ptr(w.W1), _ptr(w.W1_scales),
                             _ptr(w.W2), _ptr(w.W2_scales), _ptr(w.W1s), _ptr(w.W1s_scales), _ptr(w.W2s),
                             _ptr(w.W2s_scales), _ptr(o), _ptr(counts_out), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_forward")
    return o


def moe_forward_marked(cfg: MoEConfig, x, W_r, bias, w: ExpertWeights, events, out, counts_out=None, ws=None,
                       stream=None):
    """moe_forward that records the six torch.cuda.Event objects in `events` around its five kernels
    (router, permute, up GEMM, down GEMM, combine) for per-kernel timing inside the whole layer."""
    _cuda(x, W_r, bias, w.W1, w.W2, w.W1s, w.W2s)
    if len(events) != 6:
        raise ValueError("six events: before each of the five stages and after the last")
    st = torch.cuda.current_stream() if stream is None else stream
    for e in events:
        if not e.cuda_event:  # torch creates the CUDA event on its first record
            e.record(st)
    handles = (ctypes.c_void_p * 6)(*[e.cuda_event for e in events])
    if ws is None:
        ws = _scratch(workspace_size(cfg), x.device)
    _check(lib().moe_forward_marked(ctypes.byref(cfg), _ptr(x), _ptr(W_r), _ptr(bias), _ptr(w.W1),
                                    _ptr(w.W1_scales), _ptr(w.W2), _ptr(w.W2_scales), _ptr(w.W1s),
                                    _ptr(w.W1s_scales), _ptr(w.W2s), _ptr(w.W2s_scales), _ptr(out),
                                    _ptr(counts_out), _ptr(ws), ws.numel(), handles, _stream(st)),
           "moe_forward_marked")
    return out


def moe_forward_host(cfg: MoEConfig, x_host, W_r, bias, w: ExpertWeights, out_host, ws, stream=None):
    """x_host / out_host are CPU tensors (pinned for asynchronous copies); no synchronisation."""
    if x_host.is_cuda or out_host.is_cuda:
        raise ValueError("x_host and out_host must be host tensors")
    _check(lib().moe_forward_host(ctypes.byref(cfg), _ptr(x_host), _ptr(W_r), _ptr(bias), _ptr(w.W1),
                                  _ptr(w.W1_scales), _ptr(w.W2), _ptr(w.W2_scales), _ptr(w.W1s),
                                  _ptr(w.W1s_scales), _ptr(w.W2s), _ptr(w.W2s_scales), _ptr(out_host), _ptr(ws),
                                  ws.numel(), _stream(stream)), "moe_forward_host")
    return out_host
