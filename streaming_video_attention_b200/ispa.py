"""Thin ctypes binding of libispa (include/ispa.h). Argument marshalling only: every step
of the computation runs in the library's CUDA kernels. torch tensors are used for device
memory and streams; the library sees raw pointers.

Importing this module loads nothing. The first call loads libispa.so from the package
directory and raises if it is missing: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libispa.so")

ISPA_OK = 0
ISPA_ERR_INVALID_ARG = -1
ISPA_ERR_UNSUPPORTED = -2
ISPA_ERR_CUDA = -3
ISPA_ERR_NOT_SPD = -4
ISPA_ERR_TIMEOUT = -5
ISPA_ERR_WORKSPACE = -6

ISPA_BF16 = 0
ISPA_FP32 = 1

EXPORTS = (
    "ispa_attn_split", "ispa_attn_split_noalloc", "ispa_accum_stats", "ispa_stats_reset", "ispa_solve_absorb",
    "ispa_absorb_error", "ispa_quantize_w8", "ispa_project_w8a8", "ispa_select_layers", "ispa_rewarm_check",
    "ispa_quantize_q_i8", "ispa_k_blocks", "ispa_quantize_k_i8", "ispa_attn_split_i8",
    "ispa_attn_split_ops", "ispa_accum_ops",
    "ispa_local_attn", "ispa_project", "ispa_workspace_bytes", "ispa_device_status", "ispa_selftest_bounded_wait",
    "ispa_selftest_exp2_poly", "ispa_set_attn_kernel", "ispa_kernel_launches", "ispa_last_error", "ispa_version",
)


class IspaError(RuntimeError):
    def __init__(self, code: int, func: str, msg: str):
        super().__init__(f"{func} failed ({code}): {msg}")
        self.code = code


class AttnDesc(ctypes.Structure):
    _fields_ = [
        ("n_q", ctypes.c_int), ("n_kv", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("sink_begin", ctypes.c_int), ("sink_end", ctypes.c_int),
        ("chunk_begin", ctypes.c_int), ("chunk_end", ctypes.c_int),
        ("scale", ctypes.c_float), ("dtype", ctypes.c_int),
    ]


class CStats(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("G", ctypes.c_void_p), ("C", ctypes.c_void_p), ("H", ctypes.c_void_p),
                ("rows", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libispa.so (once). Raises if the library has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m streaming_video_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        L.ispa_attn_split.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      ctypes.POINTER(CStats), vp, sz, vp]
        L.ispa_attn_split_noalloc.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                              ctypes.POINTER(CStats), vp]
        L.ispa_attn_split_i8.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                         ctypes.POINTER(CStats), vp, sz, vp]
        L.ispa_quantize_q_i8.argtypes = [vp, i, i, i, vp, vp, vp]
        L.ispa_attn_split_ops.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.ispa_accum_ops.argtypes = [ctypes.POINTER(CStats), i, vp, vp, i, i, vp]
        L.ispa_k_blocks.argtypes = [ctypes.POINTER(AttnDesc)]
        L.ispa_quantize_k_i8.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp]
        L.ispa_accum_stats.argtypes = [ctypes.POINTER(CStats), vp, vp, i, i, vp, sz, vp]
        L.ispa_stats_reset.argtypes = [ctypes.POINTER(CStats), vp]
        L.ispa_solve_absorb.argtypes = [ctypes.POINTER(CStats), i, ctypes.POINTER(vp), i, f, vp, vp, vp,
                                        ctypes.POINTER(vp), vp, vp, sz, vp]
        L.ispa_select_layers.argtypes = [ctypes.POINTER(ctypes.c_float), i, i, ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_ubyte)]
        L.ispa_rewarm_check.argtypes = [ctypes.POINTER(ctypes.c_float), i, i, ctypes.c_double, ctypes.c_double,
                                         ctypes.POINTER(ctypes.c_ubyte)]
        L.ispa_project.argtypes = [vp, i, i, vp, i, vp, i, vp]
        L.ispa_local_attn.argtypes = [ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ispa_workspace_bytes.argtypes = [ctypes.POINTER(AttnDesc), i, i]
        L.ispa_workspace_bytes.restype = ctypes.c_size_t
        L.ispa_device_status.argtypes = [vp]
        L.ispa_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp]
        L.ispa_selftest_exp2_poly.argtypes = [vp, vp, i, vp]
        L.ispa_kernel_launches.argtypes = []
        L.ispa_kernel_launches.restype = ctypes.c_ulonglong
        L.ispa_last_error.restype = ctypes.c_char_p
        L.ispa_version.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("ispa_workspace_bytes", "ispa_last_error", "ispa_version", "ispa_kernel_launches"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int, func: str) -> int:
    if rc != ISPA_OK:
        raise IspaError(rc, func, lib().ispa_last_error().decode())
    return rc


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return ISPA_BF16
    if t == torch.float32:
        return ISPA_FP32
    raise ValueError(f"unsupported dtype {t}")


def make_desc(n_q, n_kv, heads, head_dim, sink=(0, 0), chunk=(0, 0), scale=None, dtype=ISPA_BF16) -> AttnDesc:
    if scale is None:
        scale = head_dim ** -0.5
    return AttnDesc(n_q, n_kv, heads, head_dim, sink[0], sink[1], chunk[0], chunk[1], float(scale), int(dtype))


class Stats:
    """Device buffers of one layer's ridge statistics (G, C, H float32 [D, D], rows int64)."""

    def __init__(self, D: int, device="cuda"):
        self.D = D
        self.G = torch.zeros(D, D, dtype=torch.float32, device=device)
        self.C = torch.zeros(D, D, dtype=torch.float32, device=device)
        self.H = torch.zeros(D, D, dtype=torch.float32, device=device)
        self.rows = torch.zeros(1, dtype=torch.int64, device=device)

    def c(self) -> CStats:
        return CStats(self.D, self.G.data_ptr(), self.C.data_ptr(), self.H.data_ptr(), self.rows.data_ptr())


def workspace_bytes(desc: Optional[AttnDesc], n: int, D: int) -> int:
    return int(lib().ispa_workspace_bytes(ctypes.byref(desc) if desc is not None else None, n, D))


def ispa_attn_split(desc, q, k, v, o_full, lse_full, o_loc=None, lse_loc=None, o_hist=None, lse_hist=None,
                    stats: Optional[Stats] = None, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    cs = ctypes.byref(stats.c()) if stats is not None else None
    rc = lib().ispa_attn_split(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o_full), _p(lse_full), _p(o_loc),
                               _p(lse_loc), _p(o_hist), _p(lse_hist), cs, _p(ws),
                               0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "ispa_attn_split")


def ispa_quantize_q_i8(q: torch.Tensor, q8: torch.Tensor, q_scale: torch.Tensor, stream=None) -> None:
    """q [n, heads, 128] bf16 -> q8 int8 (same shape), q_scale [n, heads] float32."""
    n, heads, hd = q.shape
    _check(lib().ispa_quantize_q_i8(_p(q), n, heads, hd, _p(q8), _p(q_scale), _stream(stream)), "ispa_quantize_q_i8")


def ispa_k_blocks(desc) -> int:
    rc = lib().ispa_k_blocks(ctypes.byref(desc))
    if rc < 0:
        _check(rc, "ispa_k_blocks")
    return rc


def ispa_quantize_k_i8(desc, k: torch.Tensor, k8: torch.Tensor, k_scale: torch.Tensor, stream=None) -> None:
    """k [n_kv, heads, 128] bf16 -> k8 int8 (same shape), k_scale [heads, ispa_k_blocks(desc)] float32."""
    _check(lib().ispa_quantize_k_i8(ctypes.byref(desc), _p(k), _p(k8), _p(k_scale), _stream(stream)),
           "ispa_quantize_k_i8")


def ispa_attn_split_i8(desc, q8, q_scale, k8, k_scale, v, o_full, lse_full, o_loc=None, lse_loc=None, o_hist=None,
                       lse_hist=None, stats: Optional[Stats] = None, ws: Optional[torch.Tensor] = None,
                       stream=None) -> None:
    cs = ctypes.byref(stats.c()) if stats is not None else None
    rc = lib().ispa_attn_split_i8(ctypes.byref(desc), _p(q8), _p(q_scale), _p(k8), _p(k_scale), _p(v), _p(o_full),
                                  _p(lse_full), _p(o_loc), _p(lse_loc), _p(o_hist), _p(lse_hist), cs, _p(ws),
                                  0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "ispa_attn_split_i8")


def ispa_attn_split_ops(desc, q, k, v, o_full, lse_full, a_ops, r_ops, o_loc=None, lse_loc=None, o_hist=None,
                        lse_hist=None, stream=None) -> None:
    """ispa_attn_split writing the statistics operands [n_q, D] to a_ops / r_ops instead of
    accumulating them."""
    rc = lib().ispa_attn_split_ops(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o_full), _p(lse_full), _p(o_loc),
                                   _p(lse_loc), _p(o_hist), _p(lse_hist), _p(a_ops), _p(r_ops), _stream(stream))
    _check(rc, "ispa_attn_split_ops")


def ispa_accum_ops(stats: Sequence[Stats], a_ops, r_ops, n_rows: int, dtype: int, stream=None) -> None:
    """G += A^T A, C += A^T R, H += R^T R for len(stats) layers whose operands lie one after the
    other in a_ops / r_ops ([layers][n_rows][D])."""
    arr = (CStats * len(stats))(*[st.c() for st in stats])
    _check(lib().ispa_accum_ops(arr, len(stats), _p(a_ops), _p(r_ops), n_rows, dtype, _stream(stream)),
           "ispa_accum_ops")


def ispa_attn_split_noalloc(desc, q, k, v, o_full, lse_full, o_loc=None, lse_loc=None, o_hist=None,
                            lse_hist=None, stats: Stats = None, stream=None) -> None:
    """ispa_attn_split with fused statistics, using the library's static scratch (no workspace)."""
    cs = ctypes.byref(stats.c()) if stats is not None else None
    rc = lib().ispa_attn_split_noalloc(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o_full), _p(lse_full), _p(o_loc),
                                       _p(lse_loc), _p(o_hist), _p(lse_hist), cs, _stream(stream))
    _check(rc, "ispa_attn_split_noalloc")


def ispa_accum_stats(stats: Stats, a_loc, a_full, n_rows: int, dtype: int, ws=None, stream=None) -> None:
    rc = lib().ispa_accum_stats(ctypes.byref(stats.c()), _p(a_loc), _p(a_full), n_rows, dtype, _p(ws),
                                0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "ispa_accum_stats")


def ispa_stats_reset(stats: Stats, stream=None) -> None:
    _check(lib().ispa_stats_reset(ctypes.byref(stats.c()), _stream(stream)), "ispa_stats_reset")


def ispa_solve_absorb(stats: Sequence[Stats], w_o: Sequence[torch.Tensor], w_dtype: int, lam: float,
                      dW: torch.Tensor, eps: torch.Tensor, err_terms: Optional[torch.Tensor] = None,
                      w_new: Optional[Sequence[torch.Tensor]] = None, layer_status: torch.Tensor = None,
                      ws: Optional[torch.Tensor] = None, stream=None) -> None:
    L = len(stats)
    arr = (CStats * L)(*[s.c() for s in stats])
    wp = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_o])
    wn = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_new]) if w_new is not None else None
    rc = lib().ispa_solve_absorb(arr, L, wp, w_dtype, float(lam), _p(dW), _p(eps), _p(err_terms), wn,
                                 _p(layer_status), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                 _stream(stream))
    _check(rc, "ispa_solve_absorb")


def ispa_absorb_error(stats: Sequence[Stats], w_o: Sequence[torch.Tensor], w_dtype: int,
                      dW: Sequence[torch.Tensor], eps: torch.Tensor, err_terms: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None, stream=None) -> None:
    L = len(stats)
    arr = (CStats * L)(*[s.c() for s in stats])
    wp = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_o])
    dp = (ctypes.c_void_p * L)(*[d.data_ptr() for d in dW])
    rc = lib().ispa_absorb_error(arr, L, wp, w_dtype, dp, _p(eps), _p(err_terms), _p(ws),
                                 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "ispa_absorb_error")


def ispa_quantize_w8(w: torch.Tensor, w_dtype: int, wq_t: torch.Tensor, w_scale: torch.Tensor, stream=None) -> None:
    d_in, d_out = w.shape
    rc = lib().ispa_quantize_w8(_p(w), w_dtype, d_in, d_out, _p(wq_t), _p(w_scale), _stream(stream))
    _check(rc, "ispa_quantize_w8")


def ispa_project_w8a8(a: torch.Tensor, wq_t: torch.Tensor, w_scale: torch.Tensor, y: torch.Tensor,
                      ws: Optional[torch.Tensor] = None, stream=None) -> None:
    n = a.shape[0]
    d_in = a.numel() // max(1, n)
    d_out = wq_t.shape[0]
    rc = lib().ispa_project_w8a8(_p(a), n, d_in, _p(wq_t), _p(w_scale), d_out, _p(y), _p(ws),
                                 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "ispa_project_w8a8")


def ispa_select_layers(eps: Sequence[float], K: int):
    """Host-side selection; returns (idx list, is_local list)."""
    L = len(eps)
    e = (ctypes.c_float * L)(*[float(x) for x in eps])
    k = max(0, min(K, L))
    idx = (ctypes.c_int * max(1, k))()
    flags = (ctypes.c_ubyte * max(1, L))()
    _check(lib().ispa_select_layers(e, L, K, idx, flags), "ispa_select_layers")
    return [idx[i] for i in range(k)], [flags[i] for i in range(L)]


def ispa_rewarm_check(history: Sequence[Sequence[float]], ratio: float, min_rise: float):
    """The trigger's decision on a [chunks][layers] history of live errors (NaN = not monitored);
    returns the fired flags per layer."""
    n_chunks = len(history)
    n_layers = len(history[0]) if n_chunks else 0
    flat = (ctypes.c_float * max(1, n_chunks * n_layers))(*[float(x) for row in history for x in row])
    fired = (ctypes.c_ubyte * max(1, n_layers))()
    rc = lib().ispa_rewarm_check(flat, n_chunks, n_layers, float(ratio), float(min_rise), fired)
    if rc < 0:
        _check(rc, "ispa_rewarm_check")
    return [fired[i] for i in range(n_layers)]


def ispa_local_attn(desc, q, k_loc, v_loc, o, lse=None, w_new=None, y=None, ws=None, stream=None) -> None:
    rc = lib().ispa_local_attn(ctypes.byref(desc), _p(q), _p(k_loc), _p(v_loc), _p(o), _p(lse), _p(w_new), _p(y),
                               _p(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check(rc, "ispa_local_attn")


def ispa_project(a: torch.Tensor, w: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """y = A W; a [n, d_in] (or [n, heads, head_dim]), w [d_in, d_out], y [n, d_out], one dtype."""
    n = a.shape[0]
    d_in, d_out = w.shape
    _check(lib().ispa_project(_p(a), n, d_in, _p(w), d_out, _p(y), dtype_code(a.dtype), _stream(stream)),
           "ispa_project")


def ispa_device_status(stream=None) -> int:
    return int(lib().ispa_device_status(_stream(stream)))


def ispa_selftest_exp2_poly(x: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    _check(lib().ispa_selftest_exp2_poly(_p(x), _p(y), x.numel(), _stream(stream)), "ispa_selftest_exp2_poly")


ISPA_ATTN_AUTO, ISPA_ATTN_SINGLE, ISPA_ATTN_PAIR, ISPA_ATTN_TWO_GROUP = 0, 1, 2, 3


def ispa_set_attn_kernel(choice: int) -> int:
    """Choose the bf16 head_dim-128 attention kernel; returns the previous choice."""
    rc = lib().ispa_set_attn_kernel(int(choice))
    if rc < 0:
        _check(rc, "ispa_set_attn_kernel")
    return rc


def ispa_kernel_launches() -> int:
    return int(lib().ispa_kernel_launches())


def ispa_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    _check(lib().ispa_selftest_bounded_wait(int(limit_us), _stream(stream)), "ispa_selftest_bounded_wait")


def alloc_workspace(nbytes: int, device="cuda") -> Optional[torch.Tensor]:
    """A 256-byte aligned byte buffer (torch's caching allocator returns 512-byte aligned blocks)."""
    if nbytes <= 0:
        return None
    t = torch.empty(nbytes, dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t
