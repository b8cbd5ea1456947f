"""fp64 CPU oracle of the RTPurbo decode-step attention (ctypes wrapper around rtp_oracle.c).

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` import this package. The CUDA library never calls it and
shares no code with it.

Every function takes numpy arrays that hold the exact stored values: bf16 and fp16 tensors
are passed as their raw 16-bit patterns (``uint16``) and widened to fp64 inside the C code.
The passages each function follows are cited in ``rtp_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from . import build as _build

_LIB = None

MODE_HIST, MODE_EXACT, MODE_DENSE = 0, 1, 2

_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_u8p = ctypes.POINTER(ctypes.c_uint8)


class _LayerCfg(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("idx_dim", ctypes.c_int), ("num_bins", ctypes.c_int),
        ("max_ctx", ctypes.c_int64), ("window", ctypes.c_int64), ("sinks", ctypes.c_int64),
        ("idx_range", ctypes.c_double), ("idx_scale", ctypes.c_double),
        ("attn_scale", ctypes.c_double), ("top_p", ctypes.c_double),
        ("top_k", ctypes.c_int64),
    ]


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_bf16_to_f64.restype = ctypes.c_double
        L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_indexer_scores.argtypes = [_u16p, _u16p, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_double, _dp]
        L.orc_hist_topp.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, ctypes.c_double,
                                    ctypes.c_int, _ip, _dp, _dp, _ip, _i64p, _i64p]
        L.orc_exact_topp.argtypes = [_dp, ctypes.c_int64, ctypes.c_double, _i64p, _i64p]
        L.orc_indexer_project.argtypes = [_u16p, _u16p, _u16p, _u16p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp]
        L.orc_hist_topk.argtypes = [_dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                    ctypes.c_int, _ip, _i64p, _i64p, _ip, _i64p, _i64p]
        L.orc_exact_topk.argtypes = [_dp, ctypes.c_int64, ctypes.c_int64, _i64p, _i64p]
        L.orc_window_sink_set.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                          _i64p, _i64p]
        L.orc_prefill_rows.argtypes = [_u16p, _u16p, _u16p, ctypes.c_int64, _i64p,
                                       ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                       ctypes.c_int, _dp]
        L.orc_sparse_attention.argtypes = [_u16p, _u16p, _u16p, _i64p, ctypes.c_int64,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp]
        L.orc_decode_layer.argtypes = [ctypes.POINTER(_LayerCfg), ctypes.c_int, _u16p, _u16p,
                                       _u16p, _u16p, _u16p, _i64p, _u8p, _dp, _i64p,
                                       ctypes.c_int]
        L.orc_max_threads.restype = ctypes.c_int
        _LIB = L
    return _LIB


def _ptr(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16, f"expected raw 16-bit patterns, got {a.dtype}"
    return a


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def bf16_to_f64(bits: int) -> float:
    return lib().orc_bf16_to_f64(int(bits) & 0xFFFF)


def f16_to_f64(bits: int) -> float:
    return lib().orc_f16_to_f64(int(bits) & 0xFFFF)


def indexer_scores(q_idx, k_idx, scale: float = 0.25) -> np.ndarray:
    """s[n] = scale * q_idx . k_idx[n] in fp64; q_idx [r] and k_idx [N, r] fp16 bit patterns."""
    q = _u16(q_idx)
    k = _u16(k_idx)
    r = q.shape[-1]
    n = k.shape[0]
    assert k.shape == (n, r)
    s = np.empty(n, np.float64)
    _check(lib().orc_indexer_scores(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), n, r,
                                    scale, _ptr(s, ctypes.c_double)), "indexer_scores")
    return s


def indexer_project(q_pre, k_pre, w_q, w_k):
    """(q_idx, k_idx) fp64 [B, Hkv, r] from bf16 bits q_pre [B, Hq, D], k_pre [B, Hkv, D],
    w_q [Hkv, r, G*D], w_k [Hkv, r, D]."""
    q_pre, k_pre, w_q, w_k = _u16(q_pre), _u16(k_pre), _u16(w_q), _u16(w_k)
    B, Hq, D = q_pre.shape
    Hkv, r, GD = w_q.shape
    assert k_pre.shape == (B, Hkv, D) and w_k.shape == (Hkv, r, D) and GD == (Hq // Hkv) * D
    qi = np.empty((B, Hkv, r), np.float64)
    ki = np.empty((B, Hkv, r), np.float64)
    _check(lib().orc_indexer_project(_ptr(q_pre, ctypes.c_uint16), _ptr(k_pre, ctypes.c_uint16),
                                     _ptr(w_q, ctypes.c_uint16), _ptr(w_k, ctypes.c_uint16), B,
                                     Hq, Hkv, D, r, _ptr(qi, ctypes.c_double),
                                     _ptr(ki, ctypes.c_double)), "indexer_project")
    return qi, ki


@dataclass
class HistSelection:
    sel: np.ndarray      # ascending token positions with bin >= b*
    bstar: int
    bins: np.ndarray     # bin of every token
    mass: np.ndarray     # M_b
    suffix: np.ndarray   # C_b


def hist_topp(s, p: float, range_: float = 16.0, nbins: int = 256) -> HistSelection:
    s = np.ascontiguousarray(s, dtype=np.float64)
    n = s.shape[0]
    bins = np.empty(n, np.int32)
    mass = np.empty(nbins, np.float64)
    suffix = np.empty(nbins, np.float64)
    sel = np.empty(n, np.int64)
    bstar = ctypes.c_int()
    nsel = ctypes.c_int64()
    _check(lib().orc_hist_topp(_ptr(s, ctypes.c_double), n, float(p), float(range_), nbins,
                               _ptr(bins, ctypes.c_int), _ptr(mass, ctypes.c_double),
                               _ptr(suffix, ctypes.c_double), ctypes.byref(bstar),
                               _ptr(sel, ctypes.c_int64), ctypes.byref(nsel)), "hist_topp")
    return HistSelection(sel[: nsel.value].copy(), bstar.value, bins, mass, suffix)


def exact_topp(s, p: float) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float64)
    sel = np.empty(s.shape[0], np.int64)
    nsel = ctypes.c_int64()
    _check(lib().orc_exact_topp(_ptr(s, ctypes.c_double), s.shape[0], float(p),
                                _ptr(sel, ctypes.c_int64), ctypes.byref(nsel)), "exact_topp")
    return sel[: nsel.value].copy()


@dataclass
class HistTopK:
    sel: np.ndarray      # ascending token positions with bin >= b*
    bstar: int
    bins: np.ndarray     # bin of every token
    count: np.ndarray    # K_b, tokens per bin
    suffix: np.ndarray   # N_b, tokens in bins >= b


def hist_topk(s, k: int, range_: float = 16.0, nbins: int = 256) -> HistTopK:
    s = np.ascontiguousarray(s, dtype=np.float64)
    n = s.shape[0]
    bins = np.empty(n, np.int32)
    count = np.empty(nbins, np.int64)
    suffix = np.empty(nbins, np.int64)
    sel = np.empty(n, np.int64)
    bstar = ctypes.c_int()
    nsel = ctypes.c_int64()
    _check(lib().orc_hist_topk(_ptr(s, ctypes.c_double), n, int(k), float(range_), nbins,
                               _ptr(bins, ctypes.c_int), _ptr(count, ctypes.c_int64),
                               _ptr(suffix, ctypes.c_int64), ctypes.byref(bstar),
                               _ptr(sel, ctypes.c_int64), ctypes.byref(nsel)), "hist_topk")
    return HistTopK(sel[: nsel.value].copy(), bstar.value, bins, count, suffix)


def exact_topk(s, k: int) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.float64)
    sel = np.empty(s.shape[0], np.int64)
    nsel = ctypes.c_int64()
    _check(lib().orc_exact_topk(_ptr(s, ctypes.c_double), s.shape[0], int(k),
                                _ptr(sel, ctypes.c_int64), ctypes.byref(nsel)), "exact_topk")
    return sel[: nsel.value].copy()


def window_sink_set(n_tok: int, window: int = 8192, sinks: int = 4) -> np.ndarray:
    sel = np.empty(n_tok, np.int64)
    nsel = ctypes.c_int64()
    _check(lib().orc_window_sink_set(n_tok, window, sinks, _ptr(sel, ctypes.c_int64),
                                     ctypes.byref(nsel)), "window_sink_set")
    return sel[: nsel.value].copy()


def sparse_attention(q, k, v, idx, scale: float | None = None) -> np.ndarray:
    """o[g] = softmax_j(scale * q[g] . k[idx_j]) @ v[idx_j]; q [G, D], k/v [rows, D] bf16 bits."""
    q = _u16(q)
    k = _u16(k)
    v = _u16(v)
    G, D = q.shape
    assert k.shape[1] == D and v.shape[1] == D
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    assert idx.size > 0 and idx.min() >= 0 and idx.max() < min(k.shape[0], v.shape[0])
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o = np.empty((G, D), np.float64)
    _check(lib().orc_sparse_attention(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                                      _ptr(v, ctypes.c_uint16), _ptr(idx, ctypes.c_int64),
                                      idx.size, G, D, float(scale), _ptr(o, ctypes.c_double)),
           "sparse_attention")
    return o


def prefill_rows(q_rows, k, v, rows, dense: bool, window: int = 8192, sinks: int = 4,
                 scale: float | None = None, num_threads: int | None = None) -> np.ndarray:
    """Prefill attention of the prompt positions `rows` for one query head (fp64): row i
    attends over {0..i} (dense: a retrieval head) or {0..sinks-1} U {i+1-window..i} (a local
    head). q_rows [len(rows), D] holds those rows' queries; k, v [n_tok, D]; bf16 bits."""
    q = _u16(q_rows)
    k = _u16(k)
    v = _u16(v)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    n_rows, D = q.shape
    assert rows.shape == (n_rows,) and k.shape[1] == D and v.shape == k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    o = np.empty((n_rows, D), np.float64)
    _check(lib().orc_prefill_rows(_ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
                                  _ptr(v, ctypes.c_uint16), k.shape[0], _ptr(rows, ctypes.c_int64),
                                  n_rows, D, 1 if dense else 0, int(window), int(sinks),
                                  float(scale), int(num_threads or 0), _ptr(o, ctypes.c_double)),
           "prefill_rows")
    return o


def decode_layer(*, q, q_idx, k_cache, v_cache, k_idx, seq_lens, retrieval_mask, top_p: float,
                 top_k: int = 0,
                 mode: int = MODE_HIST, window: int = 8192, sinks: int = 4, num_bins: int = 256,
                 idx_range: float = 16.0, idx_scale: float = 0.25, attn_scale: float | None = None,
                 num_threads: int | None = None):
    """One layer over every (batch, KV head). Returns (out [B, Hq, D] fp64, n_sel [B, Hkv])."""
    q = _u16(q)
    k_cache = _u16(k_cache)
    v_cache = _u16(v_cache)
    B, Hq, D = q.shape
    _, Hkv, Nmax, _ = k_cache.shape
    assert v_cache.shape == k_cache.shape
    if q_idx is not None:
        q_idx = _u16(q_idx)
        k_idx = _u16(k_idx)
        R = q_idx.shape[-1]
        assert q_idx.shape == (B, Hkv, R) and k_idx.shape == (B, Hkv, Nmax, R)
    else:
        R = 16
    cfg = _LayerCfg(B, Hq, Hkv, D, R, num_bins, Nmax, window, sinks, float(idx_range),
                    float(idx_scale), float(1.0 / np.sqrt(D) if attn_scale is None else attn_scale),
                    float(top_p), int(top_k))
    seq = np.ascontiguousarray(seq_lens, dtype=np.int64)
    mask = np.ascontiguousarray(retrieval_mask, dtype=np.uint8)
    assert seq.shape == (B,) and mask.shape == (Hkv,)
    out = np.empty((B, Hq, D), np.float64)
    nsel = np.empty((B, Hkv), np.int64)
    nt = num_threads if num_threads else lib().orc_max_threads()
    null16 = ctypes.POINTER(ctypes.c_uint16)()
    _check(lib().orc_decode_layer(ctypes.byref(cfg), mode, _ptr(q, ctypes.c_uint16),
                                  _ptr(q_idx, ctypes.c_uint16) if q_idx is not None else null16,
                                  _ptr(k_cache, ctypes.c_uint16), _ptr(v_cache, ctypes.c_uint16),
                                  _ptr(k_idx, ctypes.c_uint16) if q_idx is not None else null16,
                                  _ptr(seq, ctypes.c_int64), _ptr(mask, ctypes.c_uint8),
                                  _ptr(out, ctypes.c_double), _ptr(nsel, ctypes.c_int64), nt),
           "decode_layer")
    return out, nsel


def max_threads() -> int:
    return lib().orc_max_threads()


__all__ = [
    "MODE_HIST", "MODE_EXACT", "MODE_DENSE", "bf16_to_f64", "f16_to_f64", "indexer_scores",
    "indexer_project", "hist_topp", "HistSelection", "exact_topp", "hist_topk", "HistTopK",
    "exact_topk",
    "window_sink_set", "sparse_attention",
    "decode_layer", "max_threads",
]
