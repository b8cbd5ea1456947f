"""Thin ctypes binding of librtp.so (the C-ABI declared in include/rtp.h).

Argument marshalling only: every step of the decode path runs in the library's CUDA kernels.
Tensors are torch tensors already on the device (PyTorch is used for device memory and
streams); their data pointers are handed to the C entry points unchanged. There is no CPU
fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librtp.so")

RTP_OK, RTP_ERR_INVALID_ARG, RTP_ERR_UNSUPPORTED, RTP_ERR_OOM, RTP_ERR_CUDA, \
    RTP_ERR_DEVICE_STATUS = range(6)
DEV_BAD_SEQLEN, DEV_WAIT_TIMEOUT, DEV_BAD_INDEX = 0x1, 0x2, 0x4

# every entry point include/rtp.h declares
EXPORTS = ("rtp_config_default", "rtp_workspace_bytes", "rtp_create", "rtp_destroy",
           "rtp_decode_step", "rtp_dense_decode", "rtp_decode_step_host", "rtp_get_selection",
           "rtp_get_threshold", "rtp_get_device_status", "rtp_status_string", "rtp_last_error",
           "rtp_profile_enable", "rtp_profile_read", "rtp_window_attention_noalloc",
           "rtp_indexer_append", "rtp_selftest_wait_timeout", "rtp_nvtx_enable",
           "rtp_profile_launches", "rtp_prefill")
NOALLOC_MAX_HEADS = 64
KERNEL_CLASSES = ("select", "attend", "merge", "fused")


class RtpError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: status {status} ({msg})")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [
        ("num_layers", ctypes.c_int), ("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("idx_dim", ctypes.c_int),
        ("max_ctx", ctypes.c_int), ("window", ctypes.c_int), ("sinks", ctypes.c_int),
        ("num_bins", ctypes.c_int), ("idx_range", ctypes.c_float),
        ("idx_scale", ctypes.c_float), ("attn_scale", ctypes.c_float),
    ]


class NoAllocParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("max_ctx", ctypes.c_int), ("window", ctypes.c_int), ("sinks", ctypes.c_int),
        ("attn_scale", ctypes.c_float), ("dense", ctypes.c_int),
    ]


class IndexerIO(ctypes.Structure):
    _fields_ = [
        ("q_pre", ctypes.c_void_p), ("k_pre", ctypes.c_void_p), ("w_q", ctypes.c_void_p),
        ("w_k", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("head_mask", ctypes.POINTER(ctypes.c_uint8)), ("q_idx", ctypes.c_void_p),
        ("k_idx", ctypes.c_void_p),
    ]


class PrefillIO(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p), ("retrieval_mask", ctypes.POINTER(ctypes.c_uint8)),
        ("out", ctypes.c_void_p), ("t_max", ctypes.c_int32), ("dense", ctypes.c_int32),
    ]


class LayerIO(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("q_idx", ctypes.c_void_p), ("k_cache", ctypes.c_void_p),
        ("v_cache", ctypes.c_void_p), ("k_idx", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
        ("retrieval_mask", ctypes.POINTER(ctypes.c_uint8)), ("top_p", ctypes.c_float),
        ("out", ctypes.c_void_p), ("sel_count", ctypes.c_void_p), ("top_k", ctypes.c_int32),
        ("inputs_ready", ctypes.c_int32), ("single_launch", ctypes.c_int32),
    ]


_lib = None


def load(path: str = LIB_PATH):
    """Load librtp.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"librtp.so not built at {path}; run head_wise_sparse_retrieval_b200/"
                           "build.py (or __graft_entry__.build())")
    L = ctypes.CDLL(path)
    vp, i, f, u8p = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.POINTER(ctypes.c_uint8)
    L.rtp_config_default.argtypes = [ctypes.POINTER(Config), i, i, i, i, i]
    L.rtp_config_default.restype = None
    L.rtp_workspace_bytes.argtypes = [ctypes.POINTER(Config)]
    L.rtp_workspace_bytes.restype = ctypes.c_size_t
    L.rtp_create.argtypes = [ctypes.POINTER(Config), i, ctypes.POINTER(vp)]
    L.rtp_destroy.argtypes = [vp]
    L.rtp_decode_step.argtypes = [vp, i, ctypes.POINTER(LayerIO), vp]
    L.rtp_dense_decode.argtypes = [vp, ctypes.POINTER(LayerIO), vp]
    L.rtp_decode_step_host.argtypes = [vp, i, vp, vp, vp, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                       ctypes.POINTER(vp), u8p, f, vp, vp]
    L.rtp_get_selection.argtypes = [vp, i, i, ctypes.POINTER(ctypes.c_int32), ctypes.c_int64,
                                    ctypes.POINTER(ctypes.c_int64)]
    L.rtp_get_threshold.argtypes = [vp, i, i, ctypes.POINTER(ctypes.c_int),
                                    ctypes.POINTER(ctypes.c_float)]
    L.rtp_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    L.rtp_profile_enable.argtypes = [vp, i]
    L.rtp_nvtx_enable.argtypes = [vp, i]
    L.rtp_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_int64)]
    L.rtp_profile_launches.argtypes = [vp, ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_int32), ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_int64)]
    L.rtp_window_attention_noalloc.argtypes = [ctypes.POINTER(NoAllocParams), vp, vp, vp, vp,
                                               vp, vp]
    L.rtp_window_attention_noalloc.restype = ctypes.c_int
    L.rtp_indexer_append.argtypes = [vp, ctypes.POINTER(IndexerIO), vp]
    L.rtp_indexer_append.restype = ctypes.c_int
    L.rtp_prefill.argtypes = [vp, ctypes.POINTER(PrefillIO), vp]
    L.rtp_prefill.restype = ctypes.c_int
    L.rtp_selftest_wait_timeout.argtypes = [vp, i, ctypes.POINTER(LayerIO), ctypes.c_uint64, vp]
    L.rtp_selftest_wait_timeout.restype = ctypes.c_int
    L.rtp_status_string.argtypes = [i]
    L.rtp_status_string.restype = ctypes.c_char_p
    L.rtp_last_error.argtypes = []
    L.rtp_last_error.restype = ctypes.c_char_p
    for name in ("rtp_create", "rtp_destroy", "rtp_decode_step", "rtp_dense_decode",
                 "rtp_decode_step_host", "rtp_get_selection", "rtp_get_threshold",
                 "rtp_get_device_status", "rtp_profile_enable", "rtp_profile_read"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(st: int, where: str):
    if st != RTP_OK:
        msg = load().rtp_last_error().decode()
        raise RtpError(st, where, msg or load().rtp_status_string(st).decode())


def default_config(num_layers: int, batch: int, num_q_heads: int, num_kv_heads: int,
                   max_ctx: int, **overrides) -> Config:
    c = Config()
    load().rtp_config_default(ctypes.byref(c), num_layers, batch, num_q_heads, num_kv_heads,
                              max_ctx)
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def workspace_bytes(cfg: Config) -> int:
    return int(load().rtp_workspace_bytes(ctypes.byref(cfg)))


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return int(getattr(stream, "cuda_stream", stream)) or None


@dataclass
class Layer:
    """Device tensors of one layer (see include/rtp.h for layouts)."""
    q: object
    q_idx: object
    k_cache: object
    v_cache: object
    k_idx: object
    seq_lens: object


class Handle:
    """An rtp_handle: workspace for one configuration on one device."""

    def __init__(self, cfg: Config, device: int = 0):
        self.cfg = cfg
        self._h = ctypes.c_void_p()
        _check(load().rtp_create(ctypes.byref(cfg), device, ctypes.byref(self._h)), "rtp_create")
        self._mask_keep = []

    def close(self):
        if self._h:
            _check(load().rtp_destroy(self._h), "rtp_destroy")
            self._h = ctypes.c_void_p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _io(self, layer: Layer, mask, top_p: float, out, sel_count=None, top_k: int = 0,
            inputs_ready: bool = False, single_launch: bool = False) -> LayerIO:
        m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
        assert m.shape == (self.cfg.num_kv_heads,)
        io = LayerIO(_ptr(layer.q), _ptr(layer.q_idx), _ptr(layer.k_cache), _ptr(layer.v_cache),
                     _ptr(layer.k_idx), _ptr(layer.seq_lens),
                     m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), float(top_p), _ptr(out),
                     _ptr(sel_count), int(top_k), 1 if inputs_ready else 0,
                     1 if single_launch else 0)
        io._mask = m  # keep the host mask alive for the duration of the call
        return io

    def decode_step(self, layer_idx: int, layer: Layer, mask, top_p: float, out,
                    sel_count=None, stream=None, top_k: int = 0, inputs_ready: bool = False,
                    single_launch: bool = False):
        """rtp_decode_step: enqueue one layer on `stream` (default: torch's current stream).
        top_k > 0 selects by fixed top-k through the histogram instead of top-p;
        inputs_ready, single_launch: see rtp_layer_io."""
        io = self._io(layer, mask, top_p, out, sel_count, top_k, inputs_ready, single_launch)
        _check(load().rtp_decode_step(self._h, layer_idx, ctypes.byref(io), _stream_ptr(stream)),
               "rtp_decode_step")

    def dense_decode(self, layer: Layer, out, stream=None):
        io = self._io(layer, np.zeros(self.cfg.num_kv_heads, np.uint8), 1.0, out)
        _check(load().rtp_dense_decode(self._h, ctypes.byref(io), _stream_ptr(stream)),
               "rtp_dense_decode")

    def decode_step_host(self, q_host, q_idx_host, seq_lens_host, layers: list[Layer], masks,
                         top_p: float, out_host, stream=None):
        """rtp_decode_step_host: host queries in, host outputs out, device caches in between."""
        L = len(layers)
        arr = ctypes.c_void_p * L
        kc = arr(*[_ptr(x.k_cache) for x in layers])
        vc = arr(*[_ptr(x.v_cache) for x in layers])
        ki = arr(*[_ptr(x.k_idx) for x in layers])
        m = np.ascontiguousarray(np.asarray(masks, dtype=np.uint8))
        _check(load().rtp_decode_step_host(
            self._h, L, _ptr(q_host), _ptr(q_idx_host), _ptr(seq_lens_host), kc, vc, ki,
            m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), float(top_p), _ptr(out_host),
            _stream_ptr(stream)), "rtp_decode_step_host")

    def indexer_append(self, q_pre, k_pre, w_q, w_k, seq_lens, q_idx, k_idx, head_mask=None,
                       stream=None):
        """rtp_indexer_append: q_idx and the new k_idx row from the pre-RoPE q / k."""
        m = None
        mp = ctypes.POINTER(ctypes.c_uint8)()
        if head_mask is not None:
            m = np.ascontiguousarray(np.asarray(head_mask, dtype=np.uint8))
            assert m.shape == (self.cfg.num_kv_heads,)
            mp = m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
        io = IndexerIO(_ptr(q_pre), _ptr(k_pre), _ptr(w_q), _ptr(w_k), _ptr(seq_lens), mp,
                       _ptr(q_idx), _ptr(k_idx))
        _check(load().rtp_indexer_append(self._h, ctypes.byref(io), _stream_ptr(stream)),
               "rtp_indexer_append")

    def prefill(self, q, k_cache, v_cache, seq_lens, mask, out, dense: bool = False,
                stream=None):
        """rtp_prefill: q [B, Hq, t_max, 128] bf16 -> out [B, Hq, t_max, 128] fp32 (rows below
        each prompt length), over caches whose rows 0 .. T_b - 1 hold the prompt."""
        m = np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
        assert m.shape == (self.cfg.num_kv_heads,)
        io = PrefillIO(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                       m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), _ptr(out),
                       int(q.shape[2]), 1 if dense else 0)
        _check(load().rtp_prefill(self._h, ctypes.byref(io), _stream_ptr(stream)), "rtp_prefill")

    def selftest_wait_timeout(self, layer_idx: int, layer: Layer, mask, top_p: float, out,
                              wait_ns: int, stream=None):
        """rtp_selftest_wait_timeout: the layer's selection with one barrier arrival withheld."""
        io = self._io(layer, mask, top_p, out)
        _check(load().rtp_selftest_wait_timeout(self._h, layer_idx, ctypes.byref(io),
                                                int(wait_ns), _stream_ptr(stream)),
               "rtp_selftest_wait_timeout")

    def selection(self, b: int, kvh: int) -> np.ndarray:
        """Ascending positions selected for (b, kvh) by the last decode_step."""
        cnt = ctypes.c_int64()
        _check(load().rtp_get_selection(self._h, b, kvh, None, 0, ctypes.byref(cnt)),
               "rtp_get_selection")
        buf = np.empty(max(int(cnt.value), 1), np.int32)
        _check(load().rtp_get_selection(self._h, b, kvh,
                                        buf.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                        buf.size, ctypes.byref(cnt)), "rtp_get_selection")
        return buf[: cnt.value].copy()

    def threshold(self, b: int, kvh: int) -> tuple[int, float]:
        bs = ctypes.c_int()
        sm = ctypes.c_float()
        _check(load().rtp_get_threshold(self._h, b, kvh, ctypes.byref(bs), ctypes.byref(sm)),
               "rtp_get_threshold")
        return bs.value, sm.value

    def profile(self, enable: bool):
        _check(load().rtp_profile_enable(self._h, int(bool(enable))), "rtp_profile_enable")

    def nvtx(self, enable: bool):
        """rtp_nvtx_enable: one NVTX range per call around its launches (off by default)."""
        _check(load().rtp_nvtx_enable(self._h, int(bool(enable))), "rtp_nvtx_enable")

    def profile_read(self) -> dict:
        """{class: (total ms, launches)} for the launches recorded since the last read."""
        ms = (ctypes.c_double * 4)()
        n = (ctypes.c_int64 * 4)()
        _check(load().rtp_profile_read(self._h, ms, n), "rtp_profile_read")
        return {k: (ms[i], int(n[i])) for i, k in enumerate(KERNEL_CLASSES)}

    def profile_launches(self, cap: int = 1024) -> list:
        """[(class, ms)] of the launches recorded since the last read, in launch order."""
        ms = (ctypes.c_double * cap)()
        kind = (ctypes.c_int32 * cap)()
        n = ctypes.c_int64()
        _check(load().rtp_profile_launches(self._h, ms, kind, cap, ctypes.byref(n)),
               "rtp_profile_launches")
        return [(KERNEL_CLASSES[kind[i]], ms[i]) for i in range(n.value)]

    def device_status(self) -> int:
        code = ctypes.c_uint32()
        st = load().rtp_get_device_status(self._h, ctypes.byref(code))
        if st not in (RTP_OK, RTP_ERR_DEVICE_STATUS):
            _check(st, "rtp_get_device_status")
        return int(code.value)


def window_attention_noalloc(q, k_cache, v_cache, seq_lens, out, *, window: int = 8192,
                             sinks: int = 4, attn_scale: float | None = None, dense: bool = False,
                             stream=None):
    """rtp_window_attention_noalloc: window + sink (or dense) attention for every KV head,
    without a handle and without allocating: for callers that cannot call cudaMalloc. Shapes
    are read from the tensors: q [B, Hq, 128], caches [B, Hkv, max_ctx, 128]."""
    B, Hq, D = q.shape
    _, Hkv, Nmax, _ = k_cache.shape
    p = NoAllocParams(B, Hq, Hkv, Nmax, window, sinks,
                      float(attn_scale if attn_scale is not None else D ** -0.5), int(dense))
    _check(load().rtp_window_attention_noalloc(ctypes.byref(p), _ptr(q), _ptr(k_cache),
                                               _ptr(v_cache), _ptr(seq_lens), _ptr(out),
                                               _stream_ptr(stream)),
           "rtp_window_attention_noalloc")


def config_for(plan, **overrides) -> Config:
    """The library configuration matching a workloads.Plan."""
    c = default_config(plan.num_layers, plan.batch, plan.num_q_heads, plan.num_kv_heads,
                       plan.max_ctx)
    c.window = plan.window
    c.sinks = plan.sinks
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def layer_from(li) -> Layer:
    """A Layer view of workloads.LayerInputs."""
    return Layer(li.q, li.q_idx, li.k_cache, li.v_cache, li.k_idx, li.seq_lens)
