"""Python binding of librtv (the C ABI in include/rtv.h).

Argument marshalling only: every step of the append/attend path runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  There is
no fallback: if ``librtv.so`` is missing or fails to load, importing this
module raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# RTV_LIBRARY=debug selects the bounds-checking debug build (librtv_debug.so)
LIB_PATH = os.path.join(HERE, "librtv_debug.so" if os.environ.get("RTV_LIBRARY") == "debug"
                        else "librtv.so")

RTV_OK = 0
RTV_ERR_INVALID_ARG = 1
RTV_ERR_OOM = 2
RTV_ERR_CUDA = 3
RTV_ERR_STATE = 4
RTV_ERR_TIMEOUT = 5
RTV_ERR_UNSUPPORTED = 6
RTV_ERR_BOUNDS = 7
RTV_OUT_F32 = 0
RTV_OUT_BF16 = 1
RTV_MAX_SLOTS = 64
RTV_MAX_FRAMES_PER_CHUNK = 4


class rtv_cache_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("max_frames_per_chunk", ctypes.c_int), ("window_frames", ctypes.c_int),
                ("pinned_frames", ctypes.c_int), ("rope_t", ctypes.c_int),
                ("rope_h", ctypes.c_int), ("rope_w", ctypes.c_int),
                ("rope_base", ctypes.c_double)]


class rtv_cache_state(ctypes.Structure):
    _fields_ = [("frames_committed", ctypes.c_longlong),
                ("generated_committed", ctypes.c_longlong),
                ("pinned_committed", ctypes.c_int), ("head", ctypes.c_int),
                ("n_slots", ctypes.c_int), ("n_visible", ctypes.c_int),
                ("visible_slots", ctypes.c_int * RTV_MAX_SLOTS),
                ("visible_frames", ctypes.c_longlong * RTV_MAX_SLOTS),
                ("frame_of_slot", ctypes.c_longlong * RTV_MAX_SLOTS),
                ("staged_layers", ctypes.c_int), ("staged_frames", ctypes.c_int),
                ("last_attend_splits", ctypes.c_int)]


class rtv_layer_layout(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_size_t), ("v_codes", ctypes.c_size_t),
                ("k_scales", ctypes.c_size_t), ("v_scales", ctypes.c_size_t),
                ("q_codes", ctypes.c_size_t), ("q_scales", ctypes.c_size_t),
                ("v_scale_max", ctypes.c_size_t), ("scale_pitch", ctypes.c_int),
                ("q_scale_pitch", ctypes.c_int)]


_P = ctypes.c_void_p
_S = ctypes.c_int
_SIGS = {
    "rtv_status_string": (ctypes.c_char_p, [_S]),
    "rtv_cache_required_bytes": (_S, [ctypes.POINTER(rtv_cache_config), ctypes.POINTER(ctypes.c_size_t)]),
    "rtv_cache_layer_layout": (_S, [ctypes.POINTER(rtv_cache_config), _S, ctypes.POINTER(rtv_layer_layout)]),
    "rtv_cache_create": (_S, [ctypes.POINTER(rtv_cache_config), _P, ctypes.c_size_t, ctypes.POINTER(_P)]),
    "rtv_cache_destroy": (_S, [_P]),
    "rtv_cache_append": (_S, [_P, _S, _P, _P, _P, _S, _P]),
    "rtv_attend": (_S, [_P, _S, _P, _S, _P]),
    "rtv_cache_append_project": (_S, [_P, _S, _P, _P, _P, _P, _S, _S, _P]),
    "rtv_attend_static_scratch": (_S, [_P, _S, _P, _S, _P]),
    "rtv_split_plan": (_S, [_S, _S, _S, ctypes.POINTER(_S), ctypes.POINTER(_S)]),
    "rtv_cache_advance": (_S, [_P]),
    "rtv_cache_get_state": (_S, [_P, ctypes.POINTER(rtv_cache_state)]),
    "rtv_cache_device_buffer": (_S, [_P, ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_size_t)]),
    "rtv_cache_export": (_S, [_P, _S, _S, _P, _P, _P, _P, _P, _P, _P]),
    "rtv_poll_error": (_S, [_P]),
    "rtv_debug_set_wait_fault": (_S, [_P, _S, ctypes.c_longlong]),
    "rtv_debug_build": (_S, []),
    "rtv_debug_corrupt_next_attend": (_S, [_P, _S]),
    "rtv_step_graph_create": (_S, [_P, _S, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P),
                                   ctypes.POINTER(_P), _S, _P, ctypes.POINTER(_P)]),
    "rtv_step_graph_launch": (_S, [_P, _P]),
    "rtv_step_graph_destroy": (_S, [_P]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} not built ({LIB_PATH}); run "
                          "`python -m kv_cache_serving_append_b200.build [--debug]`")
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


class RtvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def status_string(status: int) -> str:
    return lib.rtv_status_string(status).decode()


def check(status: int, what: str) -> None:
    if status != RTV_OK:
        raise RtvError(status, what)


def make_config(cfg: dict) -> rtv_cache_config:
    return rtv_cache_config(cfg["n_layers"], cfg["n_heads"], cfg["head_dim"], cfg["grid_h"],
                            cfg["grid_w"], cfg["max_frames_per_chunk"], cfg["window_frames"],
                            cfg["pinned_frames"], cfg["rope_t"], cfg["rope_h"], cfg["rope_w"],
                            float(cfg.get("rope_base", 10000.0)))


def split_plan(n_units: int, n_kv_tiles: int, sm_count: int):
    """(n_split, tiles_per_split) that rtv_attend uses for this problem."""
    a, b = _S(), _S()
    check(lib.rtv_split_plan(n_units, n_kv_tiles, sm_count, ctypes.byref(a), ctypes.byref(b)), "rtv_split_plan")
    return a.value, b.value


def required_bytes(cfg: dict) -> int:
    c = make_config(cfg)
    n = ctypes.c_size_t()
    check(lib.rtv_cache_required_bytes(ctypes.byref(c), ctypes.byref(n)), "rtv_cache_required_bytes")
    return n.value


def layer_layout(cfg: dict, layer: int) -> rtv_layer_layout:
    c = make_config(cfg)
    out = rtv_layer_layout()
    check(lib.rtv_cache_layer_layout(ctypes.byref(c), layer, ctypes.byref(out)),
          "rtv_cache_layer_layout")
    return out


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


class Cache:
    """A cache whose device buffer is a torch uint8 tensor owned by this object."""

    def __init__(self, cfg: dict, device=None):
        import torch
        self.cfg = dict(cfg)
        self.device = torch.device(device or "cuda")
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.nbytes = required_bytes(cfg)
        self.buffer = torch.empty(self.nbytes, dtype=torch.uint8, device=self.device)
        self._c = make_config(cfg)
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            check(lib.rtv_cache_create(ctypes.byref(self._c), _ptr(self.buffer), self.nbytes,
                                       ctypes.byref(h)), "rtv_cache_create")
        self.handle = h
        self.T = cfg["grid_h"] * cfg["grid_w"]
        self._staged = {}          # layer -> frames staged since the last advance

    def close(self):
        if self.handle:
            check(lib.rtv_cache_destroy(self.handle), "rtv_cache_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- argument checks (the C ABI sees bare pointers and cannot check sizes)
    def tensor_status(self, t, numel: int, dtypes) -> int:
        """RTV_OK if ``t`` is a contiguous tensor of one of ``dtypes`` with
        ``numel`` elements on this cache's device, else RTV_ERR_INVALID_ARG.
        A tensor that fails here never reaches the library: a short, strided
        or foreign-device buffer would make a kernel read or write outside it."""
        try:
            ok = (t.dtype in dtypes and t.is_contiguous() and t.device == self.device
                  and t.numel() == numel)
        except AttributeError:
            ok = False
        return RTV_OK if ok else RTV_ERR_INVALID_ARG

    def _rows(self, n_frames: int) -> int:
        return n_frames * self.T * self.cfg["n_heads"] * self.cfg["head_dim"]

    # -- the hot path ----------------------------------------------------
    def append(self, layer: int, q, k, v, n_frames: int, stream=None) -> int:
        import torch
        if not isinstance(n_frames, int) or not 1 <= n_frames <= self.cfg["max_frames_per_chunk"]:
            return RTV_ERR_INVALID_ARG
        for t in (q, k, v):
            st = self.tensor_status(t, self._rows(n_frames), (torch.bfloat16,))
            if st != RTV_OK:
                return st
        st = lib.rtv_cache_append(self.handle, layer, _ptr(q), _ptr(k), _ptr(v), n_frames,
                                  _stream_ptr(stream))
        if st == RTV_OK:
            self._staged[layer] = n_frames
        return st

    def append_project(self, layer: int, x_codes, x_scales, w_codes, w_scales, n_frames: int,
                       stream=None) -> int:
        """Fused QKV projection (FP8 GEMM) + append: x_codes uint8 [n_frames*T, hidden],
        x_scales fp32 [n_frames*T], w_codes uint8 [3*H*D, hidden], w_scales fp32 [3*H*D]."""
        import torch
        if not isinstance(n_frames, int) or not 1 <= n_frames <= self.cfg["max_frames_per_chunk"]:
            return RTV_ERR_INVALID_ARG
        rows = n_frames * self.T
        feats = 3 * self.cfg["n_heads"] * self.cfg["head_dim"]
        if getattr(x_codes, "dim", lambda: 0)() != 2 or x_codes.shape[0] != rows:
            return RTV_ERR_INVALID_ARG
        hidden = x_codes.shape[1]
        for t, n, dt in ((x_codes, rows * hidden, torch.uint8), (x_scales, rows, torch.float32),
                         (w_codes, feats * hidden, torch.uint8), (w_scales, feats, torch.float32)):
            st = self.tensor_status(t, n, (dt,))
            if st != RTV_OK:
                return st
        st = lib.rtv_cache_append_project(self.handle, layer, _ptr(x_codes), _ptr(x_scales), _ptr(w_codes),
                                          _ptr(w_scales), hidden, n_frames, _stream_ptr(stream))
        if st == RTV_OK:
            self._staged[layer] = n_frames
        return st

    def _out_status(self, layer: int, out) -> tuple[int, int]:
        import torch
        n = self._staged.get(layer, 0)
        if n == 0:
            return RTV_OK, RTV_OUT_F32      # the library reports RTV_ERR_STATE (or a bad layer)
        st = self.tensor_status(out, self._rows(n), (torch.float32, torch.bfloat16))
        return st, (RTV_OUT_BF16 if getattr(out, "dtype", None) == torch.bfloat16 else RTV_OUT_F32)

    def attend(self, layer: int, out, stream=None) -> int:
        st, dt = self._out_status(layer, out)
        if st != RTV_OK:
            return st
        return lib.rtv_attend(self.handle, layer, _ptr(out), dt, _stream_ptr(stream))

    def attend_static_scratch(self, layer: int, out, stream=None) -> int:
        """rtv_attend with the split partials in the library's fixed device array."""
        st, dt = self._out_status(layer, out)
        if st != RTV_OK:
            return st
        return lib.rtv_attend_static_scratch(self.handle, layer, _ptr(out), dt, _stream_ptr(stream))

    def advance(self) -> int:
        st = lib.rtv_cache_advance(self.handle)
        if st == RTV_OK:
            self._staged.clear()
        return st

    # -- inspection ------------------------------------------------------
    def state(self) -> rtv_cache_state:
        st = rtv_cache_state()
        check(lib.rtv_cache_get_state(self.handle, ctypes.byref(st)), "rtv_cache_get_state")
        return st

    def export(self, layer: int, slot: int, stream=None) -> dict:
        """Host copies (numpy) of one slot's K/V codes and scales and of the
        layer's Q workspace, through rtv_cache_export."""
        import numpy as np
        H, D, T = self.cfg["n_heads"], self.cfg["head_dim"], self.T
        qr = self.cfg["max_frames_per_chunk"] * T
        out = dict(k_codes=np.empty((H, T, D), np.uint8), v_codes=np.empty((H, T, D), np.uint8),
                   k_scales=np.empty((H, T), np.float32), v_scales=np.empty((H, T), np.float32),
                   q_codes=np.empty((H, qr, D), np.uint8), q_scales=np.empty((H, qr), np.float32))
        a = lambda x: x.ctypes.data_as(ctypes.c_void_p)   # noqa: E731
        check(lib.rtv_cache_export(self.handle, layer, slot, a(out["k_codes"]), a(out["v_codes"]),
                                   a(out["k_scales"]), a(out["v_scales"]), a(out["q_codes"]),
                                   a(out["q_scales"]), _stream_ptr(stream)), "rtv_cache_export")
        return out

    def poll_error(self) -> int:
        return lib.rtv_poll_error(self.handle)

    def set_wait_fault(self, enable: bool, limit_cycles: int = 0) -> int:
        return lib.rtv_debug_set_wait_fault(self.handle, int(enable), limit_cycles)

    def views(self, layer: int) -> dict:
        """torch views of one layer's tensors inside the device buffer."""
        import torch
        L = layer_layout(self.cfg, layer)
        cfg = self.cfg
        H, D, T = cfg["n_heads"], cfg["head_dim"], self.T
        S = cfg["pinned_frames"] + cfg["window_frames"] + cfg["max_frames_per_chunk"]
        qr = cfg["max_frames_per_chunk"] * T
        b = self.buffer

        def sl(off, n, dtype):
            return b[off:off + n * torch.empty((), dtype=dtype).element_size()].view(dtype)

        return dict(
            k_codes=sl(L.k_codes, S * H * T * D, torch.uint8).view(S, H, T, D),
            v_codes=sl(L.v_codes, S * H * T * D, torch.uint8).view(S, H, T, D),
            k_scales=sl(L.k_scales, S * H * L.scale_pitch, torch.float32).view(S, H, L.scale_pitch)[..., :T],
            v_scales=sl(L.v_scales, S * H * L.scale_pitch, torch.float32).view(S, H, L.scale_pitch)[..., :T],
            q_codes=sl(L.q_codes, H * qr * D, torch.uint8).view(H, qr, D),
            q_scales=sl(L.q_scales, H * L.q_scale_pitch, torch.float32).view(H, L.q_scale_pitch)[:, :qr],
            v_scale_max=sl(L.v_scale_max, S * H, torch.int64).view(S, H),
        )


class StepGraph:
    """One captured steady-state step of every layer (append + attend each,
    then the device-side ring advance), replayed by :meth:`launch`.  The
    graph reads the given per-layer input tensors and writes the per-layer
    output tensors each time it runs; they stay owned by this object."""

    def __init__(self, cache: Cache, n_frames: int, qs, ks, vs, outs, stream):
        import torch
        L = cache.cfg["n_layers"]
        if not all(len(x) == L for x in (qs, ks, vs, outs)):
            raise RtvError(RTV_ERR_INVALID_ARG, "rtv_step_graph_create")
        for t in (*qs, *ks, *vs):
            check(cache.tensor_status(t, cache._rows(n_frames), (torch.bfloat16,)), "rtv_step_graph_create")
        for t in outs:
            check(cache.tensor_status(t, cache._rows(n_frames), (torch.float32, torch.bfloat16)),
                  "rtv_step_graph_create")
        if len({t.dtype for t in outs}) != 1:
            raise RtvError(RTV_ERR_INVALID_ARG, "rtv_step_graph_create")
        dt = RTV_OUT_BF16 if outs[0].dtype == torch.bfloat16 else RTV_OUT_F32
        arr = lambda ts: (_P * L)(*[t.data_ptr() for t in ts])   # noqa: E731
        self.cache, self.n_frames = cache, n_frames
        self.tensors = (list(qs), list(ks), list(vs), list(outs))
        h = _P()
        check(lib.rtv_step_graph_create(cache.handle, n_frames, arr(qs), arr(ks), arr(vs), arr(outs), dt,
                                        _stream_ptr(stream), ctypes.byref(h)), "rtv_step_graph_create")
        self.handle = h

    def launch(self, stream=None) -> int:
        return lib.rtv_step_graph_launch(self.handle, _stream_ptr(stream))

    def close(self):
        if self.handle:
            check(lib.rtv_step_graph_destroy(self.handle), "rtv_step_graph_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
