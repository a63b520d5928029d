"""Routed MXFP4 MoE FFN layer on B200 (sm_100a): Python binding of libmoe_mxfp4.so.

Thin ctypes marshalling over the C ABI in ``include/moe_mxfp4.h``: every
function here has the name of the C entry point it calls, takes torch tensors
(device memory) and passes their data pointers. All computation runs in the
library's CUDA kernels; there is no Python or CPU fallback. Importing the
package fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MoeError", "MoeDims", "MoeLayerArgs", "ACT_BF16", "ACT_MXFP4", "library_path",
    "moe_status_string", "moe_workspace_size", "moe_x_op_size", "moe_workspace_init",
    "moe_device_status", "moe_route", "moe_route_biased", "moe_route_noalloc", "moe_permute", "moe_expert_ffn", "moe_combine",
    "moe_latent_down", "moe_layer", "moe_mxf4_layout_of", "moe_tile_scales",
    "moe_selftest_bounded_wait", "STATUS_BAD_EXPERT", "STATUS_REPEATED_EXPERT",
    "STATUS_WAIT_TIMEOUT", "SCORE_SOFTMAX", "SCORE_SIGMOID", "MoeLayer", "ExpertCache",
    "moe_expert_cache_bytes",
]

# bits of the device status word (moe_device_status)
STATUS_BAD_EXPERT, STATUS_REPEATED_EXPERT, STATUS_WAIT_TIMEOUT = 1, 2, 4

ACT_BF16 = 0
ACT_MXFP4 = 1

_PKG = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.environ.get("MOE_MXFP4_LIB", os.path.join(_PKG, "libmoe_mxfp4.so"))


def _load():
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python mxfp4_routed_expert_04_b200/build.py` "
            "(there is no fallback implementation)")
    return ctypes.CDLL(path)


_lib = _load()


SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1


class MoeDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "H", "I", "E", "k", "I_shared", "L", "act_mode",
                                              "score_fn", "n_group", "topk_group")] + \
               [("route_scale", ctypes.c_float)]

    @classmethod
    def of(cls, w, act_mode: int = ACT_BF16) -> "MoeDims":
        """Dims of a workload (anything with T, H, I, E, k, I_shared, L and,
        optionally, the router variant: score_fn, n_group, topk_group,
        route_scale)."""
        return cls(w.T, w.H, w.I, w.E, w.k, w.I_shared, w.L, act_mode,
                   getattr(w, "score_fn", 0), getattr(w, "n_group", 0),
                   getattr(w, "topk_group", 0), getattr(w, "route_scale", 1.0))


_P = ctypes.c_void_p


class MoeLayerArgs(ctypes.Structure):
    _fields_ = [(n, _P) for n in (
        "x", "w_router", "wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s", "w_sgate",
        "ws_gate", "ws_up", "ws_down", "w_lat_down", "w_lat_up", "topk_idx", "topk_w",
        "counts", "offsets", "expert_list", "row_token", "row_slot", "slot_row", "x_lat", "x_op",
        "y_perm", "y", "e_bias")]


_lib.moe_status_string.restype = ctypes.c_char_p
_lib.moe_status_string.argtypes = [ctypes.c_int]
_lib.moe_last_error.restype = ctypes.c_char_p
_lib.moe_workspace_size.restype = ctypes.c_size_t
_lib.moe_workspace_size.argtypes = [ctypes.POINTER(MoeDims)]
_lib.moe_x_op_size.restype = ctypes.c_size_t
_lib.moe_x_op_size.argtypes = [ctypes.POINTER(MoeDims)]
_D = ctypes.POINTER(MoeDims)
_Z = ctypes.c_size_t
_sigs = {
    "moe_workspace_init": [_D, _P, _Z, _P],
    "moe_device_status": [_P, ctypes.POINTER(ctypes.c_int32), _P],
    "moe_route": [_D, _P, _P, _P, _P, _P, _P, _Z, _P],
    "moe_route_biased": [_D, _P, _P, _P, _P, _P, _P, _P, _Z, _P],
    "moe_route_noalloc": [_D, _P, _P, _P, _P, _P, _P],
    "moe_permute": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P],
    "moe_expert_ffn": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P],
    "moe_combine": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P],
    "moe_latent_down": [_D, _P, _P, _P, _P, _Z, _P],
    "moe_layer": [_D, ctypes.POINTER(MoeLayerArgs), _P, _Z, _P],
    "moe_mxf4_layout_of": [_D, ctypes.c_void_p],
    "moe_tile_scales": [_P, ctypes.c_int64, ctypes.c_int32, _P, _P],
    "moe_selftest_bounded_wait": [_P, _P, ctypes.c_int, ctypes.c_uint32, _P],
}
_sigs.update({
    "moe_expert_cache_create": [_D, ctypes.c_int32, _P, _Z, ctypes.POINTER(_P)],
    "moe_expert_cache_destroy": [_P],
    "moe_expert_cache_stats": [_P, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                               ctypes.POINTER(ctypes.c_int64)],
    "moe_expert_ffn_streamed": [_P, _D, _P, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _Z, _P],
})
for _n, _a in _sigs.items():
    getattr(_lib, _n).argtypes = _a
    getattr(_lib, _n).restype = ctypes.c_int
_lib.moe_expert_cache_bytes.restype = ctypes.c_size_t
_lib.moe_expert_cache_bytes.argtypes = [_D, ctypes.c_int32]


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{moe_status_string(status)} ({status}): {message}")
        self.status = status


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def _check(status: int):
    if status != 0:
        raise MoeError(status, _lib.moe_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def moe_workspace_size(dims: MoeDims) -> int:
    return _lib.moe_workspace_size(ctypes.byref(dims))


def moe_x_op_size(dims: MoeDims) -> int:
    return _lib.moe_x_op_size(ctypes.byref(dims))


class MoeMxf4Layout(ctypes.Structure):
    _fields_ = [("x_codes", ctypes.c_size_t), ("x_scales", ctypes.c_size_t),
                ("tiles", ctypes.c_size_t), ("tile_base", ctypes.c_size_t),
                ("n_tiles", ctypes.c_size_t), ("h_codes", ctypes.c_size_t),
                ("h_scales", ctypes.c_size_t), ("max_tiles", ctypes.c_int32),
                ("tile_rows", ctypes.c_int32)]


def moe_mxf4_layout_of(dims) -> MoeMxf4Layout:
    """Byte offsets of the MOE_ACT_MXFP4 operands inside x_op and the workspace."""
    out = MoeMxf4Layout()
    _check(_lib.moe_mxf4_layout_of(ctypes.byref(dims), ctypes.addressof(out)))
    return out


def moe_tile_scales(src, rows: int, K: int, dst, stream=None):
    """Canonical E8M0 scales [rows, K/32] -> the tiled layout of the tensor-core path."""
    _check(_lib.moe_tile_scales(_ptr(src), int(rows), int(K), _ptr(dst), _stream(stream)))


def moe_selftest_bounded_wait(status, src, deliver: bool, limit: int, stream=None):
    """One CTA waits (bounded, ``limit`` tries) for a stage that a bulk copy
    from ``src`` fills (deliver) or that nothing fills; a timeout ORs
    STATUS_WAIT_TIMEOUT into the device int32 ``status``."""
    _check(_lib.moe_selftest_bounded_wait(_ptr(status), _ptr(src), 1 if deliver else 0,
                                          int(limit), _stream(stream)))


def moe_workspace_init(dims, ws, stream=None):
    _check(_lib.moe_workspace_init(ctypes.byref(dims), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)))


def moe_device_status(ws, stream=None) -> int:
    """Device status word (0 = no data error); raises nothing for a flagged word."""
    out = ctypes.c_int32(0)
    st = _lib.moe_device_status(_ptr(ws), ctypes.byref(out), _stream(stream))
    if st not in (0, 6):
        _check(st)
    return out.value


def _nbytes(t):
    return t.numel() * t.element_size()


def moe_route(dims, x, w_router, topk_idx, topk_w, logits, ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(dims), _ptr(x), _ptr(w_router), _ptr(topk_idx),
                          _ptr(topk_w), _ptr(logits), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_route_biased(dims, x, w_router, e_bias, topk_idx, topk_w, logits, ws, stream=None):
    _check(_lib.moe_route_biased(ctypes.byref(dims), _ptr(x), _ptr(w_router), _ptr(e_bias),
                                 _ptr(topk_idx), _ptr(topk_w), _ptr(logits), _ptr(ws), _nbytes(ws),
                                 _stream(stream)))


def moe_route_noalloc(dims, x, w_router, topk_idx, topk_w, logits, stream=None):
    """moe_route without a workspace (partials in the library's static device array)."""
    _check(_lib.moe_route_noalloc(ctypes.byref(dims), _ptr(x), _ptr(w_router), _ptr(topk_idx),
                                  _ptr(topk_w), _ptr(logits), _stream(stream)))


def moe_permute(dims, topk_idx, x_in, counts, offsets, expert_list, row_token, row_slot, slot_row,
                x_op, ws, stream=None):
    _check(_lib.moe_permute(ctypes.byref(dims), _ptr(topk_idx), _ptr(x_in), _ptr(counts),
                            _ptr(offsets), _ptr(expert_list), _ptr(row_token), _ptr(row_slot),
                            _ptr(slot_row), _ptr(x_op), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_expert_ffn(dims, x_op, offsets, expert_list, row_token, wg_q, wg_s, wu_q, wu_s, wd_q, wd_s,
                   y_perm, ws, stream=None):
    _check(_lib.moe_expert_ffn(ctypes.byref(dims), _ptr(x_op), _ptr(offsets), _ptr(expert_list),
                               _ptr(row_token), _ptr(wg_q), _ptr(wg_s), _ptr(wu_q), _ptr(wu_s),
                               _ptr(wd_q), _ptr(wd_s), _ptr(y_perm), _ptr(ws), _nbytes(ws),
                               _stream(stream)))


def moe_combine(dims, y_perm, slot_row, topk_w, x, w_sgate, ws_gate, ws_up, ws_down, w_lat_up, y,
                ws, stream=None):
    _check(_lib.moe_combine(ctypes.byref(dims), _ptr(y_perm), _ptr(slot_row), _ptr(topk_w),
                            _ptr(x), _ptr(w_sgate), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down),
                            _ptr(w_lat_up), _ptr(y), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_latent_down(dims, x, w_lat_down, x_lat, ws, stream=None):
    _check(_lib.moe_latent_down(ctypes.byref(dims), _ptr(x), _ptr(w_lat_down), _ptr(x_lat),
                                _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_layer(dims, args: MoeLayerArgs, ws, stream=None):
    _check(_lib.moe_layer(ctypes.byref(dims), ctypes.byref(args), _ptr(ws), _nbytes(ws),
                          _stream(stream)))


def moe_expert_cache_bytes(dims, slots: int) -> int:
    return _lib.moe_expert_cache_bytes(ctypes.byref(dims), int(slots))


class ExpertCache:
    """An LRU cache of `slots` routed experts in device memory (one torch
    buffer) in front of experts kept in host memory (moe_expert_cache_*).

    host_experts: a sequence of E tuples (wg_q, wg_s, wu_q, wu_s, wd_q, wd_s)
    of host tensors (page-locked for asynchronous copies) in the canonical
    layout."""

    def __init__(self, dims: MoeDims, slots: int, host_experts, device="cuda"):
        self.dims = dims
        nbytes = moe_expert_cache_bytes(dims, slots)
        if nbytes == 0:
            raise MoeError(2, _lib.moe_last_error().decode())
        self.mem = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.mem.data_ptr()) % 256
        self._host = list(host_experts)         # keeps the host tensors alive
        ptrs = (ctypes.c_void_p * (6 * dims.E))()
        for e, arrs in enumerate(self._host):
            for a, t in enumerate(arrs):
                ptrs[6 * e + a] = t.data_ptr()
        self._ptrs = ptrs
        h = ctypes.c_void_p()
        _check(_lib.moe_expert_cache_create(ctypes.byref(dims), int(slots), self.mem.data_ptr() + off,
                                            nbytes, ctypes.byref(h)))
        self._h = h

    def ffn(self, active, x_op, offsets, row_token, y_perm, ws, stream=None):
        """moe_expert_ffn_streamed for the experts in `active` (host ints)."""
        act = (ctypes.c_int32 * max(1, len(active)))(*[int(e) for e in active])
        _check(_lib.moe_expert_ffn_streamed(self._h, ctypes.byref(self.dims), act, len(active),
                                            _ptr(x_op), _ptr(offsets), _ptr(row_token), self._ptrs,
                                            _ptr(y_perm), _ptr(ws), _nbytes(ws), _stream(stream)))

    def stats(self):
        h, m, b = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(_lib.moe_expert_cache_stats(self._h, ctypes.byref(h), ctypes.byref(m), ctypes.byref(b)))
        return {"hits": h.value, "misses": m.value, "bytes_copied": b.value}

    def close(self):
        if self._h:
            _lib.moe_expert_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------------------
# convenience: device buffers of one layer (allocation through torch only)
# ---------------------------------------------------------------------------

class MoeLayer:
    """Owns the device buffers of one layer shape and calls the C ABI on them.

    ``weights``: dict of device tensors (x excluded) named like the C ABI
    (w_router, wg_q, wg_s, wu_q, wu_s, wd_q, wd_s, w_sgate, ws_gate, ws_up,
    ws_down and, for latent layers, w_lat_down, w_lat_up; optionally e_bias,
    the router's fp32 selection bias [E]); bf16 tensors as
    int16/uint16 bit patterns or torch.bfloat16. Scales in the canonical
    layout; for ACT_MXFP4 the layer keeps tiled copies (moe_tile_scales) in
    ``self.w``, the weights every call uses.
    """

    def __init__(self, dims: MoeDims, weights: dict, device="cuda"):
        self.dims = dims
        d, T, k = dims, dims.T, dims.k
        W = d.L if d.L else d.H
        R = T * k
        self.w = dict(weights)
        if d.act_mode == ACT_MXFP4:
            for name, rows, K in (("wg_s", d.E * d.I, W), ("wu_s", d.E * d.I, W),
                                  ("wd_s", d.E * W, d.I)):
                tiled = torch.empty_like(weights[name])
                moe_tile_scales(weights[name], rows, K, tiled)
                self.w[name] = tiled
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        ws_bytes = moe_workspace_size(dims)
        if ws_bytes == 0:
            _check(1 if _lib.moe_last_error() else 2)
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        self.x_op = torch.empty(moe_x_op_size(dims), dtype=torch.uint8, device=dev)
        self.topk_idx = torch.empty(T, k, **i32)
        self.topk_w = torch.empty(T, k, **f32)
        self.logits = torch.empty(T, d.E, **f32)
        self.counts = torch.empty(d.E, **i32)
        self.offsets = torch.empty(d.E + 1, **i32)
        self.expert_list = torch.empty(d.E + 1, **i32)
        self.row_token = torch.empty(R, **i32)
        self.row_slot = torch.empty(R, **i32)
        self.slot_row = torch.empty(T, k, **i32)
        self.x_lat = torch.empty(T, d.L, dtype=torch.int16, device=dev) if d.L else None
        self.y_perm = torch.empty(R, W, **f32)
        self.y = torch.empty(T, d.H, **f32)
        moe_workspace_init(dims, self.ws)

    def layer_args(self, x) -> MoeLayerArgs:
        w = self.w
        g = lambda n: _ptr(w.get(n))
        return MoeLayerArgs(
            x=_ptr(x), w_router=g("w_router"), wg_q=g("wg_q"), wg_s=g("wg_s"), wu_q=g("wu_q"),
            wu_s=g("wu_s"), wd_q=g("wd_q"), wd_s=g("wd_s"), w_sgate=g("w_sgate"),
            ws_gate=g("ws_gate"), ws_up=g("ws_up"), ws_down=g("ws_down"),
            w_lat_down=g("w_lat_down"), w_lat_up=g("w_lat_up"), topk_idx=_ptr(self.topk_idx),
            topk_w=_ptr(self.topk_w), counts=_ptr(self.counts), offsets=_ptr(self.offsets),
            expert_list=_ptr(self.expert_list),
            row_token=_ptr(self.row_token), row_slot=_ptr(self.row_slot),
            slot_row=_ptr(self.slot_row), x_lat=_ptr(self.x_lat), x_op=_ptr(self.x_op),
            y_perm=_ptr(self.y_perm), y=_ptr(self.y), e_bias=g("e_bias"))

    def __call__(self, x, stream=None):
        """Whole layer (moe_layer); returns the fp32 output tensor [T, H]."""
        moe_layer(self.dims, self.layer_args(x), self.ws, stream)
        return self.y

    def stages(self, x, stream=None):
        """The same layer through the four step calls (route, [latent], permute,
        expert_ffn, combine); also fills self.logits."""
        d, w = self.dims, self.w
        moe_route_biased(d, x, w["w_router"], w.get("e_bias"), self.topk_idx, self.topk_w,
                         self.logits, self.ws, stream)
        xin = x
        if d.L:
            moe_latent_down(d, x, w["w_lat_down"], self.x_lat, self.ws, stream)
            xin = self.x_lat
        moe_permute(d, self.topk_idx, xin, self.counts, self.offsets, self.expert_list,
                    self.row_token, self.row_slot, self.slot_row, self.x_op, self.ws, stream)
        moe_expert_ffn(d, self.x_op, self.offsets, self.expert_list, self.row_token, w["wg_q"], w["wg_s"],
                       w["wu_q"], w["wu_s"], w["wd_q"], w["wd_s"], self.y_perm, self.ws, stream)
        moe_combine(d, self.y_perm, self.slot_row, self.topk_w, x, w["w_sgate"], w["ws_gate"],
                    w["ws_up"], w["ws_down"], w.get("w_lat_up"), self.y, self.ws, stream)
        return self.y
