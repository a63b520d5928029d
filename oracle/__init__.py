"""fp64 CPU oracle of the routed MXFP4 MoE layer: ctypes shim over the plain C++
implementation in oracle/moe_oracle.cpp (compiled to oracle/libmoe_oracle.so).

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline and --impl reference legs import this package; the product
package never does, and this package imports nothing from it. Every function
below only marshals numpy arrays to the C++ library and back: the arithmetic
of each step (a1 router ... a10 latent) is in moe_oracle.cpp, which cites the
passage it follows. ``oracle.moe_oracle_np`` is an independent numpy
restatement of the same definitions, kept as a cross-check of this one.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

__all__ = [
    "E2M1_MAGNITUDES", "TIE_SET", "TIE_ORDER", "TIE_GROUP", "SOFTMAX", "SIGMOID", "set_threads",
    "threads", "e2m1_decode", "e8m0_decode", "mxfp4_dequant", "mxfp4_values", "mxfp4_pack",
    "bf16_to_f64", "round_to_bf16_bits", "silu", "sigmoid", "mxfp4_quantize", "mxfp4_matmul",
    "bf16_matmul", "router_logits", "route", "topk_route", "selection_weights", "permute",
    "expert_ffn", "shared_expert", "combine", "latent_down", "moe_layer", "library_path",
]

TIE_SET, TIE_ORDER, TIE_GROUP = 1, 2, 4      # bits of the routing near-tie flags
SOFTMAX, SIGMOID = 0, 1                      # score functions of the router


def library_path() -> str:
    return _build.LIB


_lib = ctypes.CDLL(_build.build())

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_D = ctypes.c_double


def _sig(name, args, res=None):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_sig("moe_o_set_threads", [_I])
_sig("moe_o_threads", [], _I)
for _n in ("moe_o_e2m1_decode", "moe_o_e8m0_decode", "moe_o_bf16_decode", "moe_o_silu",
           "moe_o_sigmoid", "moe_o_mxfp4_pack"):
    _sig(_n, [_P, _I64, _P])
_sig("moe_o_round_bf16", [_P, _I64, _P])
_sig("moe_o_mxfp4_values", [_P, _P, _I64, _P])
_sig("moe_o_mxfp4_dequant", [_P, _P, _I64, _I64, _P])
_sig("moe_o_mxfp4_quantize", [_P, _I64, _I64, _P, _P])
_sig("moe_o_mxfp4_matmul", [_P, _P, _I64, _I64, _P, _I64, _P])
_sig("moe_o_bf16_matmul", [_P, _I64, _I64, _P, _I64, _P])
_sig("moe_o_router_logits", [_P, _P, _I, _I, _I, _P])
_sig("moe_o_route", [_P, _P, _I, _I, _I, _I, _I, _I, _D, _D, _P, _P, _P, _P], _I)
_sig("moe_o_permute", [_P, _I, _I, _I, _P, _P, _P, _P, _P], _I)
_sig("moe_o_expert_ffn", [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P], _I)
_sig("moe_o_shared_expert", [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P])
_sig("moe_o_combine", [_P, _I, _P, _P, _I, _I, _P, _P, _I, _P])
_sig("moe_o_latent_down", [_P, _I, _I, _P, _I, _P])


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "H", "I", "E", "k", "I_shared", "L", "act",
                                              "score_fn", "n_group", "topk_group")] + \
               [("route_scale", ctypes.c_double), ("near_tie", ctypes.c_double)]


class _Inputs(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("x", "w_router", "e_bias", "w_sgate", "ws_gate", "ws_up",
                                  "ws_down", "w_lat_down", "w_lat_up", "wg_q", "wg_s", "wu_q",
                                  "wu_s", "wd_q", "wd_s", "idx_override")]


class _Outputs(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("logits", "idx", "w", "flags", "counts", "offsets",
                                  "row_token", "row_slot", "slot_row", "x_lat", "y_perm",
                                  "h_perm", "shared", "gate", "y")]


_sig("moe_o_layer", [ctypes.POINTER(_Dims), ctypes.POINTER(_Inputs), ctypes.POINTER(_Outputs)],
     _I)


def _c(a, dtype):
    return np.asarray(a, dtype=dtype, order="C")


def _p(a):
    return None if a is None else a.ctypes.data


def set_threads(n: int) -> None:
    """Threads the oracle splits independent outputs over (0: all cores).
    Results do not depend on it: every sum runs in one thread in one order."""
    _lib.moe_o_set_threads(int(n))


def threads() -> int:
    return int(_lib.moe_o_threads())


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def _map(fn, a, in_dtype, out_dtype=np.float64):
    a = _c(a, in_dtype)
    out = np.empty(a.shape, out_dtype)
    fn(_p(a), a.size, _p(out))
    return out if out.ndim else out[()]


def e2m1_decode(codes):
    """Value of 4-bit E2M1 codes 0..15 (code 8 is -0)."""
    return _map(_lib.moe_o_e2m1_decode, np.asarray(codes) & 0xF, np.uint8)


def e8m0_decode(codes):
    """2^(c - 127) for E8M0 codes 0..254; NaN for 255."""
    c = np.asarray(codes)
    if np.any((c < 0) | (c > 255)):
        raise ValueError("E8M0 codes are 0..255")
    return _map(_lib.moe_o_e8m0_decode, c, np.uint8)


E2M1_MAGNITUDES = e2m1_decode(np.arange(8, dtype=np.uint8))


def bf16_to_f64(bits):
    return _map(_lib.moe_o_bf16_decode, bits, np.uint16)


def round_to_bf16_bits(v):
    """Nearest bf16 (ties to even), one rounding from float64; uint16 bits."""
    return _map(_lib.moe_o_round_bf16, v, np.float64, np.uint16)


def silu(z):
    return _map(_lib.moe_o_silu, z, np.float64)


def sigmoid(z):
    return _map(_lib.moe_o_sigmoid, z, np.float64)


def mxfp4_dequant(q, s):
    """Dense value [..., N, K] of MXFP4 matrices q [..., N, K/2], s [..., N, K/32]."""
    q = _c(q, np.uint8)
    s = _c(s, np.uint8)
    K = q.shape[-1] * 2
    rows = q.size // (K // 2) if K else 0
    out = np.empty(q.shape[:-1] + (K,), np.float64)
    _lib.moe_o_mxfp4_dequant(_p(q), _p(s), rows, K, _p(out))
    return out


def mxfp4_values(codes, scale_codes):
    """Values of unpacked element codes [..., K] with scale codes [..., K/32]."""
    c = _c(codes, np.uint8)
    s = _c(scale_codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    _lib.moe_o_mxfp4_values(_p(c), _p(s), c.size, _p(out))
    return out


def mxfp4_pack(codes):
    """Element codes [..., K] -> bytes [..., K/2], element 2j in the low nibble."""
    c = _c(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] // 2,), np.uint8)
    _lib.moe_o_mxfp4_pack(_p(c), c.size, _p(out))
    return out


def mxfp4_quantize(v):
    """OCP MX v1.0 conversion to MXFP4 along the last axis (a multiple of 32):
    (codes [..., K] uint8 unpacked, scale codes [..., K/32] uint8)."""
    v = _c(v, np.float64)
    K = v.shape[-1]
    rows = v.size // K if K else 0
    codes = np.empty(v.shape, np.uint8)
    scales = np.empty(v.shape[:-1] + (K // 32,), np.uint8)
    _lib.moe_o_mxfp4_quantize(_p(v), rows, K, _p(codes), _p(scales))
    return codes, scales


def mxfp4_matmul(q, s, x):
    """x @ W^T for an MXFP4 matrix W [N, K] (q [N, K/2], s [N, K/32]) and rows x [R, K]."""
    q = _c(q, np.uint8)
    s = _c(s, np.uint8)
    x = _c(np.atleast_2d(x), np.float64)
    N, K = q.shape[0], q.shape[1] * 2
    out = np.empty((x.shape[0], N), np.float64)
    _lib.moe_o_mxfp4_matmul(_p(q), _p(s), N, K, _p(x), x.shape[0], _p(out))
    return out


def bf16_matmul(w_bits, x):
    """x @ W^T for a bf16 matrix W [N, K] (uint16 bits) and float64 rows x [R, K]."""
    w = _c(w_bits, np.uint16)
    x = _c(np.atleast_2d(x), np.float64)
    N, K = w.shape
    out = np.empty((x.shape[0], N), np.float64)
    _lib.moe_o_bf16_matmul(_p(w), N, K, _p(x), x.shape[0], _p(out))
    return out


# ---------------------------------------------------------------------------
# a1-a3
# ---------------------------------------------------------------------------

def router_logits(x_bits, w_router_bits):
    x = _c(np.atleast_2d(x_bits), np.uint16)
    wr = _c(w_router_bits, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float64)
    _lib.moe_o_router_logits(_p(x), _p(wr), T, H, E, _p(out))
    return out


def route(logits, k, score_fn=SOFTMAX, bias=None, n_group=1, topk_group=1, scale=1.0,
          near_tie=1e-5, idx_in=None):
    """Top-k routing (a2) and its variants: returns idx [T, k] int32, w [T, k]
    float64 and the near-tie flags [T] uint8 (TIE_SET | TIE_ORDER | TIE_GROUP).
    With idx_in, w holds the weights of that given selection instead."""
    lg = _c(logits, np.float64)
    T, E = lg.shape
    b = None if bias is None else _c(bias, np.float64)
    ii = None if idx_in is None else _c(idx_in, np.int32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    flags = np.empty(T, np.uint8)
    st = _lib.moe_o_route(_p(lg), _p(b), T, E, k, score_fn, n_group, topk_group, scale,
                          near_tie, _p(ii), _p(idx), _p(w), _p(flags))
    if st:
        raise ValueError(f"routing configuration rejected (code {st})")
    return idx, w, flags


def topk_route(logits, k, near_tie=1e-5):
    """Softmax top-k: (idx, w, flagged) with flagged = the k-th and (k+1)-th
    logits closer than near_tie (the selected set depends on rounding)."""
    idx, w, flags = route(logits, k, near_tie=near_tie)
    return idx, w, (flags & TIE_SET) != 0


def selection_weights(logits, idx, score_fn=SOFTMAX, scale=1.0):
    """Weights of a GIVEN selection idx [T, k] under the router's weight rule."""
    idx = _c(idx, np.int32)
    return route(logits, idx.shape[1], score_fn=score_fn, scale=scale, idx_in=idx)[1]


def permute(idx, E):
    """(counts [E], offsets [E+1], row_token, row_slot [T*k], slot_row [T, k])."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    row_token = np.empty(T * k, np.int32)
    row_slot = np.empty(T * k, np.int32)
    slot_row = np.empty((T, k), np.int32)
    if _lib.moe_o_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(row_token),
                          _p(row_slot), _p(slot_row)):
        raise ValueError("expert index outside [0, E)")
    return counts, offsets, row_token, row_slot, slot_row


# ---------------------------------------------------------------------------
# a4-a10
# ---------------------------------------------------------------------------

_ACT = {"exact": 0, "mxfp4": 1}


def expert_ffn(x_rows, wg_q, wg_s, wu_q, wu_s, wd_q, wd_s, act="exact", h_raw=False):
    """One routed expert on its rows x [n, W]: (y [n, W], h [n, I] as it entered
    the down projection[, h before any rounding])."""
    x = _c(np.atleast_2d(x_rows), np.float64)
    n, W = x.shape
    arrs = [_c(a, np.uint8) for a in (wg_q, wg_s, wu_q, wu_s, wd_q, wd_s)]
    I = arrs[0].shape[0]
    y = np.empty((n, W), np.float64)
    h = np.empty((n, I), np.float64)
    hr = np.empty((n, I), np.float64) if h_raw else None
    if _lib.moe_o_expert_ffn(_p(x), n, W, I, *[_p(a) for a in arrs], _ACT[act], _p(y), _p(h),
                             _p(hr)):
        raise ValueError(act)
    return (y, h, hr) if h_raw else (y, h)


def shared_expert(x_bits, ws_gate_bits, ws_up_bits, ws_down_bits, w_sgate_bits):
    """(s [T, H], gate [T]) of the gated bf16 shared expert."""
    x = _c(np.atleast_2d(x_bits), np.uint16)
    T, H = x.shape
    g, u, dn, sg = (_c(a, np.uint16) for a in (ws_gate_bits, ws_up_bits, ws_down_bits,
                                               w_sgate_bits))
    s = np.empty((T, H), np.float64)
    gate = np.empty(T, np.float64)
    _lib.moe_o_shared_expert(_p(x), T, H, g.shape[0], _p(g), _p(u), _p(dn), _p(sg), _p(s),
                             _p(gate))
    return s, gate


def combine(y_perm, slot_row, w, shared_out=None, w_lat_up_bits=None):
    """y[t] = [W_lu] sum_j w[t, j] y_perm[slot_row[t, j]] + shared[t]."""
    yp = _c(y_perm, np.float64)
    sr = _c(slot_row, np.int32)
    wt = _c(w, np.float64)
    T, k = sr.shape
    W = yp.shape[1]
    sh = None if shared_out is None else _c(shared_out, np.float64)
    lu = None if w_lat_up_bits is None else _c(w_lat_up_bits, np.uint16)
    H = lu.shape[0] if lu is not None else W
    y = np.empty((T, H), np.float64)
    _lib.moe_o_combine(_p(yp), W, _p(sr), _p(wt), T, k, _p(sh), _p(lu), H, _p(y))
    return y


def latent_down(x_bits, w_lat_down_bits):
    """x_lat = bf16(W_ld x), uint16 bits [T, L]."""
    x = _c(np.atleast_2d(x_bits), np.uint16)
    wl = _c(w_lat_down_bits, np.uint16)
    T, H = x.shape
    L = wl.shape[0]
    out = np.empty((T, L), np.uint16)
    _lib.moe_o_latent_down(_p(x), T, H, _p(wl), L, _p(out))
    return out


def moe_layer(inp: dict, k: int, experts, act: str = "exact", idx_override=None,
              near_tie: float = 1e-5, score_fn: int = SOFTMAX, e_bias=None, n_group: int = 1,
              topk_group: int = 1, route_scale: float = 1.0):
    """The whole layer (moe_o_layer): router, top-k, permutation, [latent
    down-projection], routed experts, gated shared expert, combine.

    inp: x, w_router, ws_gate, ws_up, ws_down, w_sgate (uint16 bf16 bits) and,
         for latent layers, w_lat_down / w_lat_up.
    experts: callable e -> (wg_q, wg_s, wu_q, wu_s, wd_q, wd_s) in the canonical
         MXFP4 layout, or a mapping; only the selected experts are fetched.
    idx_override: [T, k] selection to use instead of the oracle's own (the
         GPU's choice at a near-tie token), with that selection's weights.
    Returns a dict of every intermediate (logits, idx, w, flagged (set near
    tie), flags, counts, offsets, row_token, row_slot, slot_row, x_lat,
    y_perm, h_perm, shared, gate, y)."""
    get = experts if callable(experts) else experts.__getitem__
    x = _c(np.atleast_2d(inp["x"]), np.uint16)
    wr = _c(inp["w_router"], np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    latent = "w_lat_down" in inp and inp["w_lat_down"] is not None
    L = inp["w_lat_down"].shape[0] if latent else 0
    W = L or H
    Is = inp["ws_gate"].shape[0]
    bias = None if e_bias is None else _c(e_bias, np.float64)
    # the selection decides which experts' weights are needed
    if idx_override is not None:
        sel = _c(idx_override, np.int32)
    else:
        sel = route(router_logits(x, wr), k, score_fn, bias, n_group, topk_group, route_scale,
                    near_tie)[0]
    keep = []
    tables = {n: (ctypes.c_void_p * E)() for n in ("wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s")}
    I = None
    for e in np.unique(sel):
        arrs = [_c(a, np.uint8) for a in get(int(e))]
        keep.append(arrs)
        I = arrs[0].shape[0]
        for n, a in zip(("wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s"), arrs):
            tables[n][int(e)] = a.ctypes.data
    dense = {n: _c(inp[n], np.uint16) for n in ("w_sgate", "ws_gate", "ws_up", "ws_down")}
    lat = {n: _c(inp[n], np.uint16) for n in ("w_lat_down", "w_lat_up")} if latent else {}
    out = dict(
        logits=np.empty((T, E)), idx=np.empty((T, k), np.int32), w=np.empty((T, k)),
        flags=np.empty(T, np.uint8), counts=np.empty(E, np.int32),
        offsets=np.empty(E + 1, np.int32), row_token=np.empty(T * k, np.int32),
        row_slot=np.empty(T * k, np.int32), slot_row=np.empty((T, k), np.int32),
        x_lat=np.empty((T, L), np.uint16) if latent else None,
        y_perm=np.zeros((T * k, W)), h_perm=np.zeros((T * k, I or 1)), shared=np.empty((T, H)),
        gate=np.empty(T), y=np.empty((T, H)))
    dims = _Dims(T, H, I or 0, E, k, Is, L, _ACT[act], score_fn, n_group, topk_group,
                 route_scale, near_tie)
    ins = _Inputs(x=_p(x), w_router=_p(wr), e_bias=_p(bias), w_sgate=_p(dense["w_sgate"]),
                  ws_gate=_p(dense["ws_gate"]), ws_up=_p(dense["ws_up"]),
                  ws_down=_p(dense["ws_down"]), w_lat_down=_p(lat.get("w_lat_down")),
                  w_lat_up=_p(lat.get("w_lat_up")),
                  idx_override=_p(sel) if idx_override is not None else None,
                  **{n: ctypes.cast(tables[n], _P) for n in tables})
    outs = _Outputs(**{n: _p(v) for n, v in out.items()})
    st = _lib.moe_o_layer(ctypes.byref(dims), ctypes.byref(ins), ctypes.byref(outs))
    if st:
        raise ValueError(f"moe_o_layer failed (code {st})")
    out["flagged"] = (out["flags"] & TIE_SET) != 0
    return out
