"""Seeded synthetic inputs for the routed MXFP4 MoE layer.

This module only draws numbers: it holds none of the layer's arithmetic (no
decoding, routing, FFN or combine). Both the CUDA path (through the binding)
and the fp64 oracle consume what it produces, so that parity is checked on the
same bytes.

Recipe (the pages print no numeric example, so the value distributions are the
ones the workload descriptions state):

* activations ``x``                ~ N(0, 1), rounded to bf16 (RNE)
* router, shared-expert, shared-gate and latent weights ~ N(0, 0.02), bf16
* routed MXFP4 weights: element codes uniform over the 16 E2M1 codes (so each
  packed byte is uniform over 0..255) and E8M0 scale codes uniform over
  120..127 (block scales 2^-7 .. 2^0)
* router-variant workloads: a per-expert fp32 selection bias ~ N(0, bias_std)
* skewed routing (small-batch decode and prefill workloads): each skewed token
  receives a set S_t of k distinct experts drawn without replacement with
  probability proportional to rank^-1.1 (Zipf 1.1 over a seeded ranking), and
  x_t += 8 * sum_{e in S_t} Wr[e] / |Wr[e]|^2, which lifts those router logits
  by about 8 (router logit std is about 1.8). Decode-32 skews 60% of the
  tokens over a hot set of 64 experts; prefill skews every token over all E.

Every stream is a numpy PCG64 generator keyed by ``SeedSequence([seed,
stream, index])`` so any single expert matrix can be regenerated on its own.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class MoeWorkload:
    name: str
    T: int          # tokens
    H: int          # hidden width
    I: int          # routed-expert intermediate width
    E: int          # routed experts
    k: int          # experts per token
    I_shared: int   # shared-expert intermediate width
    L: int = 0      # latent width (0: routed experts run at width H)
    skew: str = "none"   # "none" | "hot64" | "zipf"
    seed: int = 1000
    # router variant (default: softmax top-k): score function 0 softmax /
    # 1 sigmoid, expert groups and groups kept, weight scale, and the standard
    # deviation of a seeded per-expert selection bias (0: none)
    score_fn: int = 0
    n_group: int = 0
    topk_group: int = 0
    route_scale: float = 1.0
    bias_std: float = 0.0

    @property
    def W(self) -> int:
        """Width the routed experts compute in (L for latent layers, else H)."""
        return self.L if self.L else self.H


WORKLOADS = {
    "tiny": MoeWorkload("tiny", T=4, H=256, I=128, E=16, k=2, I_shared=128, seed=1000),
    "decode1": MoeWorkload("decode1", T=1, H=8192, I=2048, E=512, k=10, I_shared=2048, seed=1001),
    "decode32": MoeWorkload("decode32", T=32, H=8192, I=2048, E=512, k=10, I_shared=2048,
                            skew="hot64", seed=1002),
    "prefill4096": MoeWorkload("prefill4096", T=4096, H=8192, I=2048, E=512, k=10,
                               I_shared=2048, skew="zipf", seed=1003),
    "latent16": MoeWorkload("latent16", T=16, H=7168, I=1024, E=896, k=8, I_shared=2048,
                            L=2048, seed=1004),
}

# stream ids
_S_X, _S_ROUTER, _S_SG, _S_SU, _S_SD, _S_SGATE, _S_LD, _S_LU = 1, 2, 3, 4, 5, 6, 7, 8
_S_SKEW = 9
_S_BIAS = 10
_S_WG, _S_WU, _S_WD = 20, 21, 22


def _rng(seed: int, stream: int, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, index])))


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even); returns uint16 bits."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(seed, stream, shape, std, index=0) -> np.ndarray:
    v = _rng(seed, stream, index).standard_normal(shape, dtype=np.float32) * np.float32(std)
    return f32_to_bf16_bits(v)


# ---------------------------------------------------------------------------
# routed MXFP4 expert weights
# ---------------------------------------------------------------------------

def expert_matrix(seed: int, which: str, e: int, N: int, K: int):
    """MXFP4 matrix [N, K] of expert ``e``: (q [N, K/2] uint8, s [N, K/32] uint8).

    ``which`` is "gate", "up" or "down"."""
    stream = {"gate": _S_WG, "up": _S_WU, "down": _S_WD}[which]
    rng = _rng(seed, stream, e)
    q = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    s = rng.integers(120, 128, (N, K // 32), dtype=np.uint8)
    return q, s


def expert_shapes(w: MoeWorkload):
    """(N, K) of the gate/up and down matrices of one routed expert."""
    return (w.I, w.W), (w.W, w.I)


def expert_weights(w: MoeWorkload, experts, threads: int | None = None):
    """Stacked weights for the listed experts (in that order).

    Returns dict with wg_q, wg_s, wu_q, wu_s, wd_q, wd_s, each [len(experts), ...]."""
    experts = list(experts)
    (Ng, Kg), (Nd, Kd) = expert_shapes(w)
    n = len(experts)
    out = {
        "wg_q": np.empty((n, Ng, Kg // 2), np.uint8), "wg_s": np.empty((n, Ng, Kg // 32), np.uint8),
        "wu_q": np.empty((n, Ng, Kg // 2), np.uint8), "wu_s": np.empty((n, Ng, Kg // 32), np.uint8),
        "wd_q": np.empty((n, Nd, Kd // 2), np.uint8), "wd_s": np.empty((n, Nd, Kd // 32), np.uint8),
    }

    def fill(j):
        e = experts[j]
        out["wg_q"][j], out["wg_s"][j] = expert_matrix(w.seed, "gate", e, Ng, Kg)
        out["wu_q"][j], out["wu_s"][j] = expert_matrix(w.seed, "up", e, Ng, Kg)
        out["wd_q"][j], out["wd_s"][j] = expert_matrix(w.seed, "down", e, Nd, Kd)

    threads = threads or min(16, os.cpu_count() or 1)
    if n <= 2 or threads <= 1:
        for j in range(n):
            fill(j)
    else:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(n)))
    return out


# ---------------------------------------------------------------------------
# dense inputs
# ---------------------------------------------------------------------------

def dense_inputs(w: MoeWorkload) -> dict:
    """Activations and bf16 weights (uint16 bit arrays) of one workload."""
    s = w.seed
    d = {
        "w_router": _normal_bf16(s, _S_ROUTER, (w.E, w.H), 0.02),
        "ws_gate": _normal_bf16(s, _S_SG, (w.I_shared, w.H), 0.02),
        "ws_up": _normal_bf16(s, _S_SU, (w.I_shared, w.H), 0.02),
        "ws_down": _normal_bf16(s, _S_SD, (w.H, w.I_shared), 0.02),
        "w_sgate": _normal_bf16(s, _S_SGATE, (w.H,), 0.02),
    }
    if w.L:
        d["w_lat_down"] = _normal_bf16(s, _S_LD, (w.L, w.H), 0.02)
        d["w_lat_up"] = _normal_bf16(s, _S_LU, (w.H, w.L), 0.02)
    if w.bias_std > 0:
        d["e_bias"] = (_rng(s, _S_BIAS).standard_normal(w.E, dtype=np.float32)
                       * np.float32(w.bias_std))
    x = _rng(s, _S_X).standard_normal((w.T, w.H), dtype=np.float32)
    if w.skew != "none":
        x = x + _skew_boost(w, bf16_bits_to_f32(d["w_router"]))
    d["x"] = f32_to_bf16_bits(x)
    return d


def skew_sets(w: MoeWorkload):
    """Per-token preferred expert sets (list of arrays, empty for unskewed tokens)."""
    rng = _rng(w.seed, _S_SKEW)
    if w.skew == "hot64":
        pool = rng.permutation(w.E)[:64]
        p_skew = 0.6
    elif w.skew == "zipf":
        pool = rng.permutation(w.E)
        p_skew = 1.0
    else:
        return [np.zeros(0, np.int64)] * w.T
    ranks = np.arange(1, len(pool) + 1, dtype=np.float64)
    p = ranks ** -1.1
    p /= p.sum()
    sets = []
    for _ in range(w.T):
        if rng.random() < p_skew:
            sets.append(pool[rng.choice(len(pool), size=w.k, replace=False, p=p)])
        else:
            sets.append(np.zeros(0, np.int64))
    return sets


def _skew_boost(w: MoeWorkload, wr: np.ndarray) -> np.ndarray:
    boost = np.zeros((w.T, w.H), np.float32)
    norms2 = (wr.astype(np.float64) ** 2).sum(axis=1)
    for t, S in enumerate(skew_sets(w)):
        for e in S:
            boost[t] += (8.0 * wr[e] / norms2[e]).astype(np.float32)
    return boost


def workload_inputs(w: MoeWorkload, experts=None, threads=None) -> dict:
    """Dense inputs plus the routed weights of ``experts`` (default: all E)."""
    d = dense_inputs(w)
    d.update(expert_weights(w, range(w.E) if experts is None else experts, threads))
    return d


# ---------------------------------------------------------------------------
# device copies (plumbing only)
# ---------------------------------------------------------------------------

def to_device(w: MoeWorkload, dense: dict | None = None, device="cuda", chunk: int = 32,
              pinned: bool = False) -> dict:
    """Upload a workload's weights (all E experts) and x to the GPU as torch tensors.

    bf16 arrays become int16 tensors holding the bit patterns. Experts are
    generated and copied ``chunk`` at a time to bound host memory."""
    import torch

    dense = dense_inputs(w) if dense is None else dense
    out = {}
    for name, arr in dense.items():
        arr = np.ascontiguousarray(arr)
        t = torch.from_numpy(arr if arr.dtype == np.float32 else arr.view(np.int16))
        out[name] = t.to(device)
    (Ng, Kg), (Nd, Kd) = expert_shapes(w)
    shapes = {"wg_q": (Ng, Kg // 2), "wg_s": (Ng, Kg // 32), "wu_q": (Ng, Kg // 2),
              "wu_s": (Ng, Kg // 32), "wd_q": (Nd, Kd // 2), "wd_s": (Nd, Kd // 32)}
    for name, shp in shapes.items():
        out[name] = torch.empty((w.E,) + shp, dtype=torch.uint8, device=device)
    for e0 in range(0, w.E, chunk):
        ids = list(range(e0, min(w.E, e0 + chunk)))
        ex = expert_weights(w, ids)
        for name in shapes:
            src = torch.from_numpy(ex[name])
            if pinned:
                src = src.pin_memory()
            out[name][e0:e0 + len(ids)].copy_(src, non_blocking=pinned)
    if device != "cpu":
        torch.cuda.synchronize()
    return out
