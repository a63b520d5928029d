"""Independent numpy restatement of the fp64 oracle (cross-check of the C++ one).

The oracle proper is the plain C++ implementation in oracle/moe_oracle.cpp;
this module states the same definitions with numpy primitives (matmul,
stable sorts) so that tests can check the two implementations against each
other on random layers.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product path (the CUDA library and its binding) never imports,
calls or links it, and this module imports nothing from the product package.

It is the plain definition of what the layer computes, written as directly as
possible in float64 numpy: one function per step so that the CUDA path can be
checked stage by stage. Library primitives used as steps: ``@`` (matmul),
``np.argsort(kind="stable")`` and ``np.lexsort``. There is no blocking, fusion
or reordering beyond what each definition states.

Sources. The pages describe the layer only by its shape:

* rabbit README (ferrumox/rabbit), model table, row "MoE routing": softmax
  routing to 10 of 512 experts plus a gated shared expert; row "native
  quantization read": OCP MXFP4 routed experts, read byte for byte.
* rabbit README, phase breakdown: the "expert matmul" phase is the routed
  experts' matmuls, the part of a decode step this layer reproduces.
* "Ran Moonshot's 2.8T-parameter Kimi K3 on a GPU-less mini-PC" (wpnews),
  architecture paragraph: Stable LatentMoE, routed experts compute in a
  narrower latent width than the hidden size; 896 experts per layer in OCP MXFP4.

Everything else is a reading, stated beside the function that takes it:
the E2M1/E8M0 encodings and 32-element blocks follow the OCP Microscaling
Formats (MX) v1.0 specification, section 5 (MXFP4 = E2M1 elements, E8M0
shared scale, block size 32); the SwiGLU expert, the sigmoid shared-expert
gate, top-k renormalisation and the lowest-index tie-break are the plainest
readings of a softmax top-k router with a gated shared expert.

Pinned by tests/test_oracle_pins.py (values from the OCP definition, closed
forms, brute force on tiny inputs, a dense-FFN special case computed by torch,
and invariances).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "E2M1_MAGNITUDES", "e2m1_decode", "e8m0_decode", "mxfp4_dequant", "bf16_to_f64",
    "round_to_bf16_bits", "router_logits", "topk_route", "selection_weights", "permute",
    "mxfp4_quantize",
    "silu", "sigmoid", "expert_ffn", "shared_expert", "combine", "latent_down", "moe_layer",
]

# ---------------------------------------------------------------------------
# number formats (OCP MX v1.0, section 5.3: E2M1 element, E8M0 scale)
# ---------------------------------------------------------------------------

#: magnitude of an E2M1 code's low three bits (2 exponent bits, bias 1, and 1
#: mantissa bit; exponent field 0 is subnormal: 0 and 0.5). Bit 3 is the sign.
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_decode(codes) -> np.ndarray:
    """Value of 4-bit E2M1 codes (uint8 in 0..15); code 8 is -0."""
    c = np.asarray(codes, dtype=np.uint8) & np.uint8(0xF)
    mag = E2M1_MAGNITUDES[c & np.uint8(7)]
    return np.where((c & np.uint8(8)) != 0, -mag, mag)


def e8m0_decode(codes) -> np.ndarray:
    """Value of E8M0 scale codes: 2^(c - 127) for c in 0..254, NaN for 255."""
    c = np.asarray(codes, dtype=np.int64)
    return np.where(c == 255, np.nan, np.ldexp(1.0, c - 127))


def mxfp4_dequant(q, s) -> np.ndarray:
    """Dense float64 value of an MXFP4 matrix.

    q: [..., N, K/2] uint8, two E2M1 codes per byte; element 2j of a row is the
       LOW nibble of byte j, element 2j+1 the HIGH nibble (reading: the pages do
       not state the nibble order; this is the order of the OCP reference
       packing and of the C++ oracle and the CUDA kernels).
    s: [..., N, K/32] uint8 E8M0 codes, one per 32 consecutive elements of a row.
    """
    q = np.asarray(q, dtype=np.uint8)
    s = np.asarray(s, dtype=np.uint8)
    # value pair of every byte: (low-nibble element, high-nibble element)
    byte_vals = np.stack([e2m1_decode(np.arange(256) & 0xF), e2m1_decode(np.arange(256) >> 4)],
                         axis=-1)
    vals = byte_vals[q].reshape(*q.shape[:-1], q.shape[-1] // 16, 32)   # [..., N, K/32, 32]
    with np.errstate(invalid="ignore"):
        vals *= e8m0_decode(s)[..., None]
    return vals.reshape(*q.shape[:-1], q.shape[-1] * 2)


def bf16_to_f64(bits) -> np.ndarray:
    """Value of bf16 numbers given as uint16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_to_bf16_bits(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even); uint16 bits.

    bf16 keeps 8 significant bits, so the unit in the last place of a value in
    [2^(e-1), 2^e) is 2^(e-8) (never below 2^-133, the subnormal spacing).
    Dividing by that power of two is exact, ``np.rint`` rounds half to even,
    and the product is then exactly a bf16 value (or >= 2^128, i.e. inf)."""
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    ulp_exp = np.maximum(e - 8, -133)
    with np.errstate(over="ignore", invalid="ignore"):
        r = np.ldexp(np.rint(np.ldexp(v, -ulp_exp)), ulp_exp)
        f32 = r.astype(np.float32)
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# a1-a2: router (rabbit README, model table "MoE routing": softmax top-k)
# ---------------------------------------------------------------------------

def router_logits(x_bits, w_router_bits) -> np.ndarray:
    """logits[t, e] = sum_h x[t, h] * Wr[e, h], in float64 from the bf16 inputs."""
    return bf16_to_f64(x_bits) @ bf16_to_f64(w_router_bits).T


def topk_route(logits, k: int, near_tie: float = 1e-5):
    """Softmax top-k with renormalised weights.

    Selection: the k largest logits (ranking by logit equals ranking by softmax
    probability, which is monotone); equal logits are ordered by LOWER expert
    index first. Slots are in that order (descending logit).

    Weights: w[t, j] = p[t, idx[t, j]] / sum_j' p[t, idx[t, j']] with p the
    softmax over all E experts; the full denominator cancels, so this is
    exp(l_j - m) / sum_sel exp(l_i - m) with m the largest logit.

    near-tie flag: a token is flagged when its k-th and (k+1)-th largest
    logits differ by less than ``near_tie`` (the selected set then depends on
    rounding).

    Returns idx [T, k] int32, w [T, k] float64, flagged [T] bool.
    """
    logits = np.asarray(logits, dtype=np.float64)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    flagged = np.zeros(T, dtype=bool)
    experts = np.arange(E)
    for t in range(T):
        order = np.lexsort((experts, -logits[t]))      # primary: -logit, then index
        sel = order[:k]
        idx[t] = sel
        ex = np.exp(logits[t, sel] - logits[t, sel[0]])
        w[t] = ex / ex.sum()
        if k < E and logits[t, order[k - 1]] - logits[t, order[k]] < near_tie:
            flagged[t] = True
    return idx, w, flagged


def selection_weights(logits, idx):
    """Renormalised softmax weights of a GIVEN selection idx [T, k] (the weight
    rule of topk_route applied to another valid choice, e.g. the GPU's choice
    at a near-tie token): w[t, j] = exp(l_j - m) / sum_j' exp(l_j' - m), m the
    largest selected logit."""
    logits = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(logits, np.asarray(idx, dtype=np.int64), axis=1)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    return ex / ex.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# a3: permutation (token -> expert dispatch)
# ---------------------------------------------------------------------------

def permute(idx, E: int):
    """Group the T*k (token, slot) pairs by expert.

    counts[e]  number of pairs routed to expert e
    offsets    exclusive prefix sum of counts, E+1 entries
    rows       pairs sorted by expert, ascending token inside an expert
               (reading: the pages never describe the dispatch; "stable by
               token" is the plainest order). Each token has at most one slot
               per expert, so (expert, token) is a strict order.
    row_token[r], row_slot[r]   the pair placed at permuted row r
    slot_row[t, j]              the permuted row of pair (t, j)
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    order = np.argsort(flat, kind="stable")             # pair p = t*k + j
    row_token = (order // k).astype(np.int32)
    row_slot = (order % k).astype(np.int32)
    slot_row = np.empty(T * k, dtype=np.int32)
    slot_row[order] = np.arange(T * k, dtype=np.int32)
    return counts, offsets, row_token, row_slot, slot_row.reshape(T, k)


# ---------------------------------------------------------------------------
# a4: MXFP4 activation quantisation (prefill with MXFP4 activations)
# ---------------------------------------------------------------------------

def mxfp4_quantize(v):
    """OCP MX v1.0 conversion of float values to MXFP4, 32-element blocks.

    Per block: amax = max |v|; shared exponent X = floor(log2 amax) - 2 (2 is
    the largest E2M1 exponent), scale code 127 + X clamped to 0..254; each
    v / 2^X is rounded to the nearest E2M1 value, ties to the even code
    (0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4), magnitudes above
    6 saturate to 6. The sign bit is the sign bit of v (so a negative value
    that rounds to 0 gives code 8, negative zero). A block of zeros gets scale
    code 0 and codes 0. NaN inputs are not handled (not produced by the layer
    on finite inputs).

    v: [..., K] (K a multiple of 32). Returns (codes [..., K] uint8, scale codes
    [..., K/32] uint8).
    """
    v = np.asarray(v, dtype=np.float64)
    K = v.shape[-1]
    blk = v.reshape(*v.shape[:-1], K // 32, 32)
    amax = np.abs(blk).max(axis=-1)
    # floor(log2 amax) from the float exponent, exactly: amax = f * 2^e, f in [0.5, 1)
    _, e = np.frexp(np.where(amax > 0, amax, 1.0))
    X = np.where(amax > 0, (e - 1) - 2, -127).astype(np.int64)
    code_s = np.clip(127 + X, 0, 254)
    scaled = np.abs(blk) / np.ldexp(1.0, code_s - 127)[..., None]
    # nearest E2M1 magnitude with ties to the even code: compare against the
    # midpoints; at an exact midpoint pick the neighbour whose code is even.
    mags = E2M1_MAGNITUDES
    idx = np.searchsorted(mags, scaled, side="left").clip(0, 7)   # first mag >= scaled
    lo = (idx - 1).clip(0, 7)
    d_lo = scaled - mags[lo]
    d_hi = mags[idx] - scaled
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (idx % 2 == 0))
    code = np.where(scaled >= 6.0, 7, np.where(pick_hi, idx, lo))
    code = np.where(scaled <= 0.0, 0, code)
    sign = np.signbit(blk).astype(np.uint8) << np.uint8(3)
    codes = (code.astype(np.uint8) | sign).reshape(v.shape)
    return codes, code_s.astype(np.uint8)


def mxfp4_pack(codes) -> np.ndarray:
    """Pack element codes [..., K] into bytes [..., K/2] (low nibble = even element)."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def mxfp4_values(codes, scale_codes) -> np.ndarray:
    """Value of unpacked element codes [..., K] with their scale codes [..., K/32]."""
    with np.errstate(invalid="ignore"):
        return e2m1_decode(codes) * np.repeat(e8m0_decode(scale_codes), 32, axis=-1)


# ---------------------------------------------------------------------------
# a5-a7: routed expert SwiGLU FFN on MXFP4 weights
# ---------------------------------------------------------------------------

def silu(z):
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def sigmoid(z):
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def expert_ffn(x_rows, wg, wu, wd, act: str = "exact"):
    """One expert on its tokens: y = Wd (silu(Wg x) * (Wu x)).

    x_rows: [n, W] float64 activation rows routed to this expert.
    wg, wu: [I, W] and wd: [W, I] dense float64 (e.g. from mxfp4_dequant).
    act: where the activations are rounded before a matmul
      "exact"  no rounding (decode: bf16 x is exact, h stays unrounded)
      "mxfp4"  x and h are MXFP4-quantised per 32-block (prefill, MXFP4 acts)
    Returns (y [n, W], h [n, I]) with h as it entered the down projection.

    Reading: the expert activation is SwiGLU (silu(gate) * up), silu(z) =
    z / (1 + e^-z); the Kimi K3 page names its activation "SituAndMul" without
    defining it.
    """
    x = np.asarray(x_rows, dtype=np.float64)
    if act == "mxfp4":
        c, s = mxfp4_quantize(x)
        x = mxfp4_values(c, s)
    g = x @ wg.T
    u = x @ wu.T
    h = silu(g) * u
    if act == "mxfp4":
        c, s = mxfp4_quantize(h)
        h = mxfp4_values(c, s)
    return h @ wd.T, h


# ---------------------------------------------------------------------------
# a8: gated shared expert (rabbit README, model table row "MoE routing")
# ---------------------------------------------------------------------------

def shared_expert(x_bits, ws_gate_bits, ws_up_bits, ws_down_bits, w_sgate_bits):
    """s[t] = sigmoid(x[t] . w_sg) * Wsd (silu(Wsg x[t]) * (Wsu x[t])).

    Reading: the gate is one sigmoid scalar per token from a learned vector
    w_sg (the pages say only "gated shared expert"); the shared expert is a
    bf16 SwiGLU FFN of width I_shared that is always applied.
    Returns (s [T, H], gate [T])."""
    x = bf16_to_f64(x_bits)
    gate = sigmoid(x @ bf16_to_f64(w_sgate_bits))
    g = x @ bf16_to_f64(ws_gate_bits).T
    u = x @ bf16_to_f64(ws_up_bits).T
    h = silu(g) * u
    return gate[:, None] * (h @ bf16_to_f64(ws_down_bits).T), gate


# ---------------------------------------------------------------------------
# a9: combine
# ---------------------------------------------------------------------------

def combine(y_perm, slot_row, w, shared_out=None, w_lat_up_bits=None):
    """y[t] = sum_j w[t, j] * y_perm[slot_row[t, j]]  (+ latent up-projection) + s[t].

    With a latent up-projection W_lu [H, L] the weighted sum is formed at width
    L and mapped once: y[t] = W_lu (sum_j w y_perm) + s[t] (reading of the
    Kimi K3 page's latent-width routed experts)."""
    y_perm = np.asarray(y_perm, dtype=np.float64)
    T, k = slot_row.shape
    acc = np.zeros((T, y_perm.shape[1]), dtype=np.float64)
    for j in range(k):
        acc += w[:, j:j + 1] * y_perm[slot_row[:, j]]
    if w_lat_up_bits is not None:
        acc = acc @ bf16_to_f64(w_lat_up_bits).T
    if shared_out is not None:
        acc = acc + shared_out
    return acc


# ---------------------------------------------------------------------------
# a10: latent down-projection (Kimi K3 page: Stable LatentMoE)
# ---------------------------------------------------------------------------

def latent_down(x_bits, w_lat_down_bits):
    """x_lat = bf16( W_ld x ): the routed experts' input at latent width L.

    Reading: the projection is a dense bf16 matrix [L, H] and its result is
    rounded to bf16 (a defined rounding point, the same on both sides).
    Returns uint16 bf16 bits [T, L]."""
    return round_to_bf16_bits(bf16_to_f64(x_bits) @ bf16_to_f64(w_lat_down_bits).T)


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

def moe_layer(inp: dict, k: int, experts, act: str = "exact", idx_override=None,
              near_tie: float = 1e-5):
    """End-to-end layer.

    inp: x, w_router, ws_gate, ws_up, ws_down, w_sgate (uint16 bf16 bits) and,
         for latent layers, w_lat_down / w_lat_up.
    experts: callable e -> (wg_q, wg_s, wu_q, wu_s, wd_q, wd_s) in the
         canonical MXFP4 layout (or a dict with that mapping).
    idx_override: [T, k] expert selection to use instead of the oracle's own
         (for near-tie tokens, evaluated with the GPU's selection).
    Returns a dict of every intermediate: logits, idx, w, flagged, counts,
    offsets, row_token, row_slot, slot_row, x_lat, y_perm, h_perm, shared,
    gate, y.
    """
    get = experts if callable(experts) else experts.__getitem__
    x_bits = np.asarray(inp["x"], dtype=np.uint16)
    T = x_bits.shape[0]
    E = inp["w_router"].shape[0]
    logits = router_logits(x_bits, inp["w_router"])
    idx, w, flagged = topk_route(logits, k, near_tie)
    if idx_override is not None:
        idx = np.asarray(idx_override, dtype=np.int32)
        w = selection_weights(logits, idx)
    counts, offsets, row_token, row_slot, slot_row = permute(idx, E)
    latent = "w_lat_down" in inp
    if latent:
        x_lat_bits = latent_down(x_bits, inp["w_lat_down"])
        xin = bf16_to_f64(x_lat_bits)
    else:
        x_lat_bits = None
        xin = bf16_to_f64(x_bits)
    W = xin.shape[1]
    y_perm = np.zeros((T * k, W), dtype=np.float64)
    h_perm = None
    for e in np.nonzero(counts)[0]:
        r0, r1 = offsets[e], offsets[e + 1]
        wg_q, wg_s, wu_q, wu_s, wd_q, wd_s = get(int(e))
        y, h = expert_ffn(xin[row_token[r0:r1]], mxfp4_dequant(wg_q, wg_s),
                          mxfp4_dequant(wu_q, wu_s), mxfp4_dequant(wd_q, wd_s), act)
        if h_perm is None:
            h_perm = np.zeros((T * k, h.shape[1]), dtype=np.float64)
        y_perm[r0:r1] = y
        h_perm[r0:r1] = h
    shared, gate = shared_expert(x_bits, inp["ws_gate"], inp["ws_up"], inp["ws_down"],
                                 inp["w_sgate"])
    y = combine(y_perm, slot_row, w, shared, inp.get("w_lat_up") if latent else None)
    return dict(logits=logits, idx=idx, w=w, flagged=flagged, counts=counts, offsets=offsets,
                row_token=row_token, row_slot=row_slot, slot_row=slot_row, x_lat=x_lat_bits,
                y_perm=y_perm, h_perm=h_perm, shared=shared, gate=gate, y=y)
