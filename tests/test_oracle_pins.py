"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a value the OCP MX definition fixes (golden
fixtures worked by hand), a closed form, brute force on tiny inputs, an
independent library computation (torch float64, scipy), or an invariance of
the layer. A wrong table entry, nibble order, sign, tie-break, index or
transposed operand in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def test_e2m1_table_matches_ocp_fixture():
    for ln in _lines("e2m1_codes.txt"):
        code, val = ln.split()
        got = O.e2m1_decode(np.uint8(int(code, 16)))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), ln


def test_e2m1_table_matches_bitfield_definition():
    # closed form of a 1-2-1 minifloat with exponent bias 1 (subnormal at field 0)
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        mag = (m * 0.5) if e == 0 else (2.0 ** (e - 1)) * (1 + m / 2)
        assert O.e2m1_decode(np.uint8(c)) == (-mag if s else mag)


def test_e8m0_fixture_and_closed_form():
    for ln in _lines("e8m0_codes.txt"):
        code, val = ln.split()
        got = float(O.e8m0_decode(np.int64(int(code))))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val)
    c = np.arange(255)
    assert np.array_equal(O.e8m0_decode(c), np.array([math.ldexp(1.0, int(i) - 127) for i in c]))


def test_mxfp4_hand_worked_row():
    lines = _lines("mxfp4_row.txt")
    q = np.array([int(b, 16) for b in lines[0].split()[1:]], dtype=np.uint8)[None]
    s = np.array([int(v) for v in lines[1].split()[1:]], dtype=np.uint8)[None]
    vals = O.mxfp4_dequant(q, s)[0]
    expect = np.zeros(64)
    for ln in lines[2:]:
        _, i, v = ln.split()
        expect[int(i)] = float(v)
    assert np.array_equal(vals, expect)
    assert math.copysign(1, vals[2]) == -1.0     # code 8 is negative zero


def test_mxfp4_nan_scale_poisons_its_block_only():
    q = np.full((1, 32), 0x22, np.uint8)
    s = np.array([[255, 127]], np.uint8)
    v = O.mxfp4_dequant(q, s)[0]
    assert np.all(np.isnan(v[:32])) and np.all(v[32:] == 1.0)


def test_mxfp4_dequant_against_torch_table():
    # an independent decode: torch float64, nibbles unpacked by integer division
    rng = np.random.default_rng(5)
    q = rng.integers(0, 256, (7, 64), dtype=np.uint8)
    s = rng.integers(100, 140, (7, 4), dtype=np.uint8)
    tq = torch.from_numpy(q.astype(np.int64))
    codes = torch.stack([tq % 16, tq // 16], dim=-1).reshape(7, 128)
    table = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6] * 2, dtype=torch.float64)
    sign = torch.where(codes >= 8, -1.0, 1.0).double()
    vals = sign * table[codes]
    scale = torch.pow(2.0, torch.from_numpy(s.astype(np.float64)) - 127).repeat_interleave(32, 1)
    assert np.array_equal(O.mxfp4_dequant(q, s), (vals * scale).numpy())


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    f32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(1e3),
        rng.standard_normal(2000).astype(np.float32) * np.float32(1e-39),   # subnormal range
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3.39e38, 3.4e38, 0.0, -0.0],
                 np.float32),
    ])
    # float32 inputs are exact in float64, so torch's float32 -> bf16 conversion is a
    # single rounding of the same value
    want = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.round_to_bf16_bits(f32.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_rounding_of_float64_ties_is_single_rounding():
    # 1 + 2^-8 + 2^-40 is above the tie: rounds up; a float32 detour would round to the
    # tie first and then to even (down)
    v = np.array([1 + 2 ** -8 + 2 ** -40, 1 + 2 ** -8 - 2 ** -40])
    assert list(O.round_to_bf16_bits(v)) == [0x3F81, 0x3F80]


# ---------------------------------------------------------------------------
# quantiser
# ---------------------------------------------------------------------------

def test_quantize_hand_worked_blocks():
    for ln in _lines("mxfp4_quantize_blocks.txt"):
        _, rest = ln.split(" ", 1)
        name, vals, scale, codes = [p.strip() for p in rest.split("|")]
        vals = [float(v) for v in vals.split()]
        block = np.zeros(32)
        block[:len(vals)] = vals
        c, s = O.mxfp4_quantize(block[None])
        assert int(s[0, 0]) == int(scale), name
        assert [int(v) for v in c[0, :len(vals)]] == [int(v) for v in codes.split()], name
        assert np.all(c[0, len(vals):] == 0), name


def test_quantize_roundtrips_every_representable_value():
    # any block whose values are already E2M1 x 2^X with amax in [4, 8) * 2^X
    # quantises to itself
    for X in (-20, -3, 0, 5, 40):
        mags = np.array(list(O.E2M1_MAGNITUDES) * 4)
        vals = np.where(np.arange(32) % 3 == 0, -1, 1) * mags * 2.0 ** X
        vals[0] = 6.0 * 2.0 ** X
        c, s = O.mxfp4_quantize(vals[None])
        assert int(s[0, 0]) == 127 + X
        assert np.array_equal(O.mxfp4_values(c, s)[0], vals)


def test_quantize_error_bound():
    rng = np.random.default_rng(3)
    v = rng.standard_normal((50, 128)) * 10 ** rng.uniform(-3, 3, (50, 1))
    c, s = O.mxfp4_quantize(v)
    d = O.mxfp4_values(c, s)
    scale = np.repeat(O.e8m0_decode(s), 32, axis=-1)
    # between representable neighbours the error is at most half the local spacing,
    # which is at most 1 (between 4 and 6) in units of the scale, and values above
    # 6 * scale saturate to 6 * scale
    err = np.abs(v - d) / scale
    assert np.all((err <= 1.0 + 1e-12) | (np.abs(v) > 6 * scale))
    assert np.all(np.abs(v) / scale < 8)      # amax / 2^X < 8 by the choice of X


def test_quantize_zero_block():
    c, s = O.mxfp4_quantize(np.zeros((1, 32)))
    assert s[0, 0] == 0 and np.all(c == 0)


def test_pack_is_low_nibble_first():
    codes = np.tile(np.arange(16, dtype=np.uint8), 2)[None]
    packed = O.mxfp4_pack(codes)
    assert packed[0, 0] == 0x10 and packed[0, 1] == 0x32


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

def _brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-row[e], e))
    return order[:k]


def test_topk_brute_force_with_exact_ties():
    rng = np.random.default_rng(7)
    logits = np.round(rng.standard_normal((40, 12)) * 2) / 2     # many exact ties
    for k in (1, 2, 3, 12):
        idx, w, flagged = O.topk_route(logits, k)
        for t in range(40):
            assert list(idx[t]) == _brute_topk(list(logits[t]), k)


def test_topk_weights_equal_renormalised_full_softmax():
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((30, 64)) * 1.8
    idx, w, _ = O.topk_route(logits, 10)
    p = scipy.special.softmax(logits, axis=1)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-13)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-13)
    assert np.all(np.diff(w, axis=1) <= 0)      # slots in descending weight


def test_selection_weights_of_any_choice_equal_renormalised_full_softmax():
    # any k distinct experts, not only the top k (the weight rule of a near-tie choice)
    rng = np.random.default_rng(9)
    logits = rng.standard_normal((20, 48)) * 1.8
    idx = np.stack([rng.permutation(48)[:6] for _ in range(20)]).astype(np.int32)
    p = scipy.special.softmax(logits, axis=1)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(O.selection_weights(logits, idx), sel / sel.sum(axis=1, keepdims=True),
                               rtol=1e-13)


def test_topk_near_tie_flags_split_set_boundary_from_slot_order():
    logits = np.array([[3.0, 2.0, 1.0, 1.0 - 5e-6, 0.0],     # k-th vs (k+1)-th: the set
                       [3.0, 2.0, 1.0, 0.5, 0.0],            # no tie
                       [3.0, 3.0 - 1e-6, 1.0, 0.5, 0.0]])    # inside the set: the order only
    _, _, flagged = O.topk_route(logits, 3)
    assert list(flagged) == [True, False, False]
    _, _, flags = O.route(logits, 3)
    assert list(flags) == [O.TIE_SET, 0, O.TIE_ORDER]


def test_router_logits_against_torch():
    w = synth.WORKLOADS["tiny"]
    d = synth.dense_inputs(w)
    x = torch.from_numpy(d["x"].view(np.int16)).view(torch.bfloat16).double()
    wr = torch.from_numpy(d["w_router"].view(np.int16)).view(torch.bfloat16).double()
    np.testing.assert_allclose(O.router_logits(d["x"], d["w_router"]), (x @ wr.T).numpy(),
                               rtol=1e-12, atol=1e-12)


def test_permute_brute_force():
    rng = np.random.default_rng(9)
    for T, E, k in ((1, 4, 2), (5, 6, 3), (17, 9, 4), (8, 3, 3)):
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
        counts, offsets, row_token, row_slot, slot_row = O.permute(idx, E)
        rows = []
        for e in range(E):
            for t in range(T):
                for j in range(k):
                    if idx[t, j] == e:
                        rows.append((t, j))
        assert [(int(a), int(b)) for a, b in zip(row_token, row_slot)] == rows
        assert list(counts) == [sum(1 for t in range(T) for j in range(k) if idx[t, j] == e)
                                for e in range(E)]
        assert offsets[0] == 0 and offsets[-1] == T * k and np.all(np.diff(offsets) == counts)
        for r, (t, j) in enumerate(rows):
            assert slot_row[t, j] == r


# ---------------------------------------------------------------------------
# expert FFN, shared expert, combine, whole layer
# ---------------------------------------------------------------------------

def _torch_dense_swiglu(x, wg, wu, wd):
    x, wg, wu, wd = (torch.from_numpy(np.asarray(a, np.float64)) for a in (x, wg, wu, wd))
    return (torch.nn.functional.silu(x @ wg.T) * (x @ wu.T)) @ wd.T


def _torch_decode(q, s):
    tq = torch.from_numpy(np.asarray(q).astype(np.int64))
    n = tq.shape[-1] * 2
    codes = torch.stack([tq % 16, tq // 16], dim=-1).reshape(*tq.shape[:-1], n)
    table = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6] * 2, dtype=torch.float64)
    vals = torch.where(codes >= 8, -1.0, 1.0).double() * table[codes]
    return vals * torch.pow(2.0, torch.from_numpy(np.asarray(s).astype(np.float64)) - 127) \
        .repeat_interleave(32, -1)


def _tiny_layer_inputs(E=1, k=1, T=5, H=64, I=96, seed=11):
    w = synth.MoeWorkload("t", T=T, H=H, I=I, E=E, k=k, I_shared=32, seed=seed)
    d = synth.dense_inputs(w)
    ex = synth.expert_weights(w, range(E))
    get = lambda e: tuple(ex[n][e] for n in ("wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s"))
    return w, d, ex, get


def test_single_expert_top1_equals_dense_swiglu_in_torch():
    w, d, ex, get = _tiny_layer_inputs(E=1, k=1)
    out = O.moe_layer(d, 1, get)
    x = O.bf16_to_f64(d["x"])
    wg = _torch_decode(ex["wg_q"][0], ex["wg_s"][0]).numpy()
    wu = _torch_decode(ex["wu_q"][0], ex["wu_s"][0]).numpy()
    wd = _torch_decode(ex["wd_q"][0], ex["wd_s"][0]).numpy()
    routed = _torch_dense_swiglu(x, wg, wu, wd).numpy()
    assert np.all(out["w"] == 1.0)
    xs = torch.from_numpy(x)
    bf = lambda a: torch.from_numpy(O.bf16_to_f64(d[a]))
    shared = torch.sigmoid(xs @ bf("w_sgate"))[:, None] * _torch_dense_swiglu(
        x, bf("ws_gate").numpy(), bf("ws_up").numpy(), bf("ws_down").numpy())
    np.testing.assert_allclose(out["y"], routed + shared.numpy(), rtol=1e-12, atol=1e-9)
    np.testing.assert_allclose(out["shared"], shared.numpy(), rtol=1e-12, atol=1e-12)


def test_zero_gate_vector_gives_half_gate():
    w, d, ex, get = _tiny_layer_inputs(E=2, k=1)
    d = dict(d, w_sgate=np.zeros_like(d["w_sgate"]))
    _, gate = O.shared_expert(d["x"], d["ws_gate"], d["ws_up"], d["ws_down"], d["w_sgate"])
    assert np.all(gate == 0.5)


def test_dense_masked_equivalence():
    # sum over ALL experts of mask * weight * FFN_e equals the routed layer
    w, d, ex, get = _tiny_layer_inputs(E=6, k=3, T=7)
    out = O.moe_layer(d, 3, get)
    x = O.bf16_to_f64(d["x"])
    y = out["shared"].copy()
    for e in range(6):
        wg = _torch_decode(ex["wg_q"][e], ex["wg_s"][e]).numpy()
        wu = _torch_decode(ex["wu_q"][e], ex["wu_s"][e]).numpy()
        wd = _torch_decode(ex["wd_q"][e], ex["wd_s"][e]).numpy()
        ffn = _torch_dense_swiglu(x, wg, wu, wd).numpy()
        mask = np.zeros(7)
        for t in range(7):
            for j in range(3):
                if out["idx"][t, j] == e:
                    mask[t] = out["w"][t, j]
        y += mask[:, None] * ffn
    scale = np.sqrt(np.mean(y ** 2))
    np.testing.assert_allclose(out["y"], y, rtol=0, atol=1e-11 * scale)


def test_expert_relabelling_invariance():
    w, d, ex, get = _tiny_layer_inputs(E=8, k=3, T=6)
    base = O.moe_layer(d, 3, get)
    perm = np.random.default_rng(2).permutation(8)        # new id of old expert e is perm[e]
    inv = np.argsort(perm)
    d2 = dict(d, w_router=d["w_router"][inv])
    get2 = lambda e: get(int(inv[e]))
    out = O.moe_layer(d2, 3, get2)
    assert np.array_equal(out["idx"], perm[base["idx"]])
    np.testing.assert_array_equal(out["y"], base["y"])


def test_batch_invariance():
    w, d, ex, get = _tiny_layer_inputs(E=5, k=2, T=6)
    full = O.moe_layer(d, 2, get)
    for t in range(6):
        one = O.moe_layer(dict(d, x=d["x"][t:t + 1]), 2, get)
        # equal up to float64 reassociation inside the BLAS matmul
        np.testing.assert_allclose(one["y"][0], full["y"][t], rtol=1e-12,
                                   atol=1e-12 * np.abs(full["y"]).max())
        np.testing.assert_array_equal(one["idx"][0], full["idx"][t])


def test_latent_identity_reduces_to_plain_layer():
    # with L = H and identity projections the latent layer is the plain layer
    w, d, ex, get = _tiny_layer_inputs(E=4, k=2, T=3, H=64)
    eye = synth.f32_to_bf16_bits(np.eye(64, dtype=np.float32))
    plain = O.moe_layer(d, 2, get)
    lat = O.moe_layer(dict(d, w_lat_down=eye, w_lat_up=eye), 2, get)
    np.testing.assert_array_equal(lat["x_lat"], d["x"])
    np.testing.assert_allclose(lat["y"], plain["y"], rtol=1e-13, atol=0)


def test_mxfp4_activation_mode_quantises_both_operands():
    # with act="mxfp4" the expert equals the exact expert run on pre-quantised x,
    # with h quantised before the down projection (products in torch float64)
    w, d, ex, get = _tiny_layer_inputs(E=1, k=1, T=3)
    wg = _torch_decode(ex["wg_q"][0], ex["wg_s"][0])
    wu = _torch_decode(ex["wu_q"][0], ex["wu_s"][0])
    wd = _torch_decode(ex["wd_q"][0], ex["wd_s"][0])
    x = O.bf16_to_f64(d["x"])
    y, h, h_raw = O.expert_ffn(x, *get(0), act="mxfp4", h_raw=True)
    xq = torch.from_numpy(O.mxfp4_values(*O.mxfp4_quantize(x)))
    h_ref = (torch.nn.functional.silu(xq @ wg.T) * (xq @ wu.T)).numpy()
    np.testing.assert_allclose(h_raw, h_ref, rtol=1e-12, atol=1e-300)
    hq = O.mxfp4_values(*O.mxfp4_quantize(h_ref))
    np.testing.assert_array_equal(h, hq)
    np.testing.assert_allclose(y, (torch.from_numpy(hq) @ wd.T).numpy(), rtol=1e-12)
    assert not np.array_equal(xq.numpy(), x)
    # and act="exact" leaves both unrounded
    y0, h0 = O.expert_ffn(x, *get(0))
    xt = torch.from_numpy(x)
    np.testing.assert_allclose(y0, _torch_dense_swiglu(x, wg.numpy(), wu.numpy(), wd.numpy()).numpy(),
                               rtol=1e-11, atol=1e-12 * np.abs(y0).max())
    np.testing.assert_allclose(h0, (torch.nn.functional.silu(xt @ wg.T) * (xt @ wu.T)).numpy(),
                               rtol=1e-11, atol=1e-300)


def test_mxfp4_matmul_against_torch():
    rng = np.random.default_rng(12)
    q = rng.integers(0, 256, (24, 48), dtype=np.uint8)
    s = rng.integers(115, 135, (24, 3), dtype=np.uint8)
    x = rng.standard_normal((5, 96))
    want = (torch.from_numpy(x) @ _torch_decode(q, s).T).numpy()
    np.testing.assert_allclose(O.mxfp4_matmul(q, s, x), want, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# latent layers (L != H)
# ---------------------------------------------------------------------------

def _latent_inputs(T=4, H=96, L=64, I=64, E=6, k=2, seed=21):
    w = synth.MoeWorkload("lat", T=T, H=H, I=I, E=E, k=k, I_shared=32, L=L, seed=seed)
    d = synth.dense_inputs(w)
    ex = synth.expert_weights(w, range(E))
    get = lambda e: tuple(ex[n][e] for n in ("wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s"))
    return w, d, ex, get


def _torch_latent_layer(d, ex, idx, wts, x_lat):
    """The latent layer in torch float64 from a given routing and expert input x_lat [T, L]."""
    bf = lambda a: torch.from_numpy(O.bf16_to_f64(d[a]))
    xl = torch.as_tensor(x_lat, dtype=torch.float64)
    T, k = idx.shape
    acc = torch.zeros(T, xl.shape[1], dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            wg, wu, wd = (_torch_decode(ex[a][e], ex[b][e])
                          for a, b in (("wg_q", "wg_s"), ("wu_q", "wu_s"), ("wd_q", "wd_s")))
            h = torch.nn.functional.silu(xl[t] @ wg.T) * (xl[t] @ wu.T)
            acc[t] += float(wts[t, j]) * (h @ wd.T)
    x = bf("x")
    shared = torch.sigmoid(x @ bf("w_sgate"))[:, None] * (
        (torch.nn.functional.silu(x @ bf("ws_gate").T) * (x @ bf("ws_up").T)) @ bf("ws_down").T)
    return (acc @ bf("w_lat_up").T + shared).numpy()


def test_latent_down_against_torch_with_random_projection():
    w, d, ex, get = _latent_inputs()
    x = torch.from_numpy(O.bf16_to_f64(d["x"]))
    prod = (x @ torch.from_numpy(O.bf16_to_f64(d["w_lat_down"])).T).numpy()
    got = O.latent_down(d["x"], d["w_lat_down"])
    # torch rounds float64 -> bfloat16 through float32; that double rounding can
    # differ from one rounding only where the float32 value lands on a bf16 tie
    want = torch.from_numpy(prod).float().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    f32 = prod.astype(np.float32).view(np.uint32)
    on_tie = (f32 & 0xFFFF) == 0x8000
    assert np.array_equal(got[~on_tie], want[~on_tie])
    assert got.shape == (w.T, w.L)


def test_latent_layer_against_torch_and_rounding_point_matters():
    w, d, ex, get = _latent_inputs()
    out = O.moe_layer(d, w.k, get)
    x_lat = O.bf16_to_f64(out["x_lat"])
    ref = _torch_latent_layer(d, ex, out["idx"], out["w"], x_lat)
    scale = np.abs(ref).max()
    np.testing.assert_allclose(out["y"], ref, rtol=0, atol=1e-12 * scale)
    # the bf16 rounding of x_lat changes the input bits, and an oracle without
    # that rounding point would be far outside the bound above
    prod = (torch.from_numpy(O.bf16_to_f64(d["x"]))
            @ torch.from_numpy(O.bf16_to_f64(d["w_lat_down"])).T).numpy()
    assert np.mean(x_lat != prod) > 0.9
    unrounded = _torch_latent_layer(d, ex, out["idx"], out["w"], prod)
    assert np.abs(unrounded - out["y"]).max() > 1e-6 * scale
    # the routing sees the full-width x, not x_lat
    np.testing.assert_array_equal(out["idx"], O.topk_route(O.router_logits(d["x"], d["w_router"]),
                                                           w.k)[0])


# ---------------------------------------------------------------------------
# the C++ oracle against the independent numpy restatement
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kind", ["plain", "latent", "mxfp4", "skewed"])
def test_cpp_oracle_matches_numpy_restatement(kind):
    from oracle import moe_oracle_np as N
    if kind == "latent":
        w, d, ex, get = _latent_inputs(T=5, E=7, k=3, seed=31)
    elif kind == "skewed":
        w = synth.MoeWorkload("sk", T=9, H=128, I=64, E=16, k=4, I_shared=32, skew="hot64",
                              seed=33)
        d = synth.dense_inputs(w)
        ex = synth.expert_weights(w, range(w.E))
        get = lambda e: tuple(ex[n][e] for n in ("wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s"))
    else:
        w, d, ex, get = _tiny_layer_inputs(E=8, k=3, T=6, seed=32)
    act = "mxfp4" if kind == "mxfp4" else "exact"
    a = O.moe_layer(d, w.k, get, act=act)
    b = N.moe_layer(d, w.k, get, act=act)
    for name in ("idx", "counts", "offsets", "row_token", "row_slot", "slot_row", "flagged"):
        np.testing.assert_array_equal(a[name], b[name], err_msg=name)
    if kind == "latent":
        np.testing.assert_array_equal(a["x_lat"], b["x_lat"])
    for name in ("logits", "w", "y_perm", "shared", "gate", "y"):
        scale = max(np.abs(b[name]).max(), 1e-300)
        np.testing.assert_allclose(a[name], b[name], rtol=0, atol=1e-12 * scale, err_msg=name)


def test_silu_sigmoid_match_torch_including_extremes():
    z = np.concatenate([np.linspace(-50, 50, 1001), [-800.0, 800.0, 0.0]])
    np.testing.assert_allclose(O.silu(z), torch.nn.functional.silu(torch.from_numpy(z)).numpy(),
                               rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(O.sigmoid(z), torch.sigmoid(torch.from_numpy(z)).numpy(),
                               rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------------------
# router variants: sigmoid scores with a selection bias ("noaux_tc sigmoid"),
# group-limited selection ("grouped routing")
# ---------------------------------------------------------------------------

def test_sigmoid_router_without_bias_selects_like_softmax():
    # sigmoid and softmax are both monotone in the logit: same experts, same order
    rng = np.random.default_rng(41)
    logits = rng.standard_normal((25, 32)) * 1.8
    a, _, _ = O.route(logits, 6)
    b, w, _ = O.route(logits, 6, score_fn=O.SIGMOID, scale=2.5)
    np.testing.assert_array_equal(a, b)
    s = scipy.special.expit(np.take_along_axis(logits, b.astype(np.int64), axis=1))
    np.testing.assert_allclose(w, 2.5 * s / s.sum(axis=1, keepdims=True), rtol=1e-14)


def test_sigmoid_router_with_bias_brute_force():
    rng = np.random.default_rng(42)
    logits = rng.standard_normal((30, 12)) * 1.8
    bias = np.round(rng.standard_normal(12) * 0.2, 3)
    idx, w, _ = O.route(logits, 4, score_fn=O.SIGMOID, bias=bias)
    for t in range(30):
        s = [1.0 / (1.0 + math.exp(-v)) for v in logits[t]]
        order = sorted(range(12), key=lambda e: (-(s[e] + bias[e]), e))[:4]
        assert list(idx[t]) == order
        tot = sum(s[e] for e in order)
        np.testing.assert_allclose(w[t], [s[e] / tot for e in order], rtol=1e-14)
    # the bias changes the selection somewhere, and not the weight rule
    plain, _, _ = O.route(logits, 4, score_fn=O.SIGMOID)
    assert not np.array_equal(np.sort(plain, axis=1), np.sort(idx, axis=1))


def test_softmax_router_ignores_the_selection_bias():
    rng = np.random.default_rng(43)
    logits = rng.standard_normal((10, 16))
    a = O.route(logits, 3)
    b = O.route(logits, 3, bias=rng.standard_normal(16))
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_grouped_sigmoid_router_hand_worked():
    # 8 experts in 4 groups of 2, keep 2 groups, top-3, weights x 2.5.
    # logits 0 except expert 6 (ln 3): sigmoid scores 0.5, and 0.75 for expert 6;
    # with the bias, selection scores
    #   [0.625, 0.5 | 0.875, 0.1875 | 0.5625, 0.5 | 0.75, 0.8125]
    # group scores (sum of the two largest): 1.125, 1.0625, 1.0625, 1.5625
    # -> keep groups 3 and 0; expert 2 (0.875, the best overall) is excluded;
    # top-3 of {0, 1, 6, 7}: 7 (0.8125), 6 (0.75), 0 (0.625);
    # weights 2.5 * [0.5, 0.75, 0.5] / 1.75 from the unbiased scores
    logits = np.zeros((1, 8))
    logits[0, 6] = math.log(3.0)
    bias = np.array([0.125, 0, 0.375, -0.3125, 0.0625, 0, 0, 0.3125])
    idx, w, flags = O.route(logits, 3, score_fn=O.SIGMOID, bias=bias, n_group=4, topk_group=2,
                            scale=2.5)
    assert list(idx[0]) == [7, 6, 0]
    np.testing.assert_allclose(w[0], 2.5 * np.array([0.5, 0.75, 0.5]) / 1.75, rtol=1e-14)
    assert flags[0] == 0
    # without groups expert 2 wins
    idx2, _, _ = O.route(logits, 3, score_fn=O.SIGMOID, bias=bias)
    assert list(idx2[0]) == [2, 7, 6]


def test_grouped_softmax_router_hand_worked():
    # 8 experts in 4 groups of 2, keep 2 groups, top-3; group scores on the
    # probabilities (exp(l - 3)): g0 = e^-1 + e^-1.1 = 0.7008,
    # g1 = 1 + e^-8 = 1.0003, g2 = 2 e^-3 = 0.0996, g3 = e^-0.5 + e^-3 = 0.6563
    # -> keep g1, g0; expert 6 (logit 2.5, second overall) is excluded;
    # top-3 of {0, 1, 2, 3}: 2, 0, 1; weights = softmax renormalised over them
    logits = np.array([[2.0, 1.9, 3.0, -5.0, 0.0, 0.0, 2.5, 0.0]])
    idx, w, flags = O.route(logits, 3, n_group=4, topk_group=2)
    assert list(idx[0]) == [2, 0, 1]
    e = np.array([1.0, math.exp(-1.0), math.exp(-1.1)])
    np.testing.assert_allclose(w[0], e / e.sum(), rtol=1e-14)
    assert flags[0] == 0
    assert list(O.route(logits, 3)[0][0]) == [2, 6, 0]


def test_grouped_router_reduces_to_plain_routing():
    rng = np.random.default_rng(44)
    logits = rng.standard_normal((20, 24)) * 1.8
    bias = rng.standard_normal(24) * 0.1
    for fn, b in ((O.SOFTMAX, None), (O.SIGMOID, bias)):
        plain = O.route(logits, 5, score_fn=fn, bias=b)
        # every group kept
        allg = O.route(logits, 5, score_fn=fn, bias=b, n_group=4, topk_group=4)
        # one expert per group, k groups kept: the group scores rank like the experts
        single = O.route(logits, 5, score_fn=fn, bias=b, n_group=24, topk_group=5)
        for other in (allg, single):
            np.testing.assert_array_equal(plain[0], other[0])
            np.testing.assert_allclose(plain[1], other[1], rtol=1e-15)


def test_grouped_router_group_near_tie_flag_and_rejections():
    logits = np.zeros((1, 8))
    bias = np.array([0.25, 0.25, 0.25, 0.25, 0.0, 0.0, 0.0, 0.0])
    _, _, flags = O.route(logits, 2, score_fn=O.SIGMOID, bias=bias, n_group=4, topk_group=1)
    assert flags[0] & O.TIE_GROUP        # groups 0 and 1 tie exactly
    with pytest.raises(ValueError):
        O.route(logits, 2, n_group=3, topk_group=1)       # 8 experts do not split in 3
    with pytest.raises(ValueError):
        O.route(logits, 3, n_group=4, topk_group=1)       # one group of 2 cannot give 3
