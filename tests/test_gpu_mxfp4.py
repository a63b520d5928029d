"""GPU parity of the MXFP4-activation path (MOE_ACT_MXFP4: activations and the
SwiGLU output h quantised to MXFP4, expert GEMMs on the tcgen05 block-scaled
tensor cores) against the fp64 oracle, stage by stage:

* x operand: E2M1 codes and E8M0 scales bit-exact (both sides quantise the
  same bf16 values, and the decision is exact in fp32);
* h operand: the oracle's own MXFP4 encoding of its fp64 h, bit-exact except
  where the oracle's value sits within a small window of a rounding decision
  (a midpoint between two E2M1 values, zero, or a block maximum at a power of
  two); there the GPU's choice must be one of the two valid encodings and is
  then used as the reference (the same rule as for near-tie routing);
* expert rows y_perm = h Wd^T and the layer output: max |err| <= 1e-2 x RMS.

Full-size prefill (T=4096, H=8192, I=2048, E=512, top-10) is checked on sampled
tokens; the smaller shapes span several M, N and K tiles, ragged N tails, a K
that is not a multiple of 256, a W that is not a multiple of 256 and experts
with more than one token tile.
"""
import gc

import numpy as np
import pytest
import torch

import mxfp4_routed_expert_04_b200 as M
import oracle as O
import synth

from parity_harness import TOL, DeviceRun, check_permutation, check_routing, expert_getter, max_rel_err

pytestmark = pytest.mark.gpu

MID = (O.E2M1_MAGNITUDES[1:] + O.E2M1_MAGNITUDES[:-1]) / 2     # rounding decisions of E2M1
WIN = 2e-4          # decision window, in units of the block scale (scaled values are < 8)
WIN_POW2 = 2e-5     # relative window of a block maximum around a power of two

MEDIUM = synth.MoeWorkload("mx_medium", T=300, H=512, I=384, E=6, k=3, I_shared=256, seed=81)
SKEWED = synth.MoeWorkload("mx_skewed", T=1024, H=1024, I=256, E=16, k=4, I_shared=256,
                           skew="zipf", seed=82)
# H = 384: the down projection's last 256-row pair of Wd has a single 128-row tile
ODD_H = synth.MoeWorkload("mx_odd_h", T=200, H=384, I=128, E=5, k=2, I_shared=128, seed=83)

CASES = [
    (synth.WORKLOADS["tiny"], None),
    (MEDIUM, None),
    (SKEWED, None),
    (ODD_H, None),
    # sampled tokens at full size: fixed ones plus, chosen from the GPU's routing,
    # a token of the hottest expert in its last tile and one in the ragged last
    # tile of an expert with several tiles
    (synth.WORKLOADS["prefill4096"], [0, 1, 2047, 4095, "hot", "ragged"]),
]


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def _untile(buf, tiles, R, K):
    """Canonical [R, K/32] scales from the tiled layout (the header's formula:
    row n of tile t, K-block j at (t*K/128 + j/4)*512 + 16*(n%32) + 4*(n/32) + j%4)."""
    out = np.zeros((R, K // 32), dtype=np.uint8)
    j = np.arange(K // 32)[None, :]
    for t, (e, row0, nrows, _) in enumerate(tiles):
        n = np.arange(nrows)[:, None]
        off = (t * (K // 128) + j // 4) * 512 + 16 * (n % 32) + 4 * (n // 32) + j % 4
        out[row0:row0 + nrows] = buf[off]
    return out


def _tile_list_reference(offsets, expert_list, tile_rows):
    tiles = []
    for e in expert_list[1:1 + expert_list[0]]:
        first, cnt = int(offsets[e]), int(offsets[e + 1] - offsets[e])
        for j in range(0, cnt, tile_rows):
            tiles.append((int(e), first + j, min(tile_rows, cnt - j), 0))
    return np.array(tiles, dtype=np.int32).reshape(-1, 4)


def _mxf4_operands(run, gpu):
    """x operand, tile list and h operand of the MXFP4 path, in canonical form."""
    w, L = run.w, run.layer
    lay = M.moe_mxf4_layout_of(run.dims)
    R = w.T * w.k
    xo = gpu["x_op"]
    n_tiles = int(xo[lay.n_tiles:lay.n_tiles + 4].view(np.int32)[0])
    tiles = xo[lay.tiles:lay.tiles + 16 * n_tiles].view(np.int32).reshape(n_tiles, 4)
    tile_base = xo[lay.tile_base:lay.tile_base + 4 * w.E].view(np.int32)
    x_codes = xo[:R * w.W // 2].reshape(R, w.W // 2)
    x_scales = _untile(xo[lay.x_scales:], tiles, R, w.W)
    ws = L.ws
    h_codes = ws[lay.h_codes:lay.h_codes + R * w.I // 2].cpu().numpy().reshape(R, w.I // 2)
    h_buf = ws[lay.h_scales:lay.h_scales + lay.max_tiles * (w.I // 128) * 512].cpu().numpy()
    return dict(tiles=tiles, tile_base=tile_base, tile_rows=lay.tile_rows, x_codes=x_codes,
                x_scales=x_scales, h_codes=h_codes, h_scales=_untile(h_buf, tiles, R, w.I))


def _unpack(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


@pytest.fixture(scope="module", params=CASES, ids=lambda c: c[0].name)
def case(request):
    w, sample = request.param
    run = DeviceRun(w, act_mode=M.ACT_MXFP4)
    gpu = run.run_stages()
    gpu.update(_mxf4_operands(run, gpu))
    assert M.moe_device_status(run.layer.ws) == 0
    yield w, sample, run, gpu
    del run
    _free()


def _sample_tokens(w, gpu, sample):
    """Token ids of a sample; "hot" and "ragged" pick tokens from the GPU's
    routing (validated separately against the oracle)."""
    if sample is None:
        return np.arange(w.T)
    counts = np.diff(gpu["offsets"])
    tr = int(gpu["tile_rows"])
    out = []
    for s in sample:
        if s == "hot":
            e = int(np.argmax(counts))
            out.append(int(gpu["row_token"][gpu["offsets"][e + 1] - 1]))
        elif s == "ragged":
            multi = np.nonzero((counts > tr) & (counts % tr != 0))[0]
            assert len(multi), "no expert with a ragged last tile"
            e = int(multi[np.argmax(counts[multi])])
            out.append(int(gpu["row_token"][gpu["offsets"][e + 1] - 1]))
        else:
            out.append(int(s))
    return np.unique(np.array(out))


def _rows_of(w, gpu, sample):
    return np.concatenate([gpu["slot_row"][t] for t in _sample_tokens(w, gpu, sample)])


def test_routing_and_permutation(case):
    w, sample, run, gpu = case
    check_routing(gpu, O.router_logits(run.dense["x"], run.dense["w_router"]), w.k)
    check_permutation(gpu, w.E)


def test_tile_list(case):
    w, sample, run, gpu = case
    ref = _tile_list_reference(gpu["offsets"], gpu["expert_list"], gpu["tile_rows"])
    np.testing.assert_array_equal(gpu["tiles"], ref)
    firsts = {}
    for t, (e, _, _, _) in enumerate(ref):
        firsts.setdefault(e, t)
    for e, t in firsts.items():
        assert gpu["tile_base"][e] == t


def test_x_operand_bit_exact(case):
    """Every permuted row r holds the MXFP4 encoding of token row_token[r]."""
    w, sample, run, gpu = case
    codes, scales = O.mxfp4_quantize(O.bf16_to_f64(run.dense["x"]))
    tok = gpu["row_token"]
    np.testing.assert_array_equal(gpu["x_codes"], O.mxfp4_pack(codes)[tok])
    np.testing.assert_array_equal(gpu["x_scales"], scales[tok])


def _reference_h(h64, g_codes, g_scales):
    """Oracle encoding of h64 [n, I], with the GPU's choice taken (after checking
    it is valid) only inside the decision windows. Returns (values [n, I],
    number of elements taken from the GPU)."""
    n, I = h64.shape
    codes, scales = O.mxfp4_quantize(h64)
    gc_ = _unpack(g_codes).reshape(n, I)
    gs = np.asarray(g_scales).reshape(n, I // 32)
    blk = h64.reshape(n, I // 32, 32)
    amax = np.abs(blk).max(axis=-1)
    l2 = np.log2(np.where(amax > 0, amax, 1.0))
    near_pow2 = (amax > 0) & (np.abs(l2 - np.round(l2)) < WIN_POW2)
    scale_diff = gs != scales
    assert not np.any(scale_diff & ~near_pow2), "block scale differs away from a power of two"
    assert np.all(np.abs(gs.astype(int) - scales.astype(int)) <= 1)
    ref = O.mxfp4_values(codes, scales)
    gpu_vals = O.mxfp4_values(gc_, gs)
    # blocks whose scale decision went the other way: every value within the
    # coarser grid's largest half-step (or the saturation at 6) of h64
    taken = 0
    for b in zip(*np.nonzero(scale_diff)):
        r, j = b
        sl = slice(32 * j, 32 * j + 32)
        unit = np.ldexp(1.0, int(max(gs[r, j], scales[r, j])) - 127)
        assert np.all(np.abs(gpu_vals[r, sl] - h64[r, sl]) <= 2 * unit)
        ref[r, sl] = gpu_vals[r, sl]
        taken += 32
    same = ~np.repeat(scale_diff, 32, axis=1)
    s = np.abs(h64) / np.repeat(np.ldexp(1.0, scales.astype(int) - 127), 32, axis=1)
    near = (np.min(np.abs(s[..., None] - MID), axis=-1) < WIN) | (s < WIN)
    mag_o, mag_g = codes & 7, gc_ & 7
    differ = same & ((mag_o != mag_g) | ((codes != gc_) & (mag_o != 0)))
    assert not np.any(differ & ~near), (
        f"{int(np.sum(differ & ~near))} h codes differ outside the decision windows")
    # inside a window the GPU code is one of the two neighbours of the decision
    d = differ & near
    assert np.all(np.abs(mag_o[d].astype(int) - mag_g[d].astype(int)) <= 1)
    ref[d] = gpu_vals[d]
    return ref, taken + int(np.sum(d))


def _oracle_rows(w, run, gpu, rows):
    """h64 and the reference h / y_perm of permuted rows `rows` (GPU permutation,
    validated by test_routing_and_permutation)."""
    get = expert_getter(w)
    x64 = O.bf16_to_f64(run.dense["x"])
    off = gpu["offsets"]
    ex = np.searchsorted(off, rows, side="right") - 1
    h_ref = np.zeros((len(rows), w.I))
    y_ref = np.zeros((len(rows), w.W))
    taken = 0
    for e in np.unique(ex):
        sel = np.nonzero(ex == e)[0]
        rr = rows[sel]
        wg_q, wg_s, wu_q, wu_s, wd_q, wd_s = get(int(e))
        # h before its quantisation (the oracle's expert with MXFP4 activations)
        _, _, h64 = O.expert_ffn(x64[gpu["row_token"][rr]], wg_q, wg_s, wu_q, wu_s, wd_q, wd_s,
                                 act="mxfp4", h_raw=True)
        href, t = _reference_h(h64, gpu["h_codes"][rr], gpu["h_scales"][rr])
        taken += t
        h_ref[sel] = href
        y_ref[sel] = O.mxfp4_matmul(wd_q, wd_s, href)
    return h_ref, y_ref, taken


@pytest.fixture(scope="module")
def rows_ref(case):
    w, sample, run, gpu = case
    rows = _rows_of(w, gpu, sample)
    h_ref, y_ref, taken = _oracle_rows(w, run, gpu, rows)
    return rows, h_ref, y_ref, taken


def test_h_operand(case, rows_ref):
    w, sample, run, gpu = case
    rows, h_ref, y_ref, taken = rows_ref
    # all checks happen in _reference_h; the GPU's choice may be taken only rarely
    assert taken <= max(8, 1e-4 * h_ref.size), taken


def test_expert_rows(case, rows_ref):
    w, sample, run, gpu = case
    rows, h_ref, y_ref, taken = rows_ref
    err, rms = max_rel_err(gpu["y_perm"][rows], y_ref)
    assert err <= TOL, (err, rms)


def test_layer_output(case, rows_ref):
    w, sample, run, gpu = case
    rows, h_ref, y_ref, taken = rows_ref
    d = run.dense
    tokens = _sample_tokens(w, gpu, sample)
    # the oracle's weights of the GPU's selection (equal to the oracle's own
    # selection as a set wherever that is not a near tie:
    # test_routing_and_permutation), whose rows y_ref holds
    logits = O.router_logits(d["x"][tokens], d["w_router"])
    w_ref = O.selection_weights(logits, gpu["idx"][tokens])
    y_perm = np.zeros((w.T * w.k, w.W))
    y_perm[rows] = y_ref
    shared, _ = O.shared_expert(d["x"][tokens], d["ws_gate"], d["ws_up"], d["ws_down"], d["w_sgate"])
    ref = O.combine(y_perm, gpu["slot_row"][tokens], w_ref, shared)
    err, rms = max_rel_err(gpu["y"][tokens], ref)
    assert err <= TOL, (err, rms)
    # the fused moe_layer path against the same reference
    y_layer = run.run_layer()
    err, rms = max_rel_err(y_layer[tokens], ref)
    assert err <= TOL, ("moe_layer", err, rms)


def test_fused_layer_matches_stages_bitwise(case):
    w, sample, run, gpu = case
    y = run.run_layer()
    np.testing.assert_array_equal(y, gpu["y"])


def test_sample_covers_hot_and_ragged_tiles(case):
    w, sample, run, gpu = case
    if sample is None:
        pytest.skip("every token is checked")
    tokens = _sample_tokens(w, gpu, sample)
    counts = np.diff(gpu["offsets"])
    experts = set(gpu["idx"][tokens].ravel().tolist())
    assert int(np.argmax(counts)) in experts
    assert counts.max() > 2 * int(gpu["tile_rows"])


def test_tile_scales_matches_the_tiled_layout():
    rng = np.random.default_rng(5)
    for rows, K in ((128, 128), (384, 640), (256, 8192)):
        src = rng.integers(0, 256, size=(rows, K // 32), dtype=np.uint8)
        s_dev = torch.from_numpy(src).cuda()
        d_dev = torch.empty_like(s_dev)
        M.moe_tile_scales(s_dev, rows, K, d_dev)
        torch.cuda.synchronize()
        tiles = [(0, 128 * t, 128, 0) for t in range(rows // 128)]
        np.testing.assert_array_equal(_untile(d_dev.cpu().numpy().ravel(), tiles, rows, K), src)
