"""GPU parity of the CUDA path against the fp64 oracle, stage by stage.

Each workload runs through the C ABI (route -> [latent_down] -> permute ->
expert_ffn -> combine, and the fused moe_layer) and is compared with the
oracle on the same seeded inputs:

* router logits within fp32 accumulation error; expert indices bit-exact
  except tokens the oracle flags as near-ties (|l_k - l_k+1| < 1e-5), whose
  GPU choice must be a valid top-k inside the tie window; weights to 2e-6;
* permutation arrays bit-exact (integer work, given the same indices);
* activation operand exact (bf16 -> f16 with a power-of-two row scale);
* expert outputs, shared expert and the layer output: max |err| <= 1e-2 x RMS.
"""
import dataclasses
import gc

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

from parity_harness import (TOL, DeviceRun, check_permutation, check_routing, check_x_op_f16,  # noqa: E402
                            expert_getter, layer_kw, max_rel_err, route_kw)

MEDIUM = synth.MoeWorkload("medium_ragged", T=70, H=640, I=384, E=6, k=3, I_shared=256, seed=77)
LATENT_SMALL = synth.MoeWorkload("latent_small", T=5, H=384, I=128, E=12, k=3, I_shared=128, L=256,
                                 seed=78)
# T >= 128: router and shared expert on the tcgen05 bf16 GEMM (E = 6 < 128 rows,
# I_shared = 384 = three 128-row tiles, H = 640 = two 256-row pairs + one tile)
WIDE = synth.MoeWorkload("wide_tc", T=260, H=640, I=256, E=6, k=2, I_shared=384, seed=79)
# one token with K multiples of 1024: router, sigmoid gate and shared expert on
# the whole-row CUDA-core GEMV (E = 10 router rows: the last stage holds two;
# the sigmoid-gate row is a segment of its own)
ROWS_T1 = synth.MoeWorkload("rows_t1", T=1, H=2048, I=256, E=10, k=3, I_shared=1024, seed=80)
# latent layers: one token on the row GEMV (the latent rows a third segment of
# the router launch), and T >= 128 on the tcgen05 GEMM (router rows, the
# sigmoid-gate row and the latent rows as three segments of one pass over x)
ROWS_LATENT_T1 = synth.MoeWorkload("rows_latent_t1", T=1, H=1024, I=128, E=12, k=3, I_shared=1024,
                                   L=256, seed=81)
WIDE_LATENT = synth.MoeWorkload("wide_latent", T=130, H=512, I=128, E=6, k=2, I_shared=256, L=384,
                                seed=82)
# W and I multiples of 512: experts with 2+ tokens on the TMA-ring tensor-core
# kernels; more than 16 tokens per expert (several passes over the weights),
# and a mix of single-token (CUDA-core) and multi-token experts
MMA_MANY = synth.MoeWorkload("mma_many", T=44, H=1024, I=512, E=6, k=2, I_shared=256, seed=83)
# one token with H off the row GEMV's lengths: router and shared expert on the
# tcgen05 GEMM (16-token tile), dispatch and operand from the top-k launch
TC_T1 = synth.MoeWorkload("tc_t1", T=1, H=640, I=256, E=12, k=3, I_shared=384, seed=85)
MMA_MIXED = synth.MoeWorkload("mma_mixed", T=24, H=1024, I=512, E=40, k=2, I_shared=256, seed=84)
# router variants (rabbit README, model table row "MoE routing"): sigmoid scores
# with a selection bias and a weight scale ("noaux_tc sigmoid"), group-limited
# selection ("grouped routing") with sigmoid and with softmax scores, one token
# at full decode size (the top-k launch writes the dispatch), and 130 tokens
# (router on the tcgen05 GEMM)
NOAUX = synth.MoeWorkload("noaux_sigmoid", T=6, H=512, I=256, E=32, k=4, I_shared=128, seed=86,
                          score_fn=1, bias_std=0.05, route_scale=2.5)
GROUPED = synth.MoeWorkload("grouped_sigmoid", T=5, H=512, I=256, E=64, k=6, I_shared=128, seed=87,
                            score_fn=1, n_group=8, topk_group=4, bias_std=0.02)
GROUPED_SM = synth.MoeWorkload("grouped_softmax", T=9, H=512, I=256, E=48, k=4, I_shared=128,
                               seed=88, n_group=6, topk_group=2)
GROUPED_WIDE = synth.MoeWorkload("grouped_wide", T=130, H=512, I=128, E=64, k=4, I_shared=256,
                                 seed=89, n_group=4, topk_group=2, score_fn=1, bias_std=0.03)
DECODE1_GROUPED = synth.MoeWorkload("decode1_grouped", T=1, H=8192, I=2048, E=512, k=10,
                                    I_shared=2048, seed=90, score_fn=1, n_group=8, topk_group=4,
                                    bias_std=0.05, route_scale=2.5)

CASES = [
    (synth.WORKLOADS["tiny"], None),
    (MEDIUM, None),
    (LATENT_SMALL, None),
    (WIDE, None),
    (ROWS_T1, None),
    (ROWS_LATENT_T1, None),
    (WIDE_LATENT, None),
    (MMA_MANY, None),
    (MMA_MIXED, None),
    (TC_T1, None),
    (synth.WORKLOADS["latent16"], None),
    (synth.WORKLOADS["decode1"], None),
    (synth.WORKLOADS["decode32"], None),
    (NOAUX, None),
    (GROUPED, None),
    (GROUPED_SM, None),
    (GROUPED_WIDE, None),
    (DECODE1_GROUPED, None),
]


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def _read_layer(run):
    """Outputs of the fused moe_layer path (a second run on the same buffers)."""
    y = run.run_layer()
    L = run.layer
    out = dict(y=y, idx=L.topk_idx.cpu().numpy(), w=L.topk_w.cpu().numpy().astype(np.float64),
               expert_list=L.expert_list.cpu().numpy(), x_op=L.x_op.cpu().numpy())
    for n in ("counts", "offsets", "row_token", "row_slot", "slot_row"):
        out[n] = getattr(L, n).cpu().numpy()
    return out


@pytest.fixture(scope="module", params=CASES, ids=lambda c: c[0].name)
def case(request):
    w, sample = request.param
    run = DeviceRun(w)
    gpu = run.run_stages()
    layer = _read_layer(run)
    yield w, sample, run, gpu, layer
    del run
    _free()


@pytest.fixture(scope="module")
def ref(case):
    """The oracle's layer on the sampled tokens (all tokens when sample is None),
    evaluated with the GPU's selection only where the oracle flags a near tie."""
    w, sample, run, gpu, layer = case
    d = run.dense
    tokens = np.arange(w.T) if sample is None else np.array(sample)
    sub = dict(d, x=d["x"][tokens])
    idx_o, _, flags = O.route(O.router_logits(sub["x"], d["w_router"]), w.k, **route_kw(w, d))
    tied = flags != 0
    override = np.where(tied[:, None], gpu["idx"][tokens], idx_o) if np.any(tied) else None
    return tokens, O.moe_layer(sub, w.k, expert_getter(w), idx_override=override,
                               **layer_kw(w, d))


def test_routing_and_permutation(case):
    w, sample, run, gpu, layer = case
    ref_logits = O.router_logits(run.dense["x"], run.dense["w_router"])
    check_routing(gpu, ref_logits, w.k, **route_kw(w, run.dense))
    check_permutation(gpu, w.E)


def test_activation_operand(case):
    w, sample, run, gpu, layer = case
    x_in = gpu["x_lat"] if w.L else run.dense["x"]
    check_x_op_f16(gpu["x_op"], x_in, w.T, w.W)


def test_latent_projection(case):
    w, sample, run, gpu, layer = case
    if not w.L:
        pytest.skip("not a latent layer")
    ref = O.latent_down(run.dense["x"], run.dense["w_lat_down"])
    a = gpu["x_lat"].astype(np.int32)
    b = ref.astype(np.int32)
    # both sides round to bf16; fp32 vs fp64 sums may straddle a rounding boundary
    assert np.max(np.abs(a - b)) <= 1
    assert np.mean(a != b) < 0.01


def test_expert_rows(case, ref):
    """y_perm rows of every (token, slot) pair of the sampled tokens."""
    w, sample, run, gpu, layer = case
    tokens, r = ref
    got = gpu["y_perm"][gpu["slot_row"][tokens].ravel()]
    want = r["y_perm"][r["slot_row"].ravel()]
    err, rms = max_rel_err(got, want)
    assert err <= TOL, (err, rms)


def test_shared_expert_alone(case):
    w, sample, run, gpu, layer = case
    d = run.dense
    ref, _ = O.shared_expert(d["x"], d["ws_gate"], d["ws_up"], d["ws_down"], d["w_sgate"])
    if w.L:
        pytest.skip("latent layers add the up-projection of the routed sum before the shared part")
    got = run.shared_only()
    err, rms = max_rel_err(got, ref)
    assert err <= TOL, (err, rms)


def test_layer_output(case, ref):
    """Both the step calls and the fused moe_layer path against the oracle."""
    w, sample, run, gpu, layer = case
    tokens, r = ref
    for name, y in (("stages", gpu["y"]), ("moe_layer", layer["y"])):
        err, rms = max_rel_err(y[tokens], r["y"])
        assert err <= TOL, (name, err, rms)


def test_fused_layer_routing_and_dispatch_against_oracle(case, ref):
    """The routing, dispatch and operand that moe_layer writes (for one token
    the top-k launch writes the dispatch and the f16 operand itself), checked
    against the oracle directly."""
    w, sample, run, gpu, layer = case
    tokens, r = ref
    tied = r["flags"] != 0
    np.testing.assert_array_equal(layer["idx"][tokens][~tied], r["idx"][~tied])
    np.testing.assert_array_equal(np.sort(layer["idx"][tokens], axis=1),
                                  np.sort(gpu["idx"][tokens], axis=1))
    check_permutation(layer, w.E)
    if not w.L:
        check_x_op_f16(layer["x_op"], run.dense["x"], w.T, w.W)


def test_layer_on_a_new_input_follows_its_own_routing(case):
    """moe_layer on x, then at once on another input (x with every sign
    flipped: other experts for every token), back to back on one stream: the
    second output must match the oracle for the second input. The routed
    expert kernels read the dispatch the routing chain writes in the same
    call; reading it before that launch has finished would reuse the first
    input's experts (the same buffers, valid but stale)."""
    w, sample, run, gpu, layer = case
    d = run.dense
    x2 = np.ascontiguousarray(d["x"] ^ np.uint16(0x8000))
    x2_dev = torch.from_numpy(x2.view(np.int16)).cuda()
    run.layer(run.dev["x"])
    y2 = run.layer(x2_dev)
    torch.cuda.synchronize()
    y2 = y2.cpu().numpy().astype(np.float64)
    idx2 = run.layer.topk_idx.cpu().numpy()
    tokens = np.arange(w.T) if sample is None else np.array(sample)
    sub = dict(d, x=x2[tokens])
    idx_o, _, flags = O.route(O.router_logits(sub["x"], d["w_router"]), w.k, **route_kw(w, d))
    tied = flags != 0
    assert not np.array_equal(np.sort(idx_o[~tied], axis=1), np.sort(gpu["idx"][tokens][~tied], axis=1))
    np.testing.assert_array_equal(idx2[tokens][~tied], idx_o[~tied])
    override = np.where(tied[:, None], idx2[tokens], idx_o) if np.any(tied) else None
    ref = O.moe_layer(sub, w.k, expert_getter(w), idx_override=override, **layer_kw(w, d))
    err, rms = max_rel_err(y2[tokens], ref["y"])
    assert err <= TOL, (err, rms)


def test_fused_layer_matches_stages_bitwise(case):
    w, sample, run, gpu, layer = case
    np.testing.assert_array_equal(layer["y"], gpu["y"])
    for name in ("idx", "counts", "offsets", "row_token", "row_slot", "slot_row", "x_op"):
        np.testing.assert_array_equal(layer[name], gpu[name], err_msg=name)
    n = int(gpu["expert_list"][0])
    np.testing.assert_array_equal(layer["expert_list"][:1 + n], gpu["expert_list"][:1 + n])
    np.testing.assert_array_equal(layer["w"], gpu["w"])
    y2 = run.run_layer()
    np.testing.assert_array_equal(y2, layer["y"])


# ---------------------------------------------------------------------------
# edge cases on small shapes
# ---------------------------------------------------------------------------

def _small(T=6, E=8, k=3, **kw):
    return synth.MoeWorkload("edge", T=T, H=256, I=128, E=E, k=k, I_shared=128, seed=91, **kw)


def test_zero_input_ties_go_to_lowest_index():
    w = _small()
    d = synth.dense_inputs(w)
    d["x"] = np.zeros_like(d["x"])
    run = DeviceRun(w, dense=d)
    gpu = run.run_stages()
    assert np.all(gpu["logits"] == 0)
    np.testing.assert_array_equal(gpu["idx"], np.tile(np.arange(w.k), (w.T, 1)))
    np.testing.assert_allclose(gpu["w"], 1.0 / w.k, rtol=1e-6)
    # x = 0: every expert output and the shared expert are exactly 0
    assert np.all(gpu["y"] == 0)


def test_all_experts_selected():
    w = _small(T=3, E=4, k=4)
    run = DeviceRun(w)
    gpu = run.run_stages()
    assert np.all(gpu["counts"] == 3)
    ref = O.moe_layer(run.dense, w.k, expert_getter(w))
    err, _ = max_rel_err(gpu["y"], ref["y"])
    assert err <= TOL


def test_single_token_single_expert():
    w = _small(T=1, E=1, k=1)
    run = DeviceRun(w)
    gpu = run.run_stages()
    ref = O.moe_layer(run.dense, 1, expert_getter(w))
    assert gpu["w"][0, 0] == 1.0
    err, _ = max_rel_err(gpu["y"], ref["y"])
    assert err <= TOL


def test_nan_scale_poisons_only_its_outputs():
    w = _small(T=4, E=2, k=1)
    run = DeviceRun(w)
    gpu0 = run.run_stages()
    e = int(gpu0["idx"][0, 0])
    # E8M0 code 255 (NaN) in one scale of one gate row of expert e
    run.dev["wg_s"][e, 5, 3] = 255
    gpu = run.run_stages()
    rows_e = gpu["row_token"][gpu["offsets"][e]:gpu["offsets"][e + 1]]
    for t in range(w.T):
        r = gpu["slot_row"][t, 0]
        if t in rows_e:
            assert np.all(np.isnan(gpu["y_perm"][r]))      # h[5] is NaN and feeds every output
        else:
            assert np.all(np.isfinite(gpu["y_perm"][r]))


def test_nan_scale_multi_token_kernels():
    """The same on the TMA-ring kernels of experts with 2+ tokens (W, I multiples
    of 512): a NaN down scale poisons one output column of its expert's rows, a
    NaN gate scale every output of them; the other expert stays finite."""
    w = synth.MoeWorkload("edge_mma", T=8, H=512, I=512, E=2, k=1, I_shared=128, seed=92)
    run = DeviceRun(w)
    gpu0 = run.run_stages()
    counts = np.diff(gpu0["offsets"][:w.E + 1])
    e = int(np.argmax(counts))
    assert counts[e] >= 2
    rows_e = set(range(int(gpu0["offsets"][e]), int(gpu0["offsets"][e + 1])))
    saved = run.dev["wd_s"][e, 7, 3].clone()
    run.dev["wd_s"][e, 7, 3] = 255
    gpu = run.run_stages()
    for r in range(w.T * w.k):
        if r in rows_e:
            assert np.isnan(gpu["y_perm"][r, 7])
            assert np.all(np.isfinite(np.delete(gpu["y_perm"][r], 7)))
        else:
            assert np.all(np.isfinite(gpu["y_perm"][r]))
    run.dev["wd_s"][e, 7, 3] = saved
    run.dev["wg_s"][e, 5, 3] = 255
    gpu = run.run_stages()
    for r in range(w.T * w.k):
        if r in rows_e:
            assert np.all(np.isnan(gpu["y_perm"][r]))
        else:
            assert np.all(np.isfinite(gpu["y_perm"][r]))


def test_invalid_expert_index_sets_status_and_empties_routing():
    import mxfp4_routed_expert_04_b200 as M
    w = _small(T=4, E=8, k=2)
    run = DeviceRun(w)
    L = run.layer
    M.moe_workspace_init(run.dims, L.ws)
    bad = torch.tensor([[0, 1], [2, 8], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")
    M.moe_permute(run.dims, bad, run.dev["x"], L.counts, L.offsets, L.expert_list, L.row_token,
                  L.row_slot, L.slot_row, L.x_op, L.ws)
    assert M.moe_device_status(L.ws) & 1
    assert int(L.counts.sum()) == 0 and int(L.offsets.abs().sum()) == 0
    assert int(L.expert_list[0]) == 0
    M.moe_workspace_init(run.dims, L.ws)
    rep = torch.tensor([[0, 1], [2, 2], [3, 4], [5, 6]], dtype=torch.int32, device="cuda")
    M.moe_permute(run.dims, rep, run.dev["x"], L.counts, L.offsets, L.expert_list, L.row_token,
                  L.row_slot, L.slot_row, L.x_op, L.ws)
    assert M.moe_device_status(L.ws) & 2
    M.moe_workspace_init(run.dims, L.ws)
    assert M.moe_device_status(L.ws) == 0


def test_bounded_wait_gives_up_and_sets_the_status_bit():
    """A stage whose bytes never arrive: the bounded waits (the ones every
    stage-ring kernel uses) give up after their limit, the kernel returns, the
    status word gets STATUS_WAIT_TIMEOUT, and the context stays usable. The
    same kernel with the stage delivered leaves the word clear."""
    import mxfp4_routed_expert_04_b200 as M
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    src = torch.arange(512, dtype=torch.int32, device="cuda").to(torch.uint8)
    M.moe_selftest_bounded_wait(status, src, True, 256)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    M.moe_selftest_bounded_wait(status, None, False, 64)
    torch.cuda.synchronize()
    assert int(status[0]) == M.STATUS_WAIT_TIMEOUT
    # the context still works: a normal small layer runs and matches the oracle
    w = _small(T=2, E=4, k=2)
    run = DeviceRun(w)
    gpu = run.run_stages()
    ref = O.moe_layer(run.dense, w.k, expert_getter(w))
    err, _ = max_rel_err(gpu["y"], ref["y"])
    assert err <= TOL


def test_router_variant_selection_differs_from_softmax():
    """The variant cases really exercise other selections: the biased and
    group-limited routers pick other experts than plain softmax top-k on the
    same logits for some tokens (so a kernel ignoring the variant fails)."""
    for w in (NOAUX, GROUPED, GROUPED_SM):
        d = synth.dense_inputs(w)
        lg = O.router_logits(d["x"], d["w_router"])
        plain = O.route(lg, w.k)[0]
        var = O.route(lg, w.k, **route_kw(w, d))[0]
        assert not np.array_equal(np.sort(plain, axis=1), np.sort(var, axis=1)), w.name


def test_one_token_launch_clears_its_counters():
    """One token runs both expert projections in one launch whose roles hand
    h over through per-expert counters in the workspace's status region; the
    last CTA puts them back to zero. Calls in a row (different inputs, the
    stage calls and the fused layer) each match the oracle, leave the status
    word clear and the counters at zero, and a repeated input gives the same
    bits."""
    import mxfp4_routed_expert_04_b200 as M
    w = ROWS_T1
    run = DeviceRun(w)
    L = run.layer
    # every counter of the launch: 3 + k_max (32) words from word 16
    counters = slice(64, 64 + 4 * 35)
    first = None
    for i in range(3):
        d = dict(run.dense)
        if i:       # another token (other experts), the same weights
            d["x"] = synth.dense_inputs(dataclasses.replace(w, seed=w.seed + 7 * i))["x"]
        run.dev["x"].copy_(torch.from_numpy(d["x"].view(np.int16)).cuda())
        gpu = run.run_stages()
        assert M.moe_device_status(L.ws) == 0
        assert not L.ws[counters].any()
        tie = np.any(O.route(O.router_logits(d["x"], d["w_router"]), w.k)[2])
        ref = O.moe_layer(d, w.k, expert_getter(w), idx_override=gpu["idx"] if tie else None)
        err, _ = max_rel_err(gpu["y"], ref["y"])
        assert err <= TOL, (i, err)
        y_layer = run.run_layer()
        assert not L.ws[counters].any()
        np.testing.assert_array_equal(y_layer, gpu["y"])
        if i == 0:
            first = gpu["y_perm"]
    run.dev["x"].copy_(torch.from_numpy(run.dense["x"].view(np.int16)).cuda())
    np.testing.assert_array_equal(run.run_stages()["y_perm"], first)


def test_one_token_thirty_two_experts():
    """The one-launch routed path at its largest k (32 experts of one token)."""
    w = _small(T=1, E=40, k=32)
    run = DeviceRun(w)
    gpu = run.run_stages()
    ref = O.moe_layer(run.dense, w.k, expert_getter(w), idx_override=gpu["idx"])
    assert int(gpu["expert_list"][0]) == 32
    err, _ = max_rel_err(gpu["y_perm"][gpu["slot_row"][0]], ref["y_perm"][ref["slot_row"][0]])
    assert err <= TOL, err
    err, _ = max_rel_err(gpu["y"], ref["y"])
    assert err <= TOL, err
    assert M_status(run) == 0


def M_status(run):
    import mxfp4_routed_expert_04_b200 as M
    return M.moe_device_status(run.layer.ws)


def test_one_token_emptied_dispatch_then_a_normal_call():
    """An invalid expert index empties the one-token dispatch; the one-launch
    routed call on it streams nothing and leaves its counters at zero, and
    the next call on a valid dispatch matches the oracle."""
    import mxfp4_routed_expert_04_b200 as M
    w = _small(T=1, E=8, k=2)
    run = DeviceRun(w)
    L = run.layer
    bad = torch.tensor([[1, 8]], dtype=torch.int32, device="cuda")
    M.moe_permute(run.dims, bad, run.dev["x"], L.counts, L.offsets, L.expert_list, L.row_token,
                  L.row_slot, L.slot_row, L.x_op, L.ws)
    assert int(L.expert_list[0]) == 0
    lw = L.w
    M.moe_expert_ffn(run.dims, L.x_op, L.offsets, L.expert_list, L.row_token, lw["wg_q"], lw["wg_s"],
                     lw["wu_q"], lw["wu_s"], lw["wd_q"], lw["wd_s"], L.y_perm, L.ws)
    torch.cuda.synchronize()
    assert M.moe_device_status(L.ws) & M.STATUS_BAD_EXPERT
    M.moe_workspace_init(run.dims, L.ws)
    gpu = run.run_stages()
    assert M.moe_device_status(L.ws) == 0
    ref = O.moe_layer(run.dense, w.k, expert_getter(w), idx_override=gpu["idx"])
    err, _ = max_rel_err(gpu["y"], ref["y"])
    assert err <= TOL, err
