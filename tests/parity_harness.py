"""Shared helpers of the GPU parity tests: run the layer through the C ABI and
evaluate the fp64 oracle on the same seeded inputs (never on GPU outputs,
except where a test says it evaluates the oracle on the GPU's own routing
choice for a near-tie token)."""
from __future__ import annotations

import numpy as np
import torch

import mxfp4_routed_expert_04_b200 as M
import oracle as O
import synth

TOL = 1e-2            # max |gpu - oracle| <= TOL * RMS(oracle), per output tensor
NEAR_TIE = 1e-5


class DeviceRun:
    """Uploads a workload, runs it stage by stage, keeps host copies of every output."""

    def __init__(self, w: synth.MoeWorkload, act_mode=M.ACT_BF16, dense=None):
        self.w = w
        self.dense = synth.dense_inputs(w) if dense is None else dense
        self.dev = synth.to_device(w, self.dense)
        self.dims = M.MoeDims.of(w, act_mode)
        self.layer = M.MoeLayer(self.dims, {k: v for k, v in self.dev.items() if k != "x"})

    def run_stages(self):
        y = self.layer.stages(self.dev["x"])
        torch.cuda.synchronize()
        L = self.layer
        out = dict(
            logits=L.logits.cpu().numpy().astype(np.float64),
            idx=L.topk_idx.cpu().numpy(), w=L.topk_w.cpu().numpy().astype(np.float64),
            counts=L.counts.cpu().numpy(), offsets=L.offsets.cpu().numpy(),
            expert_list=L.expert_list.cpu().numpy(),
            row_token=L.row_token.cpu().numpy(), row_slot=L.row_slot.cpu().numpy(),
            slot_row=L.slot_row.cpu().numpy(), y_perm=L.y_perm.cpu().numpy().astype(np.float64),
            y=y.cpu().numpy().astype(np.float64), x_op=L.x_op.cpu().numpy())
        if L.x_lat is not None:
            out["x_lat"] = L.x_lat.cpu().numpy().view(np.uint16)
        return out

    def run_layer(self):
        y = self.layer(self.dev["x"])
        torch.cuda.synchronize()
        return y.cpu().numpy().astype(np.float64)

    def shared_only(self):
        """moe_combine on an all-zero routed buffer: the gated shared expert alone."""
        L = self.layer
        L.y_perm.zero_()
        d = self.dev
        M.moe_combine(self.dims, L.y_perm, L.slot_row, L.topk_w, d["x"], d["w_sgate"], d["ws_gate"],
                      d["ws_up"], d["ws_down"], d.get("w_lat_up"), L.y, L.ws)
        torch.cuda.synchronize()
        return L.y.cpu().numpy().astype(np.float64)


def expert_getter(w):
    """e -> the six MXFP4 arrays of expert e, regenerated from the seed on each
    call (nothing cached: full-size layers hold gigabytes of experts)."""
    (Ng, Kg), (Nd, Kd) = synth.expert_shapes(w)

    def get(e):
        e = int(e)
        return (synth.expert_matrix(w.seed, "gate", e, Ng, Kg)
                + synth.expert_matrix(w.seed, "up", e, Ng, Kg)
                + synth.expert_matrix(w.seed, "down", e, Nd, Kd))
    return get


def route_kw(w, dense):
    """The oracle's router configuration of a workload (score function,
    selection bias, groups, weight scale), for O.route / check_routing."""
    return dict(score_fn=w.score_fn, bias=dense.get("e_bias"), n_group=max(1, w.n_group),
                topk_group=max(1, w.topk_group), scale=w.route_scale)


def layer_kw(w, dense):
    """The same configuration in O.moe_layer's keyword names."""
    r = route_kw(w, dense)
    return dict(score_fn=r["score_fn"], e_bias=r["bias"], n_group=r["n_group"],
                topk_group=r["topk_group"], route_scale=r["scale"])


def max_rel_err(got, want):
    rms = float(np.sqrt(np.mean(np.square(want))))
    return float(np.max(np.abs(got - want))) / rms, rms


def check_routing(gpu, ref_logits, k, near_tie=NEAR_TIE, **route_kw):
    """Compare the GPU router against the oracle; returns the tokens whose
    selected SET is a near tie (the k-th and (k+1)-th selection scores, or the
    last kept and first dropped group scores, closer than near_tie), where the
    GPU's choice is checked for validity instead and used as the reference.

    Elsewhere the set is bit-exact; the slot order is bit-exact too unless two
    selected scores are a near tie (then it must be a valid order). Weights
    are compared with the weights of the GPU's own selection, within a bound
    derived from the logit error."""
    idx, w, flags = O.route(ref_logits, k, near_tie=near_tie, **route_kw)
    set_tie = (flags & (O.TIE_SET | O.TIE_GROUP)) != 0
    order_tie = (flags & O.TIE_ORDER) != 0
    scale = max(1.0, float(np.abs(ref_logits).max()))
    assert np.max(np.abs(gpu["logits"] - ref_logits)) <= 1e-5 * scale * 10
    ok = ~set_tie
    g_idx = gpu["idx"]
    np.testing.assert_array_equal(np.sort(g_idx[ok], axis=1), np.sort(idx[ok], axis=1))
    exact = ok & ~order_tie
    np.testing.assert_array_equal(g_idx[exact], idx[exact])
    assert np.all([len(set(r)) == k for r in g_idx])
    # selection scores of the oracle, to check the validity of tied choices
    sel_score = ref_logits if route_kw.get("score_fn", O.SOFTMAX) == O.SOFTMAX else \
        O.sigmoid(ref_logits) + (0.0 if route_kw.get("bias") is None else route_kw["bias"])
    for t in np.nonzero(order_tie & ok)[0]:
        s = sel_score[t, g_idx[t]]
        assert np.all(np.diff(s) <= near_tie), (t, s)
    for t in np.nonzero(set_tie & ((flags & O.TIE_GROUP) == 0))[0]:
        s = sel_score[t, g_idx[t]]
        kth = np.sort(sel_score[t])[::-1][k - 1]
        assert np.all(s >= kth - near_tie)
    # weights of the GPU's selection under the oracle's rule:
    # d log w_j / d l_i = [i == j] c_j - w_i c_i with 0 <= c <= 1 (softmax:
    # c = 1; sigmoid: c = 1 - s), so |log w_gpu - log w| <= 2 max_sel |dl|
    # (+ fp32 rounding of exp and divide)
    w_sel = O.route(ref_logits, k, near_tie=near_tie, idx_in=g_idx, **route_kw)[1]
    dl = np.abs(np.take_along_axis(gpu["logits"] - ref_logits, g_idx.astype(np.int64), axis=1))
    bound = np.abs(w_sel) * (np.expm1(2 * dl.max(axis=1, keepdims=True)) + 1e-6) + 1e-9
    assert np.all(np.abs(gpu["w"] - w_sel) <= bound)
    np.testing.assert_allclose(gpu["w"].sum(axis=1), route_kw.get("scale", 1.0), rtol=1e-6)
    return set_tie


def check_permutation(gpu, E):
    counts, offsets, row_token, row_slot, slot_row = O.permute(gpu["idx"], E)
    np.testing.assert_array_equal(gpu["counts"], counts)
    np.testing.assert_array_equal(gpu["offsets"], offsets)
    np.testing.assert_array_equal(gpu["row_token"], row_token)
    np.testing.assert_array_equal(gpu["row_slot"], row_slot)
    np.testing.assert_array_equal(gpu["slot_row"], slot_row)
    active = np.nonzero(counts)[0]
    assert gpu["expert_list"][0] == len(active)
    np.testing.assert_array_equal(gpu["expert_list"][1:1 + len(active)], active)


def check_x_op_f16(x_op, x_bits, T, W):
    """MOE_ACT_BF16 operand: f16 rows x power-of-two row scale reproduce x exactly."""
    v = x_op[:T * W * 2].view(np.float16).reshape(T, W).astype(np.float64)
    off = (T * W * 2 + 255) // 256 * 256
    sc = x_op[off:off + 4 * T].view(np.float32).astype(np.float64)
    x = O.bf16_to_f64(x_bits)
    got = v * sc[:, None]
    big = np.abs(x) >= np.abs(x).max(axis=1, keepdims=True) * 2.0 ** -29
    np.testing.assert_array_equal(got[big], x[big])
    assert np.all(np.log2(sc) == np.round(np.log2(sc)))
