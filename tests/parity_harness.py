"""Shared helpers of the GPU parity tests: run the layer through the C ABI and
evaluate the fp64 oracle on the same seeded inputs (never on GPU outputs,
except where a test says it evaluates the oracle on the GPU's own routing
choice for a near-tie token)."""
from __future__ import annotations

import functools

import numpy as np
import torch

import mxfp4_routed_expert_04_b200 as M
import oracle as O
from mxfp4_routed_expert_04_b200 import synth

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


@functools.lru_cache(maxsize=None)
def _expert_cached(w, e):
    (Ng, Kg), (Nd, Kd) = synth.expert_shapes(w)
    g = synth.expert_matrix(w.seed, "gate", e, Ng, Kg)
    u = synth.expert_matrix(w.seed, "up", e, Ng, Kg)
    d = synth.expert_matrix(w.seed, "down", e, Nd, Kd)
    return g + u + d


def expert_getter(w):
    return lambda e: _expert_cached(w, int(e))


def max_rel_err(got, want):
    rms = float(np.sqrt(np.mean(np.square(want))))
    return float(np.max(np.abs(got - want))) / rms, rms


def check_routing(gpu, ref_logits, k, near_tie=NEAR_TIE):
    """Compare the GPU router against the oracle; returns the oracle's near-tie flags."""
    idx, w, flagged = O.topk_route(ref_logits, k, near_tie)
    scale = max(1.0, float(np.abs(ref_logits).max()))
    assert np.max(np.abs(gpu["logits"] - ref_logits)) <= 1e-5 * scale * 10
    ok = ~flagged
    np.testing.assert_array_equal(gpu["idx"][ok], idx[ok])
    # w_j = exp(l_j - m) / sum_sel exp(l - m): d log w_j / d l_i = [i == j] - w_i, so
    # |log w_gpu - log w| <= 2 max_sel |l_gpu - l| (+ fp32 rounding of exp and divide)
    dl = np.abs(np.take_along_axis(gpu["logits"] - ref_logits, idx.astype(np.int64), axis=1))
    bound = w * (np.expm1(2 * dl.max(axis=1, keepdims=True)) + 1e-6) + 1e-9
    assert np.all(np.abs(gpu["w"][ok] - w[ok]) <= bound[ok])
    # near-tie tokens: the GPU choice must be a valid top-k within the tie window
    for t in np.nonzero(flagged)[0]:
        sel = ref_logits[t, gpu["idx"][t]]
        kth = np.sort(ref_logits[t])[::-1][k - 1]
        assert np.all(sel >= kth - near_tie) and len(set(gpu["idx"][t])) == k
    np.testing.assert_allclose(gpu["w"].sum(axis=1), 1.0, atol=1e-6)
    return flagged


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
