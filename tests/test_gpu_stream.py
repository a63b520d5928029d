"""Routed experts streamed from host memory through the LRU expert cache
(moe_expert_ffn_streamed): the same kernels as the resident path on the same
dispatch, so the expert rows must be bit-identical to moe_expert_ffn's; the
layer built on them is checked against the fp64 oracle. Several inputs in a
row route to different experts, so slots are evicted and reused, and a
repeated input finds every expert cached."""
import dataclasses

import numpy as np
import pytest
import torch

import mxfp4_routed_expert_04_b200 as M
import oracle as O
import synth
from parity_harness import TOL, DeviceRun, expert_getter, max_rel_err

pytestmark = pytest.mark.gpu

# W = 2048, I = 512: single-token experts on the CUDA-core GEMVs and experts
# with 2+ tokens on the TMA-ring kernels, each run as a one-expert problem
STREAM = synth.MoeWorkload("stream", T=6, H=2048, I=512, E=24, k=3, I_shared=256, seed=95)


def _host_experts(w):
    ex = synth.expert_weights(w, range(w.E))
    names = ("wg_q", "wg_s", "wu_q", "wu_s", "wd_q", "wd_s")
    return [tuple(torch.from_numpy(np.ascontiguousarray(ex[n][e])).pin_memory() for n in names)
            for e in range(w.E)]


def _inputs(w, i):
    """Input i: token rows drawn from another seed (other experts)."""
    d = synth.dense_inputs(w)
    if i:
        d["x"] = synth.dense_inputs(dataclasses.replace(w, seed=w.seed + 100 * i))["x"]
    return d


def test_streamed_experts_match_resident_and_oracle():
    w = STREAM
    run = DeviceRun(w)
    L = run.layer
    cache = M.ExpertCache(L.dims, slots=w.T * w.k, host_experts=_host_experts(w))
    try:
        seen = []
        for i in (0, 1, 2, 0):
            d = _inputs(w, i)
            x = torch.from_numpy(d["x"].view(np.int16)).cuda()
            run.dev["x"].copy_(x)
            gpu = run.run_stages()                           # resident path (moe_expert_ffn)
            n = int(gpu["expert_list"][0])
            active = [int(e) for e in gpu["expert_list"][1:1 + n]]
            # streamed path on the same dispatch and activation operand
            L.y_perm.fill_(float("nan"))
            before = cache.stats()
            cache.ffn(active, L.x_op, L.offsets, L.row_token, L.y_perm, L.ws)
            torch.cuda.synchronize()
            after = cache.stats()
            y_perm = L.y_perm.cpu().numpy().astype(np.float64)
            np.testing.assert_array_equal(y_perm, gpu["y_perm"])
            hits = after["hits"] - before["hits"]
            misses = after["misses"] - before["misses"]
            assert hits + misses == n
            seen.append(set(active))
            # the layer from the streamed rows against the oracle
            M.moe_combine(L.dims, L.y_perm, L.slot_row, L.topk_w, run.dev["x"], run.dev["w_sgate"],
                          run.dev["ws_gate"], run.dev["ws_up"], run.dev["ws_down"], None, L.y, L.ws)
            torch.cuda.synchronize()
            ref = O.moe_layer(d, w.k, expert_getter(w),
                              idx_override=gpu["idx"] if np.any(O.route(
                                  O.router_logits(d["x"], d["w_router"]), w.k)[2]) else None)
            err, rms = max_rel_err(L.y.cpu().numpy().astype(np.float64), ref["y"])
            assert err <= TOL, (i, err, rms)
        st = cache.stats()
        assert st["misses"] > len(seen[0])                   # later inputs needed other experts
        assert st["bytes_copied"] == st["misses"] * 3 * (w.I * w.W // 2 + w.I * w.W // 32)
    finally:
        cache.close()


def test_repeated_call_hits_every_expert():
    w = STREAM
    run = DeviceRun(w)
    L = run.layer
    cache = M.ExpertCache(L.dims, slots=w.T * w.k, host_experts=_host_experts(w))
    try:
        gpu = run.run_stages()
        n = int(gpu["expert_list"][0])
        active = [int(e) for e in gpu["expert_list"][1:1 + n]]
        cache.ffn(active, L.x_op, L.offsets, L.row_token, L.y_perm, L.ws)
        first = cache.stats()
        cache.ffn(active, L.x_op, L.offsets, L.row_token, L.y_perm, L.ws)
        torch.cuda.synchronize()
        second = cache.stats()
        assert first["misses"] == n and first["hits"] == 0
        assert second["hits"] - first["hits"] == n and second["misses"] == n
        np.testing.assert_array_equal(L.y_perm.cpu().numpy().astype(np.float64), gpu["y_perm"])
    finally:
        cache.close()


def test_cache_rejects_more_active_experts_than_slots():
    w = STREAM
    run = DeviceRun(w)
    L = run.layer
    cache = M.ExpertCache(L.dims, slots=2, host_experts=_host_experts(w))
    try:
        with pytest.raises(M.MoeError):
            cache.ffn([0, 1, 2], L.x_op, L.offsets, L.row_token, L.y_perm, L.ws)
    finally:
        cache.close()
