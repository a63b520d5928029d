"""moe_route_noalloc: the router for callers that cannot hand the library any
device scratch memory (for example a plug-in that only receives its input and
output tensors). Its split-K partial sums live in a device array built into
the library instead of a caller workspace.

Checked through the C ABI, twice in a row (the shared array keeps the previous
call's contents, which must not leak into the next result):
* against the fp64 oracle, with the same rules as every router test
  (selected set bit-exact except near ties, weights within the bound derived
  from the logit error);
* against moe_route on the same inputs: logits within the tolerance the
  router tests use (its logits come from another kernel, summed in another
  order), the same selected set wherever moe_route's own logits are not a near
  tie, the same slot order where two selected logits are not a near tie;
* the two calls give the same bits.

This file is collected last on purpose: it also has to pass after every other
test has run in the same process."""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_routed_expert_04_b200 as M
import oracle as O
import synth
from parity_harness import NEAR_TIE, check_routing

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def _near_ties(lg, k):
    """(set tie, order tie) of each token from a logits matrix."""
    srt = -np.sort(-lg, axis=1)
    set_tie = (srt[:, k - 1] - srt[:, k]) < NEAR_TIE if k < lg.shape[1] else np.zeros(len(lg), bool)
    order_tie = np.any(srt[:, :k - 1] - srt[:, 1:k] < NEAR_TIE, axis=1) if k > 1 else \
        np.zeros(len(lg), bool)
    return set_tie, order_tie


@pytest.mark.parametrize("name", ["tiny", "decode1", "decode32", "latent16"])
def test_noalloc_route_against_oracle_and_workspace_route_twice(name):
    w = synth.WORKLOADS[name]
    d = synth.dense_inputs(w)
    x, wr = _dev(d["x"]), _dev(d["w_router"])
    dims = M.MoeDims.of(w)
    ws = torch.empty(M.moe_workspace_size(dims), dtype=torch.uint8, device="cuda")
    M.moe_workspace_init(dims, ws)
    idx_ref = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    w_ref = torch.empty(w.T, w.k, dtype=torch.float32, device="cuda")
    lg_ref = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    M.moe_route(dims, x, wr, idx_ref, w_ref, lg_ref, ws)
    torch.cuda.synchronize()
    lg = lg_ref.cpu().numpy().astype(np.float64)
    set_tie, order_tie = _near_ties(lg, w.k)
    oracle_logits = O.router_logits(d["x"], d["w_router"])
    outs = []
    for _ in range(2):
        idx = torch.full((w.T, w.k), -1, dtype=torch.int32, device="cuda")
        wt = torch.full((w.T, w.k), -1.0, dtype=torch.float32, device="cuda")
        lgt = torch.full((w.T, w.E), float("nan"), dtype=torch.float32, device="cuda")
        M.moe_route_noalloc(dims, x, wr, idx, wt, lgt)
        torch.cuda.synchronize()
        got = dict(idx=idx.cpu().numpy(), w=wt.cpu().numpy().astype(np.float64),
                   logits=lgt.cpu().numpy().astype(np.float64))
        check_routing(got, oracle_logits, w.k)
        scale = max(1.0, float(np.abs(lg).max()))
        assert np.max(np.abs(got["logits"] - lg)) <= 1e-4 * scale
        ok = ~set_tie
        ir = idx_ref.cpu().numpy()
        np.testing.assert_array_equal(np.sort(got["idx"][ok], axis=1), np.sort(ir[ok], axis=1))
        exact = ok & ~order_tie
        np.testing.assert_array_equal(got["idx"][exact], ir[exact])
        np.testing.assert_allclose(got["w"][exact], w_ref.cpu().numpy()[exact], rtol=0,
                                   atol=2e-6)
        outs.append(got)
    for n in ("idx", "w", "logits"):
        np.testing.assert_array_equal(outs[0][n], outs[1][n])


def test_noalloc_route_rejects_shapes_beyond_its_scratch():
    # T=4096, E=512: the partial sums need 8 MiB > 4 MiB; rejected before any launch
    w = synth.WORKLOADS["prefill4096"]
    dims = M.MoeDims.of(w)
    fake = 1 << 20
    st = M._lib.moe_route_noalloc(ctypes.byref(dims), fake, fake, fake, fake, None, None)
    assert st == 2
    assert "4 MiB" in M._lib.moe_last_error().decode()
