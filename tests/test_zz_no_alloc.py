"""moe_route_noalloc: the router for callers that cannot hand the library any
device scratch memory (for example a plug-in that only receives its input and
output tensors). Its split-K partial sums live in a device array built into
the library instead of a caller workspace. Checked through the C ABI against
moe_route on the same inputs, twice in a row (the shared array keeps the
previous call's contents, which must not leak into the next result).

This file is collected last on purpose: it also has to pass after every other
test has run in the same process."""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_routed_expert_04_b200 as M
from mxfp4_routed_expert_04_b200 import synth

pytestmark = pytest.mark.gpu

NEAR_TIE = 1e-5


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


@pytest.mark.parametrize("name", ["tiny", "decode32", "latent16"])
def test_noalloc_route_matches_workspace_route_twice(name):
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
    srt = -np.sort(-lg, axis=1)
    ok = (srt[:, w.k - 1] - srt[:, w.k]) >= NEAR_TIE      # tokens whose top-k set is not a near tie
    for _ in range(2):
        idx = torch.full((w.T, w.k), -1, dtype=torch.int32, device="cuda")
        wt = torch.full((w.T, w.k), -1.0, dtype=torch.float32, device="cuda")
        lgt = torch.full((w.T, w.E), float("nan"), dtype=torch.float32, device="cuda")
        M.moe_route_noalloc(dims, x, wr, idx, wt, lgt)
        torch.cuda.synchronize()
        scale = max(1.0, float(np.abs(lg).max()))
        assert np.max(np.abs(lgt.cpu().numpy() - lg)) <= 1e-4 * scale
        np.testing.assert_array_equal(idx.cpu().numpy()[ok], idx_ref.cpu().numpy()[ok])
        np.testing.assert_allclose(wt.cpu().numpy()[ok], w_ref.cpu().numpy()[ok], rtol=0, atol=2e-6)


def test_noalloc_route_rejects_shapes_beyond_its_scratch():
    # T=4096, E=512: the partial sums need 8 MiB > 4 MiB; rejected before any launch
    w = synth.WORKLOADS["prefill4096"]
    dims = M.MoeDims.of(w)
    fake = 1 << 20
    st = M._lib.moe_route_noalloc(ctypes.byref(dims), fake, fake, fake, fake, None, None)
    assert st == 2
    assert "4 MiB" in M._lib.moe_last_error().decode()
