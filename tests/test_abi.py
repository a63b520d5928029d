"""Host-side checks of the C ABI: the library loads, exports every entry point
the header declares, and rejects bad arguments synchronously (before any CUDA
call). None of these calls reaches a kernel launch: every case fails one
host-side check, so they are safe with or without a GPU."""
import ctypes
import os
import re

import pytest

import mxfp4_routed_expert_04_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_mxfp4.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(moe_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_function():
    names = _declared_functions()
    assert len(names) >= 12, names
    lib = ctypes.CDLL(M.library_path())
    for n in names:
        assert hasattr(lib, n), n


def _dims(**kw):
    base = dict(T=4, H=256, I=128, E=16, k=2, I_shared=128, L=0, act_mode=0)
    base.update(kw)
    return M.MoeDims(**base)


@pytest.mark.parametrize("kw,field", [
    (dict(T=0), "T="), (dict(H=100), "H="), (dict(I=64), "I="), (dict(E=0), "E="),
    (dict(k=17), "k="), (dict(k=33, E=64), "k="), (dict(L=96), "L="), (dict(I_shared=0), "I_shared="),
    (dict(act_mode=7), "act_mode"), (dict(E=2048), "E="),
])
def test_invalid_dims_have_no_workspace(kw, field):
    assert M.moe_workspace_size(_dims(**kw)) == 0
    assert field in M._lib.moe_last_error().decode()


def test_valid_dims_workspace_grows_with_tokens():
    a = M.moe_workspace_size(_dims(T=4))
    b = M.moe_workspace_size(_dims(T=64))
    assert 0 < a < b and a % 256 == 0


FAKE = 1 << 20          # 16-byte aligned fake address; never dereferenced (validation fails first)


def _route(dims, x=FAKE, wr=FAKE, idx=FAKE, w=FAKE, logits=None, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = M.moe_workspace_size(dims)
    return M._lib.moe_route(ctypes.byref(dims), x, wr, idx, w, logits, ws, ws_bytes, None)


def test_null_pointer_is_invalid_arg():
    assert _route(_dims(), x=None) == 1
    assert "x is NULL" in M._lib.moe_last_error().decode()


def test_misaligned_pointer_is_alignment_error():
    assert _route(_dims(), wr=FAKE + 8) == 3
    assert "w_router" in M._lib.moe_last_error().decode()


def test_small_workspace_is_rejected():
    d = _dims()
    assert _route(d, ws_bytes=M.moe_workspace_size(d) - 256) == 4


def test_bad_shape_is_rejected_before_pointers():
    assert _route(_dims(H=200), x=None) == 2


def test_null_dims():
    assert M._lib.moe_route(None, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None) == 1


def test_latent_down_needs_latent_dims():
    d = _dims()
    st = M._lib.moe_latent_down(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE,
                                M.moe_workspace_size(d), None)
    assert st == 1


def test_combine_rejects_latent_weight_without_latent_width():
    d = _dims()
    st = M._lib.moe_combine(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                            FAKE, FAKE, FAKE, M.moe_workspace_size(d), None)
    assert st == 1


def test_status_strings():
    assert M.moe_status_string(0) == "ok"
    assert "workspace" in M.moe_status_string(4)
    assert M.moe_status_string(99) == "unknown status"


def test_x_op_size_by_mode():
    d0, d1 = _dims(act_mode=0), _dims(act_mode=1)
    # bf16 mode: f16 rows + row scales, one row per token (T=4, W=256)
    assert M.moe_x_op_size(d0) >= 4 * 256 * 2 + 16
    # mxfp4 mode: packed E2M1 + E8M0 scales, one row per permuted row (T*k = 8), + tile list
    assert M.moe_x_op_size(d1) >= 8 * 128 + 8 * 8 + 16


def test_mxf4_layout_only_for_mxfp4_activations():
    d0, d1 = _dims(act_mode=0), _dims(act_mode=1)
    with pytest.raises(M.MoeError, match="MOE_ACT_MXFP4"):
        M.moe_mxf4_layout_of(d0)
    lay = M.moe_mxf4_layout_of(d1)
    R, W, I = d1.T * d1.k, d1.H, d1.I
    assert lay.tile_rows == 112 and lay.max_tiles >= (R + lay.tile_rows - 1) // lay.tile_rows
    # x_op parts in order, 256-byte aligned, inside moe_x_op_size
    parts = [lay.x_codes, lay.x_scales, lay.tiles, lay.tile_base, lay.n_tiles]
    assert parts == sorted(parts) and all(o % 256 == 0 for o in parts)
    assert lay.x_scales >= R * W // 2
    assert lay.tiles >= lay.x_scales + lay.max_tiles * (W // 128) * 512
    assert lay.n_tiles + 4 <= M.moe_x_op_size(d1)
    # h regions inside the workspace, disjoint
    ws = M.moe_workspace_size(d1)
    hc, hs = (lay.h_codes, R * I // 2), (lay.h_scales, lay.max_tiles * (I // 128) * 512)
    assert hc[0] + hc[1] <= ws and hs[0] + hs[1] <= ws
    assert hc[0] + hc[1] <= hs[0] or hs[0] + hs[1] <= hc[0]


@pytest.mark.parametrize("rows,K", [(100, 256), (128, 96), (0, 128), (256, 130)])
def test_tile_scales_rejects_bad_shapes(rows, K):
    st = M._lib.moe_tile_scales(1 << 20, rows, K, 1 << 21, None)
    assert st == 2
    assert "multiples of 128" in M._lib.moe_last_error().decode()


def test_tile_scales_rejects_null_and_misaligned():
    assert M._lib.moe_tile_scales(None, 128, 128, 1 << 20, None) == 1
    assert M._lib.moe_tile_scales((1 << 20) + 4, 128, 128, 1 << 20, None) == 3


def test_selftest_bounded_wait_validates_arguments():
    lib = M._lib
    assert lib.moe_selftest_bounded_wait(None, None, 0, 16, None) == 1          # no status word
    assert lib.moe_selftest_bounded_wait(FAKE, None, 1, 16, None) == 3          # deliver, no source
    assert lib.moe_selftest_bounded_wait(FAKE, FAKE + 4, 1, 16, None) == 3      # misaligned source
    assert lib.moe_selftest_bounded_wait(FAKE, None, 0, 0, None) == 1           # limit 0
    assert lib.moe_selftest_bounded_wait(FAKE, None, 0, 5000, None) == 1        # limit too large


def test_expert_cache_validates_arguments():
    d = _dims()
    assert M.moe_expert_cache_bytes(d, 0) == 0
    assert M.moe_expert_cache_bytes(_dims(T=0), 4) == 0
    n = M.moe_expert_cache_bytes(d, 4)
    assert n > 4 * 3 * (128 * 256 // 2) and n % 256 == 0
    out = ctypes.c_void_p()
    lib = M._lib
    assert lib.moe_expert_cache_create(ctypes.byref(d), 4, None, n, ctypes.byref(out)) == 1
    assert lib.moe_expert_cache_create(ctypes.byref(d), 4, FAKE + 16, n, ctypes.byref(out)) == 3
    assert lib.moe_expert_cache_create(ctypes.byref(d), 4, FAKE, n - 1, ctypes.byref(out)) == 4
    assert lib.moe_expert_cache_create(ctypes.byref(_dims(act_mode=1)), 4, FAKE, n,
                                       ctypes.byref(out)) == 2
    assert lib.moe_expert_ffn_streamed(None, ctypes.byref(d), None, 0, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       FAKE, M.moe_workspace_size(d), None) == 1
    assert lib.moe_expert_cache_destroy(None) == 0
