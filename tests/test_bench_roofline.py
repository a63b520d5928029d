"""The roofline arithmetic of bench.py, on CPU: the algorithmic bytes and
flops that its fractions divide by, checked against the same quantities
written out here from the workload shapes alone.

Counting rules (MXFP4 as in the OCP MX format: 32 E2M1 codes in 16 bytes plus
one E8M0 byte per 32 weights; bf16 weights 2 bytes): every weight is read
once, x comes in as bf16, y goes out as fp32; flops are 2 per multiply-add.
"""
import importlib.util
import os

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_roofline", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mxfp4(rows, cols):
    return rows * cols // 2 + rows * cols // 32


def test_one_expert_bytes():
    b = _bench()
    w = synth.WORKLOADS["decode1"]
    # gate and up [I, W], down [W, I]
    assert b.expert_bytes(w) == 3 * _mxfp4(2048, 8192) == 26_738_688
    lat = synth.WORKLOADS["latent16"]
    # routed experts at the latent width L = 2048 with I = 1024
    assert b.expert_bytes(lat) == 3 * _mxfp4(1024, 2048) == 3_342_336


def test_decode1_layer_bytes_and_flops():
    b = _bench()
    w = synth.WORKLOADS["decode1"]
    routed = 10 * 3 * _mxfp4(2048, 8192)
    shared = 3 * 2048 * 8192 * 2            # gate, up, down in bf16
    router = 512 * 8192 * 2 + 8192 * 2      # router rows and the sigmoid-gate row
    io = 8192 * 2 + 8192 * 4                # x in (bf16), y out (fp32)
    assert b.layer_bytes(w, 10) == routed + shared + router + io == 376_504_320
    # the routed call alone: the 10 experts, the token row, its fp32 output row
    assert b.ffn_bytes(w, 10) == routed + 8192 * 2 + 8192 * 4 == 267_436_032
    assert b.ffn_flops(w) == 2 * 10 * 3 * 2048 * 8192
    assert b.layer_flops(w) == 2 * (10 * 3 * 2048 * 8192 + 3 * 2048 * 8192 + 8192 + 512 * 8192)


def test_prefill_bytes_and_flops():
    b = _bench()
    w = synth.WORKLOADS["prefill4096"]
    pairs = 4096 * 10
    weights = 512 * 3 * _mxfp4(2048, 8192)
    x_op = _mxfp4(pairs, 8192)              # one MXFP4 activation row per (token, slot)
    y = 4096 * 8192 * 4
    assert b.ffn_bytes(w, 512, "mxfp4") == weights + x_op + y == 14_002_683_904
    assert b.ffn_flops(w) == 2 * pairs * 3 * 2048 * 8192 == 4_123_168_604_160
    # intermediates of this implementation, reported apart from the roofline:
    # per-slot fp32 rows beyond the T x W output, h written and read as MXFP4
    assert b.ffn_intermediate_bytes(w, "mxfp4") == (pairs - 4096) * 8192 * 4 + 2 * _mxfp4(pairs, 2048)


def test_latent_layer_counts_both_projections():
    b = _bench()
    w = synth.WORKLOADS["latent16"]
    dense = 2 * (896 * 7168 + 3 * 2048 * 7168 + 7168) + 2 * 2 * 2048 * 7168
    assert b.dense_bytes(w) == dense
    assert b.layer_bytes(w, 119) == 119 * 3 * _mxfp4(1024, 2048) + dense + 16 * 7168 * 2 + 16 * 7168 * 4
