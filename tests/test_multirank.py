"""The multi-process host logic of bench.py on CPU: world size 2 over gloo.

With N > 1 every rank runs an independent replica of the layer (no data-path
collective); the only cross-rank steps are the timing reductions (max over
ranks) and the whole-job throughput. These tests run those steps in two
spawned CPU processes, and check that the reference arm does no work on
ranks other than 0.
"""
import datetime
import importlib.util
import os
import socket
import subprocess
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out_dir):
    import torch.distributed as dist
    b = _bench()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        step = b.max_over_ranks(values[rank][0], world, "cpu")
        e2e = b.max_over_ranks(values[rank][1], world, "cpu")
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{step!r} {e2e!r} {b.job_tokens_per_s(32, world, step)!r}\n")
    finally:
        dist.destroy_process_group()


def test_timing_is_the_max_over_ranks(tmp_path):
    world = 2
    values = [(0.250, 0.310), (0.275, 0.290)]      # step ms, end-to-end ms per rank
    mp.spawn(_worker, args=(world, _free_port(), values, str(tmp_path)), nprocs=world, join=True)
    got = [open(tmp_path / f"rank{r}.txt").read().split() for r in range(world)]
    for step, e2e, tps in got:
        assert float(step) == 0.275 and float(e2e) == 0.310   # both ranks see the slowest rank
        assert float(tps) == pytest.approx(32 * 2 / 0.275e-3)  # both replicas' tokens


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(1.25, 1, "cpu") == 1.25
    assert b.job_tokens_per_s(1, 1, 0.1) == pytest.approx(1e4)


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    b = _bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    import synth
    args = types.SimpleNamespace(steps=3, warmup=3, act=None)
    assert b.run_reference(args, synth.WORKLOADS["tiny"]) is None


def test_rank_environment():
    b = _bench()
    old = {k: os.environ.get(k) for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    try:
        os.environ.update(RANK="3", LOCAL_RANK="1", WORLD_SIZE="4")
        assert b._dist_env() == (3, 1, 4)
        for k in old:
            os.environ.pop(k, None)
        assert b._dist_env() == (0, 0, 1)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def test_reference_arm_line_on_rank_0(monkeypatch):
    """The reference arm's JSON line (the fp64 oracle on the host cores)."""
    b = _bench()
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    import synth
    args = types.SimpleNamespace(steps=2, warmup=3, act=None)
    out = b.run_reference(args, synth.WORKLOADS["tiny"])
    assert out["impl"] == "reference" and out["unit"] == "tokens/s" and out["value"] > 0
    assert out["warmup"] == 3 and 1 <= out["steps"] <= 2 and out["n_gpus"] == 1
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["value"] == out["value"]
    assert out["higher_is_better"] is True and out["metric"] == b.METRIC


def test_reference_arm_never_maps_the_product_library(repo_root):
    """The reference arm (the oracle on the host) runs in a process that never
    imports the product package nor maps its CUDA library."""
    code = (
        "import sys, types, bench, synth\n"
        "args = types.SimpleNamespace(steps=1, warmup=1, act=None)\n"
        "out = bench.run_reference(args, synth.WORKLOADS['tiny'])\n"
        "maps = open('/proc/self/maps').read()\n"
        "print('mapped' if 'libmoe_mxfp4' in maps else 'clean',\n"
        "      'imported' if 'mxfp4_routed_expert_04_b200' in sys.modules else 'clean',\n"
        "      'oracle' if 'libmoe_oracle' in maps else 'no-oracle')\n")
    env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        env.pop(k, None)
    res = subprocess.run([sys.executable, "-c", code], cwd=repo_root, env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    assert res.stdout.split() == ["clean", "clean", "oracle"], res.stdout


def test_bench_argument_defaults(monkeypatch, repo_root):
    """The extras and the streamed line default per workload (no GPU needed:
    main() is stopped before any measurement)."""
    b = _bench()
    seen = {}

    def fake_run(args, w):
        seen.update(extra=list(args.extra), streamed=args.streamed, name=w.name)
        return None
    monkeypatch.setattr(b, "run_ours", fake_run)
    for argv, want in ((["bench.py"], (["decode32", "latent16", "prefill4096"], True, "decode1")),
                       (["bench.py", "--workload", "prefill4096"], ([], False, "prefill4096")),
                       (["bench.py", "--no-extra"], ([], False, "decode1")),
                       (["bench.py", "--extra", "latent16"], (["latent16"], True, "decode1")),
                       (["bench.py", "--no-streamed"], (["decode32", "latent16", "prefill4096"],
                                                        False, "decode1"))):
        monkeypatch.setattr(sys, "argv", argv)
        b.main()
        assert (seen["extra"], seen["streamed"], seen["name"]) == want, argv
