"""Host-side logic of bench.py without a GPU: the cross-rank timing and
throughput helpers over a real two-process gloo group, and the reference arm
(the CPU oracle) under its launch contract."""
import json
import os
import socket
import subprocess
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slowest
        ms_max = bench.max_over_ranks(torch, ms, dist, "cpu")
        value = bench.job_gbps(1e9, 100, ms_max, world)
        q.put((rank, ms_max, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo_world2():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    # every rank sees the slowest rank's time; the value counts both ranks' bytes
    assert [r[1] for r in res] == [15.0, 15.0]
    expected = 2 * 1e9 * 100 / 15e-3 / 1e9
    assert all(abs(r[2] - expected) < 1e-6 * expected for r in res)


def test_job_value_single_rank():
    assert bench.job_gbps(1e6, 10, 1.0, 1) == pytest.approx(10.0)
    assert bench.max_over_ranks(None, 3.5, None, "cpu") == 3.5


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=300, cwd=ROOT)


def test_reference_arm_contract():
    r = _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3", "--ref-budget", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3", "--ref-budget", "1"],
                   {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_traffic_valid_only_for_the_captured_sources(tmp_path):
    h = bench.kernel_source_hash()
    good = tmp_path / "t.json"
    good.write_text(json.dumps({"source_sha256": h, "traffic_bytes_per_launch": 1234.5}))
    assert bench.read_traffic(str(good)) == 1234.5
    stale = tmp_path / "s.json"
    stale.write_text(json.dumps({"source_sha256": "0" * 64, "traffic_bytes_per_launch": 1234.5}))
    assert bench.read_traffic(str(stale)) is None
    assert bench.read_traffic(str(tmp_path / "missing.json")) is None


def test_traffic_hash_covers_the_gemv_not_the_tensor_core_gemm(tmp_path, monkeypatch):
    import shutil
    src = os.path.join(ROOT, "ternary_weight_bit_w2a8_b200", "csrc")
    dst = tmp_path / "ternary_weight_bit_w2a8_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    assert h0 == bench.kernel_source_hash()
    tu = (dst / "bitnet_b200.cu").read_text(encoding="utf-8")
    a = tu.index(bench.TC_SECTION[0])
    (dst / "bitnet_b200.cu").write_text(tu[:a + len(bench.TC_SECTION[0])] + "\n// edit\n" +
                                        tu[a + len(bench.TC_SECTION[0]):], encoding="utf-8")
    assert bench.kernel_source_hash() == h0          # a tensor-core GEMM edit keeps the GEMV figure
    (dst / "gemv_tma.cuh").write_text((dst / "gemv_tma.cuh").read_text(encoding="utf-8") + "\n// edit\n",
                                      encoding="utf-8")
    assert bench.kernel_source_hash() != h0          # a GEMV edit invalidates it


def test_step_plan_covers_exactly_the_steps():
    for steps in (1, 5, 20, 447, 448, 449, 896, 20000):
        plan = bench.step_plan(steps, 448)
        assert len(plan) <= 2
        assert sum(n * r for (_, n, r) in plan) == steps
        i = 0
        for (i0, n, r) in plan:  # graphs in order, each starting where the last left off
            assert i0 == i and i0 % 7 == 0
            i += n * r
