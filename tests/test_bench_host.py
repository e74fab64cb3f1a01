"""Host-side logic of bench.py: multi-rank aggregation (gloo, 2 ranks on CPU)
and the oracle reference arm on a small workload."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [10.0, 25.0][rank]                          # rank 1 is the slow one
        mx = bench.max_over_ranks(ms)
        val = bench.whole_job_tflops(1e12, world, mx)
        q.put((rank, mx, val))
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_and_replica_throughput_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, val in out:
        assert mx == 25.0                                 # every rank sees the slowest rank's time
        assert abs(val - 2 * 1e12 / 25e-3 / 1e12) < 1e-9  # all ranks' work over the max time


def test_single_process_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert abs(bench.whole_job_tflops(2e12, 1, 1.0) - 2000.0) < 1e-9


def test_reference_arm_runs_the_oracle_on_cpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_under_torchrun_two_ranks():
    # rank 0 alone prints the line; rank 1 exits 0 without work
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    port = 29700 + (os.getpid() % 200)
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port),
                        os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0", "--gpus", "2"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2


def test_ncu_traffic_only_for_the_sources_it_was_taken_at(tmp_path, monkeypatch):
    """The roofline's `traffic` comes from a profiles/ summary only while its
    source stamp matches the kernel sources; otherwise it is reported as null."""
    sys.path.insert(0, ROOT)
    import bench
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "cast_w13_dual_dsv3.md").write_text(
        "# summary\n\ntraffic_bytes_per_launch: 2.964e+10\n\nsource_hash: 0123456789ab\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "src_hash", lambda: "0123456789ab")
    assert bench.ncu_traffic("cast_w13_dual", "dsv3") == pytest.approx(2.964e10)
    assert bench.ncu_traffic("wgrad_dw13", "dsv3") is None          # no summary
    monkeypatch.setattr(bench, "src_hash", lambda: "ba9876543210")
    assert bench.ncu_traffic("cast_w13_dual", "dsv3") is None       # stale stamp


def test_source_hash_changes_with_any_kernel_source(tmp_path, monkeypatch):
    """Editing any one file of the CUDA sources changes the stamp."""
    sys.path.insert(0, ROOT)
    import bench
    csrc = tmp_path / "mxfp8_block_scaled_routed_b200" / "csrc"
    csrc.mkdir(parents=True)
    names = ["gemm.cuh", "mxmoe.cu", "quant.cuh"]
    for n in names:
        (csrc / n).write_text(f"// {n}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.src_hash()
    assert len(base) == 12 and bench.src_hash() == base
    for n in names:
        (csrc / n).write_text(f"// {n} edited\n")
        assert bench.src_hash() != base, n
        (csrc / n).write_text(f"// {n}\n")
    assert bench.src_hash() == base
