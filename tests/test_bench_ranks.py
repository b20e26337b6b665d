"""The benchmark's multi-rank bookkeeping on CPU (gloo, world size 2): each
rank times its own replica, the job time is the maximum over ranks, and the
job throughput counts every rank's tokens; the reference arm prints only on
rank 0."""
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.reduce_max(10.0 + 5.0 * rank)  # rank 1 is the slower one
        v = bench.job_throughput(world, 64, 20, t)
        q.put((rank, t, v))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, t, v in got:
        assert t == 15.0  # the slowest rank's time on every rank
        assert v == pytest.approx(2 * 64 * 20 / 0.015)


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max(3.5) == 3.5
    assert bench.job_throughput(1, 64, 10, 100.0) == pytest.approx(6400.0)


def test_reference_arm_is_silent_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    import json

    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "1"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "tiny"


def test_traffic_records_follow_the_device_code(tmp_path, monkeypatch):
    # a captured DRAM figure is reported only while the device code of its
    # kernel file hashes to the recorded value; host code and comments may
    # change without voiding it
    sys.path.insert(0, ROOT)
    import bench

    kernels = "// kernels\n__global__ void k(int* p) { p[0] = 1; }\n"
    host = bench.HOST_CODE_MARK + "\nint launch() { return 0; }\n"
    csrc = tmp_path / "mxfp4_quantised_mixture_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(kernels + host)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_src_sha("k.cu")
    monkeypatch.setattr(bench, "TRAFFIC", {"w": (1234, "k.cu", sha)})
    assert bench.captured_traffic("w") == 1234
    # host code and comments changed: still the same kernels
    (csrc / "k.cu").write_text("// another note\n" + kernels + host + "int more() { return 1; }\n")
    assert bench.captured_traffic("w") == 1234
    # a kernel changed: the figure is no longer this code's
    (csrc / "k.cu").write_text(kernels.replace("p[0] = 1", "p[0] = 2") + host)
    assert bench.captured_traffic("w") is None
    assert bench.captured_traffic("unrecorded") is None


def test_launch_count_per_gemm_path():
    # the decode workloads take the block-scaled path (five launches per
    # layer call), the prefill ones the decode-to-bf16 path (six)
    sys.path.insert(0, ROOT)
    import bench
    import synthetic as syn

    want = {"tiny": "block-scaled", "20b_decode": "block-scaled", "120b_decode": "block-scaled",
            "20b_prefill": "bf16-decode", "120b_skewed_prefill": "bf16-decode"}
    for name, path in want.items():
        assert bench.gemm_path(syn.WORKLOADS[name]) == path, name
    assert bench.LAUNCHES_PER_LAYER == {"block-scaled": 5, "bf16-decode": 6}
