"""Multi-process host logic of bench.py on CPU (gloo, world size 2): the job-level
throughput is all ranks' work over the slowest rank's time (max over ranks), and
only rank 0 of the reference arm does work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [2.0, 5.0][rank]                 # rank 1 is the slow one
        ms, rate = bench.aggregate(local_ms, 1e12, world)
        bench.barrier()
        out_q.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_aggregate_takes_max_over_ranks_and_sums_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate in res:
        assert ms == 5.0                              # the slowest rank's time
        assert rate == pytest.approx(2 * 1e12 / 5e-3)  # both ranks' work over it


def test_aggregate_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    ms, rate = bench.aggregate(4.0, 1e12, 1)
    assert ms == 4.0 and rate == pytest.approx(1e12 / 4e-3)


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_record_describes_the_current_gemm():
    # the DRAM bytes bench.py reports as roofline.traffic come from an ncu capture keyed
    # on the GEMM's sources: they must match the sources as committed
    sys.path.insert(0, ROOT)
    import bench
    nbytes, note = bench.traffic_from_profiles("nvfp4_gemm_mlp_up")
    assert nbytes is not None, note
    # at least the operands read once, at most the algorithmic bytes of the launch
    M, K, N = 4096, 3072, 12288
    operands = M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16
    assert operands <= nbytes <= operands + 2 * M * N


def test_traffic_record_goes_stale_when_a_source_changes(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import json
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    rec = {"bytes_per_launch": 123, "note": "n", "sources": ["k.cu"]}
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec["source_sha1"] = bench.source_hash(rec["sources"])
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"k": rec}))
    assert bench.traffic_from_profiles("k") == (123, "n")
    src.write_text("kernel v2\n")
    nbytes, note = bench.traffic_from_profiles("k")
    assert nbytes is None and "stale" in note
    assert bench.traffic_from_profiles("missing")[0] is None
