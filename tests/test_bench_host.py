"""Host-side logic of bench.py on CPU: the max-over-ranks timing over a real two-rank
gloo process group, the whole-job throughput, the algorithmic byte count, and the
reference arm's rank handling. The benchmark runs replicas (one independent pool and
batch per rank), so these are the only multi-rank steps it takes."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    dev = torch.device("cpu")
    bench.barrier(dev)
    t = bench.max_over_ranks(10.0 + 5.0 * rank, dev)      # rank 1 is the slow one
    v = bench.job_throughput(20480, 100, world, t / 1e3)
    q.put((rank, t, v))
    dist.destroy_process_group()


def test_max_over_ranks_with_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, v in got:
        assert t == 15.0                                   # every rank sees the max
        assert v == pytest.approx(2 * 20480 * 100 / 0.015)


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5


def test_decode_bytes_of_the_batch_256_workload():
    state, total = bench.decode_bytes(256, 80, 1, 64, 128, 4, 2)
    assert state == 20480 * 64 * 128 * 4 * 2 == 1_342_177_280
    # x, z and out (bf16) once per (row, head, dim), dt per (row, head), B and C per row
    assert total - state == 20480 * 64 * 2 * 3 + 20480 * 4 + 256 * 128 * 2 * 2 + 80 * 12 + 256 * 4


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == bench.UNIT and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"


def test_traffic_record_is_tied_to_the_decode_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from the ncu record only when it was taken on the decode
    sources built now and at the workload's batch; otherwise it is null."""
    rec = {"batch": 256, "bytes_per_launch": 1234, "source_sha256": bench.decode_source_hash()}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic(256) == 1234
    assert bench.recorded_traffic(128) is None                # another batch
    path.write_text(json.dumps(dict(rec, source_sha256="0" * 64)))
    assert bench.recorded_traffic(256) is None                # other sources
    path.write_text("not json")
    assert bench.recorded_traffic(256) is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic(256) is None
