"""Host logic of bench.py on CPU: the replica aggregation over 2 gloo ranks (work
summed, times maxed), the roofline traffic record, and the CPU reference arm."""
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


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local = {"total_ms": 10.0 + rank, "prefill_ms": 5.0 * (rank + 1), "flops": 100.0,
             "bytes": 7.0 + rank}
    agg = bench.aggregate(local, world)
    out[rank] = agg
    dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(2):
        a = res[r]
        assert a["total_ms"] == 11.0 and a["prefill_ms"] == 10.0   # max over ranks
        assert a["flops"] == 200.0 and a["bytes"] == 15.0          # summed work


def test_aggregate_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    d = {"x_ms": 1.5, "flops": 3.0}
    assert bench.aggregate(d, 1) == d


def test_traffic_record_tracks_kernel_source(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    rec = {"attn_fwd_kernel": {"src_sha": bench.source_sha(bench.KERNEL_SOURCES["attn_fwd_kernel"]),
                               "dram_bytes_per_launch": 123}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # source files are looked up under ROOT too: point them back at the repository
    monkeypatch.setattr(bench, "source_sha", lambda paths: rec["attn_fwd_kernel"]["src_sha"])
    assert bench.ncu_traffic("attn_fwd_kernel") == 123
    monkeypatch.setattr(bench, "source_sha", lambda paths: "different")
    assert bench.ncu_traffic("attn_fwd_kernel") is None


def test_reference_arm_runs_on_cpu():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=120, cwd=ROOT, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""
