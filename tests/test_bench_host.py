"""Host-side logic of bench.py on the CPU: the max-over-ranks reduction and the
per-rank seeds under a world-size-2 gloo process group, the committed-profile
lookup, and the JSON line of the reference (oracle) arm."""

import json
import os
import socket
import subprocess
import sys

import pytest
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


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    local = 1.5 + 2.0 * rank
    m = bench.max_over_ranks(local)
    bench.barrier()
    q.put((rank, m, bench.rank_seed(3, rank), bench.dist_env()))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [3.5, 3.5]
    assert res[0][2] != res[1][2]
    assert res[1][3] == (1, 1, 2)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(2.25) == 2.25


def test_recorded_traffic_requires_matching_source(tmp_path, monkeypatch):
    import hashlib
    csrc = tmp_path / "bit_decode_attention_sm_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    (tmp_path / "profiles" / "k.md").write_text(
        "# k\n- kernel_source_sha256: `%s`\n- dram_bytes_per_launch: 123456\n" % sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k.cu", "k.md") == 123456.0
    (csrc / "k.cu").write_text("kernel v2")
    assert bench.recorded_traffic("k.cu", "k.md") is None


def test_reference_arm_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    out = subprocess.check_output(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
         "--warmup", "1", "--workload", "tiny-1head-d64-T512-fp32"],
        env=env, text=True, timeout=600)
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "cached tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["steps"] == 2 and line["warmup"] == 1


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
