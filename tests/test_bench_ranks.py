"""Host-side multi-rank logic of bench.py on CPU: world-size-2 gloo process
groups check that the job time is the max over ranks, that the barrier
releases every rank, that a rank which never joins ends the others' wait
with an error (short process-group timeout), and that the reference arm
prints exactly one line, from rank 0."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out_q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        bench.barrier()
        got = bench.reduce_max(values[rank])
        bench.barrier()
        out_q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_barrier_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    values = [1.25, 3.5]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, values, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 3.5, 1: 3.5}


def _lonely_worker(port, out_q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        # rank 1 never joins: the rendezvous (or the first collective) must end
        # with an error within the short timeout instead of waiting for good
        dist.init_process_group("gloo", rank=0, world_size=2,
                                timeout=datetime.timedelta(seconds=3))
        bench.reduce_max(1.0)
        out_q.put("returned")
    except Exception as e:  # noqa: BLE001 - any error is the expected outcome
        out_q.put("error:" + type(e).__name__)


def test_missing_rank_ends_with_an_error_not_a_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_lonely_worker, args=(_free_port(), q))
    p.start()
    p.join(timeout=120)
    if p.is_alive():
        p.kill()
        pytest.fail("a rank waiting for a peer that never joined did not time out")
    assert q.get(timeout=5).startswith("error:")


def test_reference_arm_prints_one_line_from_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r1 = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                         "tiny", "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                        capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    env.update(RANK="0", LOCAL_RANK="0")
    r0 = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                         "tiny", "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                        capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_runs_chunk_steps():
    """--qlen T: the CPU oracle leg times chunk steps (T new tokens, T queries
    per head) and the line records the chunk length."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--qlen", "3", "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    d = json.loads(lines[-1])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["config"]["q_len"] == 3 and d["config"]["seq_len"] == 256 + 3
    bad = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--qlen", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=120)
    assert bad.returncode != 0
