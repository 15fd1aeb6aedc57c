"""The multi-process plumbing of bench.py on the CPU: two ranks over gloo
(the GPU run uses the same code over NCCL). The path shards as independent
replicas, so the only collectives are the barrier and the max over ranks of
the timed region; the reference arm runs on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    m = d.max(10.0 * (rank + 1))
    d.barrier()
    d.close()
    out.put((rank, d.world, m))


def test_dist_max_over_two_gloo_ranks():
    """bench.Dist over gloo with world size 2: both ranks see the maximum of
    their values (the timed region's max over ranks) and leave cleanly."""
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
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 2, 20.0), (1, 2, 20.0)]


def test_reference_arm_prints_once_under_torchrun():
    """`bench.py --impl reference` launched by torchrun with two ranks: rank 0
    times the oracle and prints one JSON line, rank 1 exits without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference", "--gpus", "2",
           "--steps", "2", "--warmup", "1", "--ref-seconds", "2"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0


def test_replicas_draw_distinct_inputs():
    """Each rank runs an independent replica: its inputs come from the seed
    offset by 1000 per rank, so two ranks do not time the same data."""
    from selective_state_space_27_b200.inputs import SCAN_WORKLOADS, make_scan_inputs
    w = SCAN_WORKLOADS["mamba130m_layer"]
    a = make_scan_inputs(w, batch=1, dim=8, seqlen=32, seed=w.seed)
    b = make_scan_inputs(w, batch=1, dim=8, seqlen=32, seed=w.seed + 1000)
    assert (a["u"] != b["u"]).any()
