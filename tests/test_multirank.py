"""The multi-GPU path of bench.py on CPU: two gloo ranks stand in for two
GPUs.  The path shards with no data exchange (every rank runs its own
sequences), so what crosses ranks is the timing only: the slowest rank's
time, reduced with a MAX all-reduce.  The reference arm under torchrun prints
one line from rank 0 while the other ranks exit without work."""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys
from datetime import timedelta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    import kv_inputs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 + 3.0 * rank, dist)
        t2 = bench.max_over_ranks(5.0 - rank, dist)
        lens = bench.rank_sequence_lengths(kv_inputs, rank)
        out.put((rank, t, t2, lens))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_own_sequences():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, t0, u0, lens0), (r1, t1, u1, lens1) = got
    assert (r0, r1) == (0, 1)
    assert t0 == t1 == 13.0 and u0 == u1 == 5.0  # every rank sees the slowest rank's time
    import bench
    assert lens0 != lens1  # weak scaling: each rank holds its own sequences
    for lens in (lens0, lens1):
        assert len(lens) == bench.N_SEQ and all(bench.LEN_LO <= n <= bench.LEN_HI for n in lens)


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--cpu-units", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
