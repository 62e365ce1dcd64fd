"""The multi-rank bookkeeping of bench.py on CPU: two gloo ranks, as torchrun would start them
(one process each, rendezvous on 127.0.0.1).  The job's time is the slowest rank's, its
tokens the sum over ranks (weak scaling), and the reference arm does no work off rank 0."""
import importlib.util
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        # rank r measured 10 + r ms over 1000 (r + 1) tokens, and 3 - r ms end to end
        mx, sm = bench.reduce_over_ranks([10.0 + rank, 3.0 - rank], [1000.0 * (rank + 1)],
                                         torch.device("cpu"))
        out.put((rank, mx, sm))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_time_and_tokens():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, mx, sm in results:
        assert mx == [11.0, 3.0]        # the slowest rank's time, per quantity
        assert sm == [3000.0]           # every rank's tokens


def test_reference_arm_is_rank0_only(capsys):
    bench = _bench()

    class Args:
        seed, warmup, steps, gpus = 0, 3, 1, 2

    bench.run_reference(Args, rank=1)   # returns at once, prints nothing
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_contract_line():
    # the reference arm (the fp64 oracle on the host cores) on rank 0: one JSON line with the
    # contract's keys; one short step keeps this test to seconds
    import json
    import subprocess
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                          timeout=600, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-2000:]
    line = json.loads(proc.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1
    for key in ("metric", "unit", "n_gpus", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
