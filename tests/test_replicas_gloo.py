"""Host side of the multi-GPU mode (replicas only): two ranks on the CPU over
gloo, rendezvous on 127.0.0.1.  Checks the max-over-ranks timing, the whole-job
rate, that each replica draws different inputs, and that the oracle arm runs
on rank 0 alone."""
import datetime
import io
import os
import socket
import sys
import contextlib

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import workloads as W
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        wsz, r, local = bench.rank_env()
        ms = [1.5, 4.0][rank]                       # rank 1 is the slow one
        m = bench.max_over_ranks(ms, True, "cpu")
        w = W.BY_NAME["elu_bf16_fwd"]
        g = torch.Generator()
        g.manual_seed(bench.replica_seed(w, r))
        first = torch.randn(4, generator=g)
        gathered = [torch.empty(4) for _ in range(world)]
        torch.distributed.all_gather(gathered, first)
        # the oracle arm: rank 0 prints a line, the others return at once
        buf = io.StringIO()
        args = type("A", (), {"workload": "elu_fp32_fwd", "steps": 1, "warmup": 0, "gpus": world})()
        if r != 0:
            with contextlib.redirect_stdout(buf):
                rc = bench.run_reference(args)
        else:
            rc = 0
        torch.distributed.barrier()
        out.put((rank, wsz, r, local, m, bench.whole_job_rate(w.B * w.N, wsz, m),
                 [t.tolist() for t in gathered], rc, buf.getvalue()))
    finally:
        torch.distributed.destroy_process_group()


def test_two_rank_replica_host_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, wsz, r, local, m, rate, gathered, rc, printed in res:
        assert (wsz, r, local) == (2, rank, rank)
        assert m == 4.0                               # both ranks see the max
        assert abs(rate - 2 * 4 * 4096 / 4e-3) < 1e-6 * rate
        assert gathered[0] != gathered[1]             # independent replicas
        if rank == 1:
            assert rc == 0 and printed == ""          # oracle arm: rank 0 only
