"""Multi-rank logic of bench.py on the CPU: two gloo ranks.

The path shards over independent (sequence, head) replicas with no data-path
collective; the only cross-rank step is the maximum of the timings.  These tests run
that step with world size 2 over gloo and check the whole-job throughput rule and
that the reference arm prints on rank 0 only."""
import io
import contextlib
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (3 + r) ms of prefill and (7 - 2r) ms of decode
        got = bench.max_over_ranks([3.0 + rank, 7.0 - 2.0 * rank])
        env = bench.rank_env()
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            if rank != 0:
                bench.run_reference(bench_args())
        dist.barrier()
        out.put((rank, got, env, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def bench_args():
    class A:
        steps = 1
        warmup = 0
    return A()


def test_max_over_ranks_and_rank0_only_reference():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, got, env, printed = out.get(timeout=120)
        res[r] = (got, env, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        got, env, printed = res[r]
        assert got == [4.0, 7.0]            # max over ranks, element-wise
        assert env == (world, r, r)
    assert res[1][2] == ""                  # reference arm: ranks other than 0 print nothing


def test_max_over_ranks_without_process_group_is_identity():
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_whole_job_rate_is_weak_scaling(world):
    # every rank processes 16384 tokens; the slowest rank took 4 ms
    assert bench.whole_job_rate(16384, 4.0, world) == pytest.approx(16384 * world / 4e-3)


def test_oracle_baseline_jobs_take_every_variant():
    """The CPU-baseline job builders of bench.py accept channel-wise decay and window
    representatives (one tiny prefill and one decode step through the oracle)."""
    import bench
    import hla_synth as syn
    for w in (syn.TINY_F32.with_(decay="channel", T=128), syn.TINY_F32.with_(window=16, T=128)):
        inp = syn.make_gdn_inputs(w)
        tok = syn.make_decode_tokens(w, 1)[0]
        assert bench._oracle_prefill_worker(bench._prefill_jobs(inp, w, [(0, 1)])[0]) >= 0.0
        assert bench._oracle_decode_worker(bench._decode_jobs(inp, w, tok, [(0, 0)])[0]) >= 0.0
