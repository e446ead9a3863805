"""The N > 1 path of the benchmark on CPU: world-size-2 gloo process group.

Every rank runs an independent replica; the job time is the slowest rank's (one
all-reduce MAX) and the job throughput counts every rank's tokens over that time.  Also:
under a multi-rank launch the reference arm runs on rank 0 only, the other ranks exit 0
without output.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        job_ms = bench.max_over_ranks(ms, "cpu", world)
        results.put((rank, job_ms, bench.job_tokens_per_s(world, 8192, 20, job_ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(results.get(timeout=10) for _ in range(2))
    for rank, job_ms, value in got:
        assert job_ms == 15.0                         # both ranks see the slowest time
        assert value == pytest.approx(2 * 8192 * 20 / 15e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, "cpu", 1) == 12.5
    assert bench.job_tokens_per_s(1, 1000, 10, 100.0) == pytest.approx(1e5)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "1", "--warmup", "1", "--gpus", "2"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-1000:]
    assert r.stdout.strip() == ""


def _ep_rank_main(rank, world, port, results):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from token_dispatch_grouped_top_b200 import ep
    from token_dispatch_grouped_top_b200._lib import EP_PEER_FIELDS, MoeEpPeer
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # this rank's entry: its token count and (stand-in) buffer addresses
        mine = {"T": 100 + rank}
        mine.update({n: (rank + 1) * 0x10000 + 0x100 * i for i, n in enumerate(EP_PEER_FIELDS)})
        # a remote rank's addresses are mapped (here: offset by 1 << 40, as a peer mapping)
        entries = ep.gather_entries(mine, map_fn=lambda r, e: {
            n: (v + (1 << 40) if n != "T" else v) for n, v in e.items()})
        table = ep.peer_table(entries, "cpu")
        arr = (MoeEpPeer * world).from_buffer_copy(bytes(table.numpy()))
        rows = [(arr[i].T,) + tuple(getattr(arr[i], n) for n in EP_PEER_FIELDS)
                for i in range(world)]
        results.put((rank, rows))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_peer_table_gloo():
    # the host side of the expert-parallel step: every rank gathers every rank's entry in
    # rank order, maps the remote ones, and packs the same moe_ep_peer layout
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_ep_rank_main, args=(r, world, port, results))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(results.get(timeout=10) for _ in range(world))
    from token_dispatch_grouped_top_b200._lib import EP_PEER_FIELDS
    for me, rows in got.items():
        assert len(rows) == world
        for r, row in enumerate(rows):
            assert row[0] == 100 + r
            shift = 0 if r == me else 1 << 40
            assert list(row[1:]) == [(r + 1) * 0x10000 + 0x100 * i + shift
                                     for i in range(len(EP_PEER_FIELDS))]
