"""Multi-rank bench plumbing on CPU: two gloo ranks, each timing its own
replica; the job time is the max over ranks and the work the sum."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.rank_env()
    assert (r, w, lr) == (rank, world, rank)
    bench.init_dist(w, "gloo", timeout_s=60)
    bench.barrier()
    ms, units = bench.reduce_over_ranks(10.0 * (rank + 1), 100.0 + rank)
    q.put((rank, ms, units))
    import torch.distributed as dist
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_time_sum_units(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, units in got:
        assert ms == 10.0 * world
        assert units == sum(100.0 + r for r in range(world))


def test_single_rank_identity():
    import bench
    assert bench.reduce_over_ranks(3.5, 7) == (3.5, 7.0)


def test_bytes_model_matches_hand_count():
    """Per-head bytes of the GDN B128 H16 d128 C8 workload: state 64 KiB,
    log entry 772 B, inputs 776 B, output 256 B.  Amortised per token:
    with a separate merge 77 978 B read and 9 220 B written; with the
    merge-token (7 appends + one step that reads and writes the base)
    552 112 / 8 = 69 014 B read and 72 988 / 8 = 9 123.5 B written."""
    import bench
    from recurrent_state_head_b200 import synth
    w = synth.WORKLOADS["gdn-b128-h16-d128-c8"]
    bm = bench.bytes_model(w, fold=False)
    assert (bm["S"], bm["E"], bm["I"], bm["O"]) == (65536, 772, 776, 256)
    assert bm["token_read"] == 77978 and bm["token_write"] == 9220
    assert bm["eager"] == (65536 + 776, 65536 + 256)
    bf = bench.bytes_model(w, fold=True)
    assert bf["token_read"] == 69014 and bf["token_write"] == 9123.5
