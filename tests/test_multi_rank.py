"""The bench's multi-rank path on CPU: two ranks in a gloo process group (127.0.0.1) run
the same barrier / max-over-ranks plumbing the GPU bench uses between its timed steps,
and every replica draws its own token stream."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist
    from decoder_only_transformer_train_b200 import synthetic as S
    w, r, _ = bench.dist_setup()
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    # each rank "measures" a different time; every rank must see the slowest
    ms = bench.dist_max(10.0 + 5.0 * r, w, "cpu")
    # the data-parallel run's logged loss: each rank's share of the mean, summed
    loss = bench.dist_max((2.0 + 4.0 * r) / w, w, "cpu", op="sum")
    stream = S.zipf_tokens(3 + r, 4097, 50257)          # the bench's per-replica token stream
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((r, ms, stream[:64].tolist(), loss))


def test_two_gloo_ranks_share_max_time_and_draw_distinct_streams():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, s0, l0), (r1, ms1, s1, l1) = res
    assert (r0, r1) == (0, 1)
    assert ms0 == ms1 == 15.0
    assert l0 == l1 == 4.0
    assert not np.array_equal(s0, s1)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse
    import bench
    args = argparse.Namespace(gpus=2, steps=1, warmup=0, micro_batch=16, seq=1024, accum=32)
    assert bench.run_reference(args, world=2, rank=1) is None
    assert capsys.readouterr().out == ""
