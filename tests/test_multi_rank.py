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


def _ddp_rank_main(rank: int, world: int, port: int, k_local: int, out):
    """One data-parallel rank on CPU: the oracle's gradient of this rank's micro-batches
    (loss / k_local each), flattened as the library's buffer is, then the bench's exchange."""
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import torch.distributed as dist
    import bench
    import oracle as O
    from decoder_only_transformer_train_b200 import synthetic as S
    w, r, _ = bench.dist_setup()
    bench.dist_init(w, "gloo")
    cfg, B, T = O.TINY, 2, 32
    params = O.init_params(cfg, 8, dtype=torch.float64)
    grads = {n: torch.zeros_like(p) for n, p in params.items()}
    loss = 0.0
    for i in range(k_local):
        # the pages' loader: rank r reads the micro-batches r, r + world, r + 2 world, ...
        x, y = S.token_batch(17, B, T, cfg.vocab_size, micro_step=i * w + r)
        l, cache = O.forward(params, cfg, torch.from_numpy(x), torch.from_numpy(y))
        O.backward(params, cfg, cache, grad_scale=1.0 / k_local, grads=grads)
        loss += float(l) / k_local
    flat = O.flatten(grads, cfg).contiguous()
    bench.average_gradients(flat, w)
    loss = bench.dist_max(loss / w, w, "cpu", op="sum")
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((r, flat.numpy(), loss))


def test_two_gloo_ranks_average_to_the_global_batch_gradient():
    """Data parallelism ("Karpathy's Zero to Hero, Lecture 9" notes, "2:46:43 – 2:59:25 Going
    multi-GPU with DDP" and "2:59:25 – 3:10:20 Synchronizing gradients and losses"): two
    ranks, each with half of the optimizer step's micro-batches and its loss divided by its
    own micro-step count, exchange gradients once through bench.average_gradients.  Both
    ranks must then hold the oracle's gradient of the whole step's four micro-batches, and
    the averaged loss its mean loss, to fp64 round-off."""
    import torch
    import oracle as O
    from decoder_only_transformer_train_b200 import synthetic as S
    world, k_local = 2, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ddp_rank_main, args=(r, world, port, k_local, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg, B, T = O.TINY, 2, 32
    params = O.init_params(cfg, 8, dtype=torch.float64)
    m = {n: torch.zeros_like(t) for n, t in params.items()}
    v = {n: torch.zeros_like(t) for n, t in params.items()}
    batches = [S.token_batch(17, B, T, cfg.vocab_size, micro_step=i) for i in range(world * k_local)]
    tb = [(torch.from_numpy(x), torch.from_numpy(y)) for x, y in batches]
    loss_ref, _, grads_ref = O.train_step(params, m, v, 1, cfg, tb, 6e-4)
    g_ref = O.flatten(grads_ref, cfg).numpy()
    for r, g, loss in res:
        assert np.linalg.norm(g - g_ref) <= 1e-12 * np.linalg.norm(g_ref), r
        assert abs(loss - loss_ref) <= 1e-12 * abs(loss_ref), r
    assert np.array_equal(res[0][1], res[1][1])
