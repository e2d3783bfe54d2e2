"""bench.py's host-side arithmetic (no GPU): the shapes each run takes, the metric names and
the FLOP model that the MFU and the roofline divide by."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _parse(*argv):
    old = sys.argv
    sys.argv = ["bench.py", *argv]
    try:
        return bench.parse()
    finally:
        sys.argv = old


def test_default_run_is_the_headline_workload():
    a = _parse()
    assert (a.gpus, a.micro_batch, a.seq, a.accum) == (1, 16, 1024, 32)
    assert a.micro_batch * a.seq * a.accum == 524288
    assert bench.metric_name(a.model, a.micro_batch, a.seq) == bench.METRIC
    assert a.warmup >= 3


def test_longer_context_keeps_the_tokens_per_step():
    a = _parse("--seq", "2048")
    assert (a.micro_batch, a.accum) == (32, 8)         # the pages' GPT-3 batch: B = 32 at T = 2048
    assert a.micro_batch * a.seq * a.accum == 524288
    name = bench.metric_name(a.model, a.micro_batch, a.seq)
    assert name != bench.METRIC and "T=2048" in name
    a = _parse("--seq", "512")
    assert a.micro_batch * a.seq * a.accum == 524288 and a.micro_batch * a.seq <= 131072


def test_medium_model_defaults():
    a = _parse("--model", "medium")
    assert (a.micro_batch, a.accum) == (8, 8)
    assert "medium" in bench.metric_name(a.model, a.micro_batch, a.seq)


def test_flop_model():
    # 6 N per token for the 124M matrices (pad columns counted) plus 6 L T C for attention
    L, C, Vp = 12, 768, 50304
    assert bench.flop_per_token("124m") == 6 * (12 * L * C * C + Vp * C) + 6 * L * 1024 * C == 798031872
    assert bench.flop_per_token("124m", 2048) - bench.flop_per_token("124m", 1024) == 6 * L * 1024 * C
    assert bench.flop_per_token("medium") == 2272002048


def test_data_parallel_runs_split_the_micro_steps():
    a = bench.ddp_shape(_parse("--ddp", "--gpus", "4"), 4)
    assert (a.accum, a.ddp_world) == (8, 4)
    cfg = bench.workload_config(a)
    assert cfg["tokens_per_step"] == 524288 and cfg["parallelism"] == "ddp4"
    a = bench.ddp_shape(_parse("--gpus", "4"), 4)          # replicas: each rank runs the whole step
    assert (a.accum, a.ddp_world) == (32, 1)
    assert bench.workload_config(a)["parallelism"] == "replicas"
    a = bench.ddp_shape(_parse("--ddp"), 1)                 # one rank: nothing to average
    assert (a.accum, a.ddp_world) == (32, 1)
    try:
        bench.ddp_shape(_parse("--ddp", "--accum", "6"), 4)
        raise AssertionError("6 micro-steps do not split over 4 ranks")
    except SystemExit:
        pass
