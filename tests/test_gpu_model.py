"""Model-level parity on a B200: the whole training step through the C ABI against the
CPU oracle on the same seeded inputs and weights.

Tolerances: fp32 mode - loss 1e-4 relative, per-tensor gradients and updated weights
1e-4 relative L2; bf16 mode - loss 2e-2 absolute, per-tensor gradient relative L2 2e-2;
token gathers, masks and the argmax bit-exact (argmax on rows whose reference top-2 gap
exceeds the bf16 logit error)."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from decoder_only_transformer_train_b200 import binding as BD
from decoder_only_transformer_train_b200 import synthetic as S
from gpu_common import cuda_i32, rel_l2, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


TINY = O.TINY   # L=2, C=64, H=4, T=64, V=512


def _bd_config(cfg: O.Config, B: int, k: int, prec: int) -> BD.Config:
    return BD.Config(n_layer=cfg.n_layer, n_embd=cfg.n_embd, n_head=cfg.n_head, block_size=cfg.block_size,
                     vocab_size=cfg.vocab_size, padded_vocab_size=cfg.padded_vocab_size, max_batch=B,
                     grad_accum_steps=k, precision=prec)


def _per_tensor(flat_gpu: np.ndarray, ref: dict, cfg: O.Config, skip_key_bias: bool = False):
    """Per-tensor relative L2.  skip_key_bias drops the key slice [C, 2C) of every
    attn.c_attn.bias: its exact gradient is zero (adding one vector to every key shifts
    all scores of a query equally and the softmax ignores it), so both sides hold rounding
    noise there, which AdamW's first step g / (|g| + eps) turns into an update of
    arbitrary sign."""
    got = O.unflatten(torch.from_numpy(flat_gpu).double(), cfg)
    out = {}
    C = cfg.n_embd
    for n, _ in O.param_specs(cfg):
        a, b = got[n], ref[n]
        if skip_key_bias and n.endswith("attn.c_attn.bias"):
            a = torch.cat([a[:C], a[2 * C:]])
            b = torch.cat([b[:C], b[2 * C:]])
        out[n] = rel_l2(a, b)
    return out


def _run_step(cfg, prec, B, T, k=1, seed_w=1, seed_d=2, lr=6e-4):
    """One optimizer step over k micro-batches on the GPU and in the oracle (fp64)."""
    params = O.init_params(cfg, seed_w, dtype=torch.float64)
    flat = O.flatten(params, cfg).numpy().astype(np.float32)
    params = O.unflatten(torch.from_numpy(flat).double(), cfg)     # oracle starts from the same fp32 values
    batches = [S.token_batch(seed_d, B, T, cfg.vocab_size, micro_step=i) for i in range(k)]
    model = BD.GPT2(_bd_config(cfg, B, k, prec), seed=seed_w)
    model.set_params(flat)
    model.zero_grad()
    losses = []
    for x, y in batches:
        losses.append(model.forward(cuda_i32(x), cuda_i32(y)))
        model.backward()
    grads_gpu = model.get_grads()
    norm_gpu = model.adamw_step(lr)
    params_gpu = model.get_params()
    m_gpu, v_gpu, t_gpu = model.get_optimizer_state()
    argmax_gpu = model.get_argmax(B * T)
    model.close()
    m = {n: torch.zeros_like(t) for n, t in params.items()}
    v = {n: torch.zeros_like(t) for n, t in params.items()}
    p_ref = {n: t.clone() for n, t in params.items()}
    tb = [(torch.from_numpy(x), torch.from_numpy(y)) for x, y in batches]
    loss_ref, norm_ref, grads_ref = O.train_step(p_ref, m, v, 1, cfg, tb, lr)
    _, cache = O.forward(params, cfg, *tb[-1])
    return dict(losses=losses, loss_ref=loss_ref, grads_gpu=grads_gpu, grads_ref=grads_ref, norm_gpu=norm_gpu,
                norm_ref=norm_ref, params_gpu=params_gpu, params_ref=p_ref, params0=params,
                m_gpu=m_gpu, v_gpu=v_gpu, t_gpu=t_gpu, m_ref=m, v_ref=v,
                argmax_gpu=argmax_gpu, logits_ref=cache["logits"])


def _check_argmax(argmax_gpu: np.ndarray, logits_ref: torch.Tensor, gap: float = 0.05):
    """The argmax over all padded columns (ties to the lowest index) is bit-exact on every
    row whose oracle top-2 gap exceeds `gap`, a bound well above the bf16 logit error at
    these scales; at least half the rows must be such rows, so the check is never empty."""
    top2 = torch.topk(logits_ref, 2, dim=1).values
    clear = (top2[:, 0] - top2[:, 1]) > gap
    assert int(clear.sum()) >= clear.numel() // 2, f"only {int(clear.sum())} of {clear.numel()} rows are clear"
    got = torch.from_numpy(argmax_gpu).long()
    assert torch.equal(got[clear], O.argmax_lowest(logits_ref).long()[clear])


def test_init_matches_oracle_generator():
    cfg = TINY
    model = BD.GPT2(_bd_config(cfg, 2, 1, BD.GPT2_FP32), seed=1234)
    got = model.get_params()
    model.close()
    ref = O.flatten(O.init_params(cfg, 1234, dtype=torch.float32), cfg).numpy()
    assert got.shape == ref.shape
    close = np.isclose(got, ref, rtol=2e-7, atol=0)
    assert close.mean() > 0.9999 and np.array_equal(got[ref == 1.0], ref[ref == 1.0])
    assert np.max(np.abs(got - ref)) < 1e-6


def test_tiny_fp32_step_matches_oracle():
    r = _run_step(TINY, BD.GPT2_FP32, B=2, T=64)
    assert abs(r["losses"][0] - r["loss_ref"]) <= 1e-4 * abs(r["loss_ref"])
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], TINY)
    assert max(errs.values()) < 1e-4, {k: v for k, v in errs.items() if v >= 1e-4}
    assert abs(r["norm_gpu"] - r["norm_ref"]) <= 1e-4 * r["norm_ref"]
    werr = _per_tensor(r["params_gpu"], r["params_ref"], TINY, skip_key_bias=True)
    assert max(werr.values()) < 1e-4, {k: v for k, v in werr.items() if v >= 1e-4}
    # the key-bias gradient is zero up to rounding on the GPU as well
    g = O.unflatten(torch.from_numpy(r["grads_gpu"]).double(), TINY)
    C = TINY.n_embd
    for l in range(TINY.n_layer):
        kb = g[f"h.{l}.attn.c_attn.bias"][C:2 * C]
        assert float(kb.abs().max()) < 1e-6 * float(g[f"h.{l}.attn.c_attn.bias"].abs().max())
    # the update itself (p1 - p0), a stricter view of the same check
    p0 = O.flatten(r["params0"], TINY).numpy()
    d_ref = {n: r["params_ref"][n] - r["params0"][n] for n in r["params0"]}
    derr = _per_tensor(r["params_gpu"] - p0, d_ref, TINY, skip_key_bias=True)
    assert max(derr.values()) < 1e-2, derr


def test_tiny_bf16_step_matches_oracle():
    r = _run_step(TINY, BD.GPT2_BF16, B=2, T=64)
    assert abs(r["losses"][0] - r["loss_ref"]) < 2e-2
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], TINY)
    assert max(errs.values()) < 2e-2, {k: v for k, v in errs.items() if v >= 2e-2}
    _check_argmax(r["argmax_gpu"], r["logits_ref"])


def _check_moments(r, cfg, tol):
    """AdamW's first and second moments after the step, per tensor (relative L2), and the
    step count: the state an exact resume needs ("Karpathy's Zero to Hero, Lecture 9" notes,
    "3:53:37 – 3:59:21 Checkpoints, fine-tuning and llm.c")."""
    assert r["t_gpu"] == 1
    merr = _per_tensor(r["m_gpu"], r["m_ref"], cfg)
    verr = _per_tensor(r["v_gpu"], r["v_ref"], cfg)
    assert max(merr.values()) < tol, {k: v for k, v in merr.items() if v >= tol}
    assert max(verr.values()) < tol, {k: v for k, v in verr.items() if v >= tol}


def test_tiny_fp32_step_optimizer_state_matches_oracle():
    r = _run_step(TINY, BD.GPT2_FP32, B=2, T=64)
    _check_moments(r, TINY, 1e-4)


def test_tiny_fp32_accumulation_over_three_micro_steps_matches_oracle():
    """Gradient accumulation ("Karpathy's Zero to Hero, Lecture 9" notes, "2:34:49 – 2:46:43
    Gradient accumulation"): each micro-step's loss is divided by k and the gradients add up,
    so the step equals one over the k micro-batches together.  Against the oracle's step over
    the same three micro-batches: the mean loss, every gradient, the norm, the updated weights
    and the moments."""
    k = 3
    r = _run_step(TINY, BD.GPT2_FP32, B=2, T=64, k=k, seed_d=12)
    loss_gpu = sum(r["losses"]) / k
    assert abs(loss_gpu - r["loss_ref"]) <= 1e-4 * abs(r["loss_ref"])
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], TINY)
    assert max(errs.values()) < 1e-4, {kk: v for kk, v in errs.items() if v >= 1e-4}
    assert abs(r["norm_gpu"] - r["norm_ref"]) <= 1e-4 * r["norm_ref"]
    werr = _per_tensor(r["params_gpu"], r["params_ref"], TINY, skip_key_bias=True)
    assert max(werr.values()) < 1e-4, {kk: v for kk, v in werr.items() if v >= 1e-4}
    _check_moments(r, TINY, 1e-4)


def test_tiny_bf16_accumulation_over_four_micro_steps_matches_oracle():
    k = 4
    r = _run_step(TINY, BD.GPT2_BF16, B=2, T=64, k=k, seed_d=13)
    assert abs(sum(r["losses"]) / k - r["loss_ref"]) < 2e-2
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], TINY)
    assert max(errs.values()) < 2e-2, {kk: v for kk, v in errs.items() if v >= 2e-2}
    _check_argmax(r["argmax_gpu"], r["logits_ref"])


def test_step_resumed_from_saved_state_matches_oracle():
    """A step taken by a fresh context restored from a saved (params, m, v, t) equals the
    oracle's step started from the same saved state ("Karpathy's Zero to Hero, Lecture 9"
    notes, "3:53:37 – 3:59:21 Checkpoints, fine-tuning and llm.c": exact resume needs the
    optimizer's moments and step count): loss, updated weights, m, v and t."""
    cfg, B, T, k = TINY, 2, 64, 2
    batches = lambda step: [S.token_batch(41, B, T, cfg.vocab_size, micro_step=step * k + i) for i in range(k)]
    flat0 = O.flatten(O.init_params(cfg, 6, dtype=torch.float64), cfg).numpy().astype(np.float32)

    def train(model, step):
        model.zero_grad()
        losses = []
        for x, y in batches(step):
            losses.append(model.forward(cuda_i32(x), cuda_i32(y)))
            model.backward()
        model.adamw_step(O.get_lr(step))
        return losses

    first = BD.GPT2(_bd_config(cfg, B, k, BD.GPT2_FP32), seed=6)
    first.set_params(flat0)
    train(first, 0)
    saved_p = first.get_params()
    saved_m, saved_v, saved_t = first.get_optimizer_state()
    first.close()
    assert saved_t == 1
    resumed = BD.GPT2(_bd_config(cfg, B, k, BD.GPT2_FP32), seed=99)   # other init: all of it is overwritten
    resumed.set_params(saved_p)
    resumed.set_optimizer_state(saved_m, saved_v, saved_t)
    losses = train(resumed, 1)
    p_gpu = resumed.get_params()
    m_gpu, v_gpu, t_gpu = resumed.get_optimizer_state()
    resumed.close()

    to64 = lambda a: O.unflatten(torch.from_numpy(a).double(), cfg)
    p_ref, m_ref, v_ref = to64(saved_p), to64(saved_m), to64(saved_v)
    tb = [(torch.from_numpy(x), torch.from_numpy(y)) for x, y in batches(1)]
    loss_ref, _, _ = O.train_step(p_ref, m_ref, v_ref, saved_t + 1, cfg, tb, O.get_lr(1))
    assert t_gpu == 2
    assert abs(sum(losses) / k - loss_ref) <= 1e-4 * abs(loss_ref)
    werr = _per_tensor(p_gpu, p_ref, cfg, skip_key_bias=True)
    assert max(werr.values()) < 1e-4, {kk: v for kk, v in werr.items() if v >= 1e-4}
    for got, ref in ((m_gpu, m_ref), (v_gpu, v_ref)):
        err = _per_tensor(got, ref, cfg)
        assert max(err.values()) < 1e-4, {kk: v for kk, v in err.items() if v >= 1e-4}


# The medium model's width (GPT-2 350M: 1024 channels, 16 heads of 64) with two layers, so
# that the oracle stays quick: LayerNorm over 1024 columns, the 1024/3072/4096-wide GEMMs and
# 16-head attention run the kernels of the 24-layer model.
MEDIUM_WIDTH = O.Config(n_layer=2, n_embd=1024, n_head=16, block_size=256, vocab_size=1000,
                        padded_vocab_size=1024)


def test_medium_width_bf16_step_matches_oracle():
    r = _run_step(MEDIUM_WIDTH, BD.GPT2_BF16, B=2, T=256)
    assert abs(r["losses"][0] - r["loss_ref"]) < 2e-2
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], MEDIUM_WIDTH)
    assert max(errs.values()) < 2e-2, {k: v for k, v in errs.items() if v >= 2e-2}
    _check_argmax(r["argmax_gpu"], r["logits_ref"])


# Fourteen layers of head size 64: the backward then leaves more parameter-gradient partials
# (LayerNorm weights and biases, the c_attn, c_fc and both c_proj biases: 3 + 8 * 13 + 7 = 114
# reductions) than one launch of the batched fixed-order reduction takes (100), so the
# reduction runs as two launches.
DEEP = O.Config(n_layer=14, n_embd=128, n_head=2, block_size=64, vocab_size=512, padded_vocab_size=512)


def test_deep_bf16_step_matches_oracle():
    r = _run_step(DEEP, BD.GPT2_BF16, B=2, T=64)
    assert abs(r["losses"][0] - r["loss_ref"]) < 2e-2
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], DEEP)
    assert max(errs.values()) < 2e-2, {k: v for k, v in errs.items() if v >= 2e-2}
    # the LayerNorm and bias gradients come only from the batched reduction
    small = {k: v for k, v in errs.items() if k.endswith(("ln_1.weight", "ln_1.bias", "ln_2.weight", "ln_2.bias",
                                                             "c_attn.bias", "c_fc.bias", "c_proj.bias"))}
    assert len(small) >= 7 * DEEP.n_layer, sorted(small)[:8]


# The GPT-3 context length with the 124M model's head size ("Karpathy's Zero to Hero, Lecture 9"
# notes, "3:41:50 – 3:53:37 Results: one epoch and an overnight run": T = 2048 to match GPT-3):
# 16 key tiles per query row in the attention kernels, a 2048-row position table.
LONG_CONTEXT = O.Config(n_layer=2, n_embd=128, n_head=2, block_size=2048, vocab_size=1000, padded_vocab_size=1024)


def test_context_2048_bf16_step_matches_oracle():
    r = _run_step(LONG_CONTEXT, BD.GPT2_BF16, B=1, T=2048)
    assert abs(r["losses"][0] - r["loss_ref"]) < 2e-2
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], LONG_CONTEXT)
    assert max(errs.values()) < 2e-2, {k: v for k, v in errs.items() if v >= 2e-2}
    _check_argmax(r["argmax_gpu"], r["logits_ref"])


# The pages' GPT-3 batch at that context: B = 32 sequences of T = 2048, 65,536 positions in one
# micro-step, which the embedding backward sorts as sixteen segments merged by ranks.
GPT3_BATCH = O.Config(n_layer=1, n_embd=128, n_head=2, block_size=2048, vocab_size=1000, padded_vocab_size=1024)


@pytest.mark.slow
def test_context_2048_batch_32_bf16_step_matches_oracle():
    r = _run_step(GPT3_BATCH, BD.GPT2_BF16, B=32, T=2048)
    assert abs(r["losses"][0] - r["loss_ref"]) < 2e-2
    errs = _per_tensor(r["grads_gpu"], r["grads_ref"], GPT3_BATCH)
    assert max(errs.values()) < 2e-2, {k: v for k, v in errs.items() if v >= 2e-2}
    _check_argmax(r["argmax_gpu"], r["logits_ref"])


def test_resume_from_saved_state_continues_bit_for_bit():
    """Exact resume ("Karpathy's Zero to Hero, Lecture 9" notes, "3:53:37 – 3:59:21
    Checkpoints, fine-tuning and llm.c": the weights alone are not enough, AdamW's m and v
    and the random state are needed too).  Three steps straight through must equal two
    steps, a save of (params, m, v, t), a fresh context restored from it, and the third
    step, bit for bit.  The token stream is a counter-based generator, so the data position
    is the micro-step index; the model itself draws no random numbers after init."""
    B, T, k = 2, 64, 2
    batches = lambda step: [S.token_batch(21, B, T, TINY.vocab_size, micro_step=step * k + i) for i in range(k)]

    def train(model, step):
        model.zero_grad()
        losses = []
        for x, y in batches(step):
            losses.append(model.forward(cuda_i32(x), cuda_i32(y)))
            model.backward()
        norm = model.adamw_step(O.get_lr(step + 1))
        return losses, norm

    straight = BD.GPT2(_bd_config(TINY, B, k, BD.GPT2_BF16), seed=3)
    log_a = [train(straight, s) for s in range(3)]
    final_a = straight.get_params()
    m_a, v_a, t_a = straight.get_optimizer_state()
    straight.close()

    first = BD.GPT2(_bd_config(TINY, B, k, BD.GPT2_BF16), seed=3)
    log_b = [train(first, s) for s in range(2)]
    saved = (first.get_params(), *first.get_optimizer_state())
    first.close()
    assert saved[3] == 2
    resumed = BD.GPT2(_bd_config(TINY, B, k, BD.GPT2_BF16), seed=77)   # other init: all of it is overwritten
    resumed.set_params(saved[0])
    resumed.set_optimizer_state(saved[1], saved[2], saved[3])
    log_b.append(train(resumed, 2))
    final_b = resumed.get_params()
    m_b, v_b, t_b = resumed.get_optimizer_state()
    resumed.close()

    assert log_a == log_b
    assert np.array_equal(final_a, final_b)
    assert np.array_equal(m_a, m_b) and np.array_equal(v_a, v_b) and t_a == t_b == 3


def test_gradient_buffer_view_and_a_one_rank_data_parallel_step():
    """grad_tensor() aliases the library's gradient buffer (what a data-parallel all-reduce
    averages in place), and a step whose gradients go through the bench's exchange on a
    one-rank NCCL group equals the plain step bit for bit (one rank only: no two kernels here wait on each other)."""
    import socket
    import datetime
    import torch.distributed as dist
    import bench
    B, T, k = 2, 64, 2
    batches = [S.token_batch(31, B, T, TINY.vocab_size, micro_step=i) for i in range(k)]

    def run(average: bool):
        model = BD.GPT2(_bd_config(TINY, B, k, BD.GPT2_BF16), seed=4)
        model.set_graphs(False)
        model.zero_grad()
        for x, y in batches:
            model.forward(cuda_i32(x), cuda_i32(y))
            model.backward()
        g = model.grad_tensor()
        model.synchronize()
        assert g.numel() == model.num_params and g.dtype == torch.float32 and g.is_cuda
        assert np.array_equal(g.cpu().numpy(), model.get_grads())
        if average:
            bench.average_gradients(g, dist.get_world_size())
            torch.cuda.synchronize()
        model.adamw_step(6e-4)
        out = model.get_params()
        del g
        model.close()
        return out

    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        plain, averaged = run(False), run(True)
    finally:
        dist.destroy_process_group()
    assert np.array_equal(plain, averaged)

    # writes through the view land in the library's buffer, which the optimizer reads
    model = BD.GPT2(_bd_config(TINY, B, k, BD.GPT2_BF16), seed=4)
    model.zero_grad()
    x, y = batches[0]
    model.forward(cuda_i32(x), cuda_i32(y))
    model.backward()
    g0 = model.get_grads()
    view = model.grad_tensor()
    view.mul_(0.5)
    torch.cuda.synchronize()
    assert np.array_equal(model.get_grads(), g0 * np.float32(0.5))
    del view
    model.close()


def test_graph_replay_matches_direct_launches():
    """Two optimizer steps of three micro-steps each: with graphs on, the first call of a
    shape runs directly, the second is captured and the rest replay the graph.  Every loss
    and every updated weight must equal the direct-launch run bit for bit, and the library's
    launch counter must count the same kernels."""
    B, T, k = 2, 64, 3
    batches = [S.token_batch(5, B, T, TINY.vocab_size, micro_step=i) for i in range(k)]
    runs = []
    for graphs in (False, True):
        model = BD.GPT2(_bd_config(TINY, B, k, BD.GPT2_BF16), seed=1)
        model.set_graphs(graphs)
        n0 = BD.lib().gpt2_kernel_launches()
        losses = []
        for _ in range(2):
            model.zero_grad()
            for x, y in batches:
                losses.append(model.forward(cuda_i32(x), cuda_i32(y)))
                model.backward()
            model.adamw_step(6e-4)
        model.synchronize()
        launches = BD.lib().gpt2_kernel_launches() - n0
        runs.append((losses, model.get_params(), launches))
        model.close()
    assert runs[0][0] == runs[1][0]
    assert np.array_equal(runs[0][1], runs[1][1])
    assert runs[0][2] == runs[1][2]


def test_grad_accumulation_fp32_equals_one_batch():
    cfg = TINY
    flat = O.flatten(O.init_params(cfg, 5, dtype=torch.float32), cfg).numpy()
    x, y = S.token_batch(6, 4, 32, cfg.vocab_size)
    big = BD.GPT2(_bd_config(cfg, 4, 1, BD.GPT2_FP32), seed=5)
    big.set_params(flat)
    big.zero_grad()
    big.forward(cuda_i32(x), cuda_i32(y))
    big.backward()
    g_big = big.get_grads()
    big.close()
    acc = BD.GPT2(_bd_config(cfg, 2, 2, BD.GPT2_FP32), seed=5)
    acc.set_params(flat)
    acc.zero_grad()
    for i in range(2):
        acc.forward(cuda_i32(x[2 * i:2 * i + 2]), cuda_i32(y[2 * i:2 * i + 2]))
        acc.backward()
    g_acc = acc.get_grads()
    acc.close()
    assert rel_l2(g_acc, g_big) < 1e-5


def test_bf16_step_is_deterministic():
    cfg = TINY
    outs = []
    for _ in range(2):
        model = BD.GPT2(_bd_config(cfg, 2, 1, BD.GPT2_BF16), seed=9)
        x, y = S.token_batch(10, 2, 64, cfg.vocab_size)
        model.zero_grad()
        model.forward(cuda_i32(x), cuda_i32(y))
        model.backward()
        outs.append(model.get_grads())
        model.close()
    assert np.array_equal(outs[0], outs[1])


def test_error_paths_return_codes_without_trapping():
    cfg = TINY
    model = BD.GPT2(_bd_config(cfg, 2, 1, BD.GPT2_BF16), seed=1)
    x, y = S.token_batch(2, 2, 64, cfg.vocab_size)
    with pytest.raises(BD.Gpt2Error) as e:
        model.backward()                                   # no forward yet
    assert e.value.code == -8
    with pytest.raises(BD.Gpt2Error) as e:
        model.forward(cuda_i32(np.zeros((3, 64))), None)   # B > max_batch
    assert e.value.code == -4
    with pytest.raises(BD.Gpt2Error) as e:
        model.forward(cuda_i32(np.zeros((2, 65))), None)   # T > block_size
    assert e.value.code == -4
    bad = x.copy()
    bad[1, 5] = cfg.vocab_size + 3
    with pytest.raises(BD.Gpt2Error) as e:
        model.forward(cuda_i32(bad), cuda_i32(y))
    assert e.value.code == -5
    badt = y.copy()
    badt[0, 0] = -7
    with pytest.raises(BD.Gpt2Error) as e:
        model.forward(cuda_i32(x), cuda_i32(badt))
    assert e.value.code == -6
    # the context stays usable after reported errors
    loss = model.forward(cuda_i32(x), cuda_i32(y))
    assert abs(loss - math.log(cfg.padded_vocab_size)) < 0.2
    model.close()


def test_ignore_index_rows_are_left_out():
    cfg = TINY
    x, y = S.token_batch(2, 2, 64, cfg.vocab_size)
    y = y.copy()
    y[0, ::3] = -1
    params = O.init_params(cfg, 1, dtype=torch.float64)
    loss_ref, _ = O.forward(params, cfg, torch.from_numpy(x), torch.from_numpy(y))
    model = BD.GPT2(_bd_config(cfg, 2, 1, BD.GPT2_FP32), seed=1)
    model.set_params(O.flatten(params, cfg).numpy().astype(np.float32))
    loss = model.forward(cuda_i32(x), cuda_i32(y))
    model.close()
    assert abs(loss - float(loss_ref)) <= 1e-4 * float(loss_ref)


@pytest.mark.slow
def test_gpt2_124m_bf16_step_matches_fp32_oracle():
    """GPT-2 124M, B=4, T=1024: one bf16 forward + backward against the fp32 oracle."""
    cfg = O.GPT2_124M
    B, T = 4, 1024
    params = O.init_params(cfg, 1, dtype=torch.float32)
    x, y = S.token_batch(2, B, T, cfg.vocab_size)
    model = BD.GPT2(_bd_config(cfg, B, 1, BD.GPT2_BF16), seed=1)
    model.set_params(O.flatten(params, cfg).numpy())
    model.zero_grad()
    loss = model.forward(cuda_i32(x), cuda_i32(y))
    model.backward()
    grads = model.get_grads()
    am = model.get_argmax(B * T)
    model.close()
    loss_ref, cache = O.forward(params, cfg, torch.from_numpy(x), torch.from_numpy(y))
    grads_ref = O.backward(params, cfg, cache)
    assert abs(loss - float(loss_ref)) < 2e-2
    errs = _per_tensor(grads, grads_ref, cfg)
    assert max(errs.values()) < 2e-2, sorted(errs.items(), key=lambda kv: -kv[1])[:5]
    _check_argmax(am, cache["logits"])
