"""Top-k sampling (gpt2op_sample_top_k, gpt2_sample_top_k) against the oracle.

The kept ids are compared bit for bit.  The drawn id is decided by comparing u * total with
cumulative sums, fp32 in the kernel and fp64 in the oracle, so where u * total lies within a
small band of a cumulative boundary either neighbour is accepted."""
import numpy as np
import pytest
import torch

import oracle as O
from decoder_only_transformer_train_b200 import binding as BD
from decoder_only_transformer_train_b200 import synthetic as S
from gpu_common import cuda_i32, require_gpu

BAND = 1e-5


def _boundaries(z, kept):
    w = np.exp(np.array([float(z[i]) for i in kept]) - float(z[kept[0]]))
    cum = np.cumsum(w)
    return cum / cum[-1]


def _check_draw(z, k, u, got_tok, got_kept):
    tok, kept = O.sample_top_k(z, k, float(u))
    assert list(got_kept) == kept
    if got_tok == tok:
        return
    c = _boundaries(z, kept)
    j_ref, j_got = kept.index(tok), kept.index(got_tok)
    assert abs(j_ref - j_got) == 1, (tok, got_tok)
    edge = c[min(j_ref, j_got)]
    assert abs(float(u) - edge) < BAND, (float(u), edge)


def _run_op(logits, ld, n_rows, rows, u, V, k, prec):
    n = len(rows)
    kk = min(k, V)
    out = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    out_topk = torch.full((n, kk), -7, dtype=torch.int32, device="cuda")
    BD.sample_top_k(logits, ld, n_rows, cuda_i32(np.array(rows)), torch.from_numpy(u.astype(np.float32)).cuda(),
                    n, V, k, prec, out, out_topk)
    torch.cuda.synchronize()
    return out.cpu().numpy(), out_topk.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("k", [50, 1, 1024])
def test_sample_top_k_bf16_logits_full_vocabulary(k):
    """bf16 logits over the 50,257-token vocabulary in rows of the padded width 50,304;
    bf16's 8-bit mantissa makes ties among the largest logits common."""
    require_gpu()
    n_rows, V, ld = 6, 50257, 50304
    z = torch.from_numpy(S.normal(61, 3, n_rows * ld).reshape(n_rows, ld) * 2.0).to(torch.bfloat16)
    rows = [5, 0, 3, 3, 2, 1, 4, 0]
    u = S.uniform01(62, 4, len(rows))
    u[-1] = 0.0
    BD.device_error()
    out, out_topk = _run_op(z.cuda(), ld, n_rows, rows, u, V, k, BD.GPT2_BF16)
    assert BD.device_error() == 0
    zd = z.double()
    for i, r in enumerate(rows):
        _check_draw(zd[r, :V], k, u[i], int(out[i]), out_topk[i])


@pytest.mark.gpu
def test_sample_top_k_f32_ties_and_k_above_vocabulary():
    require_gpu()
    n_rows, V, ld = 3, 1000, 1004
    z = torch.from_numpy(np.floor(S.normal(63, 3, n_rows * ld).reshape(n_rows, ld) * 3.0)).float()
    rows = [0, 1, 2, 2]
    u = S.uniform01(64, 4, len(rows))
    out, out_topk = _run_op(z.cuda(), ld, n_rows, rows, u, V, 100, BD.GPT2_FP32)
    for i, r in enumerate(rows):
        _check_draw(z.double()[r, :V], 100, u[i], int(out[i]), out_topk[i])
    # k above the vocabulary keeps all of it, in order
    small = z[:, :20].contiguous()
    out, out_topk = _run_op(small.cuda(), 20, n_rows, rows, u, 20, 50, BD.GPT2_FP32)
    assert out_topk.shape == (4, 20)
    for i, r in enumerate(rows):
        _check_draw(small.double()[r], 50, u[i], int(out[i]), out_topk[i])


@pytest.mark.gpu
def test_sample_top_k_bad_row_is_reported():
    require_gpu()
    z = torch.zeros(2, 8, dtype=torch.float32, device="cuda")
    BD.device_error()
    out, out_topk = _run_op(z, 8, 2, [1, 2, -1], np.array([0.5, 0.5, 0.5]), 8, 3, BD.GPT2_FP32)
    assert BD.device_error() == -1   # GPT2_ERR_ARG
    assert out[0] == 1 and list(out_topk[0]) == [0, 1, 2]   # all equal: the lowest ids; u = 0.5 of 3 picks the second
    assert out[1] == -1 and out[2] == -1 and (out_topk[1:] == -1).all()


@pytest.mark.gpu
def test_model_sampling_after_a_forward_without_targets():
    """The last positions' logits of a fp32-mode forward with no targets: the kept ids match
    the oracle's on every row whose top k+1 oracle logits are separated by more than the
    fp32 error; a backward makes sampling a state error."""
    require_gpu()
    cfg = O.TINY
    B, T, k = 4, 64, 5
    params = O.init_params(cfg, 3, dtype=torch.float64)
    flat = O.flatten(params, cfg).numpy().astype(np.float32)
    params = O.unflatten(torch.from_numpy(flat).double(), cfg)
    x, y = S.token_batch(12, B, T, cfg.vocab_size)
    model = BD.GPT2(BD.Config(n_layer=cfg.n_layer, n_embd=cfg.n_embd, n_head=cfg.n_head, block_size=cfg.block_size,
                              vocab_size=cfg.vocab_size, padded_vocab_size=cfg.padded_vocab_size, max_batch=B,
                              grad_accum_steps=1, precision=BD.GPT2_FP32), seed=3)
    model.set_params(flat)
    model.forward(cuda_i32(x), None)
    rows_np = np.array([b * T + T - 1 for b in range(B)] + [5], dtype=np.int32)
    u = S.uniform01(13, 4, len(rows_np))
    out = torch.empty(len(rows_np), dtype=torch.int32, device="cuda")
    out_topk = torch.empty(len(rows_np), k, dtype=torch.int32, device="cuda")
    model.sample_top_k(cuda_i32(rows_np), torch.from_numpy(u.astype(np.float32)).cuda(), k, out, out_topk)
    model.synchronize()
    got, got_kept = out.cpu().numpy(), out_topk.cpu().numpy()
    assert ((got >= 0) & (got < cfg.vocab_size)).all()
    _, cache = O.forward(params, cfg, torch.from_numpy(x))
    z = cache["logits"].reshape(B * T, -1)[:, :cfg.vocab_size]
    checked = 0
    for i, r in enumerate(rows_np):
        top = torch.sort(z[r], descending=True).values[: k + 1]
        if float((top[:-1] - top[1:]).min()) > 1e-4:
            _check_draw(z[r], k, u[i], int(got[i]), got_kept[i])
            checked += 1
    assert checked >= 1
    # with targets, then a backward: the logits now hold their gradient
    model.forward(cuda_i32(x), cuda_i32(y))
    model.backward()
    with pytest.raises(BD.Gpt2Error, match="GPT2_ERR_STATE"):
        model.sample_top_k(cuda_i32(rows_np), torch.from_numpy(u.astype(np.float32)).cuda(), k, out, out_topk)
    model.close()


def test_sample_top_k_rejects_bad_arguments_before_any_cuda_call():
    lib = BD.lib()
    buf = np.zeros(16, dtype=np.float32)
    p = buf.ctypes.data
    shape, arg = -4, -1

    def call(prec=BD.GPT2_FP32, ld=8, n_rows=2, n=1, V=8, k=3, ptrs=(p, p, p, p)):
        return lib.gpt2op_sample_top_k(None, prec, ptrs[0], ld, n_rows, ptrs[1], ptrs[2], n, V, k, ptrs[3], None)

    assert call(k=0) == shape
    assert call(k=BD.SAMPLE_MAX_K + 1) == shape
    assert call(ld=7) == shape
    assert call(n=0) == shape and call(V=0) == shape and call(n_rows=0) == shape
    assert call(prec=5) == arg
    for j in range(4):
        ptrs = [p] * 4
        ptrs[j] = None
        assert call(ptrs=tuple(ptrs)) == arg
