"""Kernel-level parity on a B200: each CUDA operation through the C ABI against the CPU
oracle (or, for the GEMM, the plain fp64 matrix product that defines it) on the same
seeded inputs, at sizes that span several tiles and leave ragged tails."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from decoder_only_transformer_train_b200 import binding as BD
from decoder_only_transformer_train_b200 import synthetic as S
from gpu_common import bf16_round, pad8, rel_l2, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _randn(shape, seed, scale=1.0):
    n = int(np.prod(shape))
    return torch.from_numpy(S.normal(seed, 11, n).reshape(shape) * scale)


# ------------------------------------------------------------------ GEMM
@pytest.fixture(params=["0", "1", "default"], ids=["cta", "cta_pair", "cost_model"])
def gemm_pairs(request, monkeypatch):
    """Every GEMM test runs three times: with one CTA per 128-row tile, with CTA pairs
    (tcgen05 cta_group::2, 256-row tiles) wherever the shape allows them, and with the
    launcher's own choice (what the training step runs)."""
    if request.param == "default":
        monkeypatch.delenv("GPT2_B200_GEMM_PAIRS", raising=False)
    else:
        monkeypatch.setenv("GPT2_B200_GEMM_PAIRS", request.param)
    return request.param


GEMM_SHAPES = [(128, 256, 64), (300, 200, 136), (1000, 768, 768), (129, 1000, 320), (64, 64, 16)]
LAYOUTS = [(False, False), (False, True), (True, True)]


def _layout(X, mn_major):
    """X logical [rows, K]; K-major stores X, MN-major stores X^T, rows padded to 8."""
    if mn_major:
        K, R = X.shape[1], X.shape[0]
        buf = torch.zeros(K, pad8(R), dtype=torch.bfloat16)
        buf[:, :R] = X.T.to(torch.bfloat16)
        return buf.cuda(), pad8(R)
    R, K = X.shape
    buf = torch.zeros(R, pad8(K), dtype=torch.bfloat16)
    buf[:, :K] = X.to(torch.bfloat16)
    return buf.cuda(), pad8(K)


@pytest.mark.parametrize("a_mn,b_mn", LAYOUTS)
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_bf16_all_layouts_and_epilogues(a_mn, b_mn, M, N, K, gemm_pairs):
    A = bf16_round(_randn((M, K), M + 3 * K))
    Bm = bf16_round(_randn((N, K), N + 5 * K))
    bias = _randn((N,), 17).float()
    ref = A @ Bm.T                                   # fp64 product of the bf16 operands
    Ad, lda = _layout(A, a_mn)
    Bd, ldb = _layout(Bm, b_mn)
    biasd = bias.cuda()
    ldc = pad8(N)
    # epilogue 0: bf16 out with bias
    C0 = torch.zeros(M, ldc, dtype=torch.bfloat16, device="cuda")
    BD.gemm_bf16(Ad, Bd, C0, M, N, K, lda, ldb, ldc, a_mn, b_mn, epilogue=0, bias=biasd)
    # epilogue 1: fp32 out, alpha
    C1 = torch.zeros(M, ldc, dtype=torch.float32, device="cuda")
    BD.gemm_bf16(Ad, Bd, C1, M, N, K, lda, ldb, ldc, a_mn, b_mn, epilogue=1, alpha=0.5)
    # epilogue 2: accumulate into existing values
    base = _randn((M, ldc), 23).float()
    C2 = base.clone().cuda()
    BD.gemm_bf16(Ad, Bd, C2, M, N, K, lda, ldb, ldc, a_mn, b_mn, epilogue=2, alpha=2.0)
    torch.cuda.synchronize()
    assert BD.device_error() == 0
    r0 = ref + bias.double()
    assert rel_l2(C0[:, :N].cpu(), r0) < 4e-3
    assert rel_l2(C1[:, :N].cpu(), 0.5 * ref) < 2e-5
    assert rel_l2(C2[:, :N].cpu() - base[:, :N], 2.0 * ref) < 2e-5
    # nothing written outside the logical N columns
    if ldc > N:
        assert torch.all(C1[:, N:] == 0)


FUSED_SHAPES = [(300, 200, 136), (1000, 768, 768), (129, 1000, 320), (512, 3072, 768)]


@pytest.mark.parametrize("b_mn", [False, True])
@pytest.mark.parametrize("M,N,K", FUSED_SHAPES)
def test_gemm_bf16_fused_epilogues(b_mn, M, N, K, gemm_pairs):
    """Residual add, GELU (keeping gelu'(u) for the backward) and the GELU-gradient product
    epilogues against their definitions on the fp64 product of the same bf16 operands."""
    A = bf16_round(_randn((M, K), 91 + M))
    Bm = bf16_round(_randn((N, K), 93 + N))
    bias = _randn((N,), 95).float()
    ref = A @ Bm.T
    Ad, lda = _layout(A, False)
    Bd, ldb = _layout(Bm, b_mn)
    ldc = pad8(N)
    # epilogue 3: C = aux + alpha D + bias, out of place and in place
    aux = _randn((M, ldc), 97).float()
    C3 = torch.zeros(M, ldc, dtype=torch.float32, device="cuda")
    auxd = aux.cuda()
    BD.gemm_bf16_fused(Ad, Bd, C3, M, N, K, lda, ldb, ldc, False, b_mn, 3, bias=bias.cuda(), alpha=0.5, aux=auxd,
                       ld_aux=ldc)
    inplace = aux.clone().cuda()
    BD.gemm_bf16_fused(Ad, Bd, inplace, M, N, K, lda, ldb, ldc, False, b_mn, 3, bias=bias.cuda(), alpha=0.5,
                       aux=inplace, ld_aux=ldc)
    # epilogue 4: u = D + bias, gelu'(u) kept in aux_out, C = gelu(u)
    U = torch.zeros(M, ldc, dtype=torch.bfloat16, device="cuda")
    G = torch.zeros(M, ldc, dtype=torch.bfloat16, device="cuda")
    BD.gemm_bf16_fused(Ad, Bd, G, M, N, K, lda, ldb, ldc, False, b_mn, 4, bias=bias.cuda(), aux_out=U, ld_aux_out=ldc)
    # epilogue 5: C = D * aux for a bf16 aux (the kept gelu'(u) of some pre-activation u)
    u_in = bf16_round(O.gelu_tanh_grad(_randn((M, ldc), 99) * 2.0))
    DG = torch.zeros(M, ldc, dtype=torch.bfloat16, device="cuda")
    BD.gemm_bf16_fused(Ad, Bd, DG, M, N, K, lda, ldb, ldc, False, b_mn, 5, aux=u_in.to(torch.bfloat16).cuda(),
                       ld_aux=ldc)
    torch.cuda.synchronize()
    assert BD.device_error() == 0
    r3 = aux[:, :N].double() + 0.5 * ref + bias.double()
    assert rel_l2(C3[:, :N].cpu(), r3) < 2e-5
    assert torch.equal(C3[:, :N].cpu(), inplace[:, :N].cpu())
    u_ref = ref + bias.double()
    assert rel_l2(U[:, :N].cpu(), O.gelu_tanh_grad(u_ref)) < 5e-3
    assert rel_l2(G[:, :N].cpu(), O.gelu_tanh(u_ref)) < 5e-3
    assert rel_l2(DG[:, :N].cpu(), ref * u_in[:, :N].double()) < 5e-3
    if ldc > N:   # nothing written past the logical N columns
        assert torch.all(G[:, N:] == 0) and torch.all(U[:, N:] == 0) and torch.all(DG[:, N:] == 0)


def test_gemm_split_k_weight_gradient_shape_is_deterministic(gemm_pairs):
    """dW += dY^T X with K = 16384 tokens (few output tiles, long K: split-K path)."""
    M, N, K = 768, 768, 16384
    dY = bf16_round(_randn((M, K), 31))      # logical A [M, K], stored MN-major like a [tokens, out] buffer
    X = bf16_round(_randn((N, K), 37))
    Ad, lda = _layout(dY, True)
    Bd, ldb = _layout(X, True)
    ws = torch.empty(8 * M * N, dtype=torch.float32, device="cuda")
    outs = []
    for _ in range(2):
        C = torch.ones(M, N, dtype=torch.float32, device="cuda")
        BD.gemm_bf16(Ad, Bd, C, M, N, K, lda, ldb, N, True, True, epilogue=2, alpha=1.0 / 16, workspace=ws)
        outs.append(C)
    torch.cuda.synchronize()
    ref = (dY @ X.T) / 16 + 1.0
    assert rel_l2(outs[0].cpu(), ref) < 2e-5
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("M,N,K", [(3072, 768, 4096), (2304, 768, 4096), (768, 3072, 4096), (768, 768, 8192)])
def test_gemm_weight_gradient_shapes_tile_choices(M, N, K, gemm_pairs):
    """dW += dY^T X on the weight-gradient shapes, where the launcher picks 128/192/256-wide
    tiles and split-K by its cost model."""
    dY = bf16_round(_randn((M, K), 71 + M))
    X = bf16_round(_randn((N, K), 73 + N))
    Ad, lda = _layout(dY, True)
    Bd, ldb = _layout(X, True)
    ws = torch.empty(8 * 4 * 768 * 768, dtype=torch.float32, device="cuda")
    C = torch.full((M, N), 0.25, dtype=torch.float32, device="cuda")
    BD.gemm_bf16(Ad, Bd, C, M, N, K, lda, ldb, N, True, True, epilogue=2, alpha=0.5, workspace=ws)
    torch.cuda.synchronize()
    assert rel_l2(C.cpu() - 0.25, 0.5 * (dY @ X.T)) < 2e-5


# ------------------------------------------------------------------ attention
ATTN_CASES = [(2, 64, 4, 16), (1, 200, 2, 64), (2, 256, 3, 64), (1, 1, 2, 64), (3, 130, 1, 32), (2, 1024, 12, 64),
              (3, 384, 100, 64)]


@pytest.mark.parametrize("prec", [BD.GPT2_FP32, BD.GPT2_BF16])
@pytest.mark.parametrize("B,T,H,hd", ATTN_CASES)
def test_attention_forward_backward(prec, B, T, H, hd):
    C = H * hd
    qkv = _randn((B * T, 3 * C), 41 + T)
    dout = _randn((B * T, C), 43 + T)
    if prec == BD.GPT2_BF16:
        qkv, dout = bf16_round(qkv), bf16_round(dout)
    heads = lambda t: t.reshape(B, T, H, hd).transpose(1, 2)
    q, k, v = (heads(t) for t in qkv.split(C, dim=1))
    o_ref, p = O.causal_attention_forward(q, k, v)
    dq, dk, dv = O.causal_attention_backward(heads(dout), q, k, v, p)
    merge = lambda t: t.transpose(1, 2).reshape(B * T, C)
    lse_ref = torch.logsumexp(
        (q @ k.transpose(-1, -2) / math.sqrt(hd)).masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1),
                                                              float("-inf")), dim=-1)
    dt = torch.bfloat16 if prec == BD.GPT2_BF16 else torch.float32
    qkv_d, dout_d = qkv.to(dt).cuda(), dout.to(dt).cuda()
    out_d = torch.zeros(B * T, C, dtype=dt, device="cuda")
    lse_d = torch.zeros(B * H * T, dtype=torch.float32, device="cuda")
    Dbuf = torch.zeros(B * H * T, dtype=torch.float32, device="cuda")
    dqkv_d = torch.zeros(B * T, 3 * C, dtype=dt, device="cuda")
    BD.attention_fwd(qkv_d, out_d, lse_d, B, T, H, hd, prec)
    BD.attention_bwd(qkv_d, out_d, dout_d, lse_d, Dbuf, dqkv_d, B, T, H, hd, prec)
    torch.cuda.synchronize()
    assert BD.device_error() == 0
    tol_o, tol_g = (1e-5, 1e-4) if prec == BD.GPT2_FP32 else (5e-3, 2e-2)
    assert rel_l2(out_d.cpu(), merge(o_ref)) < tol_o
    assert torch.allclose(lse_d.cpu().double(), lse_ref.reshape(-1), atol=1e-4)
    g = dqkv_d.cpu()
    assert rel_l2(g[:, :C], merge(dq)) < tol_g
    assert rel_l2(g[:, C:2 * C], merge(dk)) < tol_g
    assert rel_l2(g[:, 2 * C:], merge(dv)) < tol_g


@pytest.mark.parametrize("prec", [BD.GPT2_FP32, BD.GPT2_BF16])
@pytest.mark.parametrize("B,T,H", [(2, 1024, 3), (1, 700, 2)])
def test_attention_forward_when_the_row_max_keeps_growing(prec, B, T, H):
    """Keys scaled up along the sequence (and queries by 3) make a row's max grow by more
    than the kernel's rescale threshold from one key tile to the next, so the accumulated
    output is rescaled and the tile's probabilities recomputed many times per row."""
    hd = 64
    C = H * hd
    qkv = _randn((B * T, 3 * C), 97 + T)
    pos = torch.arange(B * T, dtype=torch.float64) % T
    qkv[:, :C] *= 3.0
    qkv[:, C:2 * C] *= (1.0 + pos / 64.0)[:, None]
    if prec == BD.GPT2_BF16:
        qkv = bf16_round(qkv)
    heads = lambda t: t.reshape(B, T, H, hd).transpose(1, 2)
    q, k, v = (heads(t) for t in qkv.split(C, dim=1))
    o_ref, _ = O.causal_attention_forward(q, k, v)
    lse_ref = torch.logsumexp(
        (q @ k.transpose(-1, -2) / math.sqrt(hd)).masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1),
                                                              float("-inf")), dim=-1)
    dt = torch.bfloat16 if prec == BD.GPT2_BF16 else torch.float32
    out_d = torch.zeros(B * T, C, dtype=dt, device="cuda")
    lse_d = torch.zeros(B * H * T, dtype=torch.float32, device="cuda")
    BD.attention_fwd(qkv.to(dt).cuda(), out_d, lse_d, B, T, H, hd, prec)
    torch.cuda.synchronize()
    assert BD.device_error() == 0
    merge = lambda t: t.transpose(1, 2).reshape(B * T, C)
    assert rel_l2(out_d.cpu(), merge(o_ref)) < (1e-5 if prec == BD.GPT2_FP32 else 5e-3)
    assert torch.allclose(lse_d.cpu().double(), lse_ref.reshape(-1), rtol=1e-5, atol=1e-4)


# ------------------------------------------------------------------ LayerNorm
@pytest.mark.parametrize("prec", [BD.GPT2_FP32, BD.GPT2_BF16])
@pytest.mark.parametrize("N,C", [(77, 64), (1000, 768), (33, 1024)])
def test_layernorm_forward(prec, N, C):
    x = _randn((N, C), 51) * 2 + 0.5
    w = _randn((C,), 52) * 0.3 + 1
    b = _randn((C,), 53) * 0.1
    y_ref, m_ref, r_ref = O.layernorm_forward(x, w, b)
    dt = torch.bfloat16 if prec == BD.GPT2_BF16 else torch.float32
    y = torch.zeros(N, C, dtype=dt, device="cuda")
    mean = torch.zeros(N, device="cuda")
    rstd = torch.zeros(N, device="cuda")
    BD.layernorm_fwd(x.float().cuda(), w.float().cuda(), b.float().cuda(), y, mean, rstd, N, C, prec)
    torch.cuda.synchronize()
    assert rel_l2(y.cpu(), y_ref) < (1e-6 if prec == BD.GPT2_FP32 else 4e-3)
    assert rel_l2(mean.cpu(), m_ref) < 1e-6
    assert rel_l2(rstd.cpu(), r_ref) < 1e-5


# ------------------------------------------------------------------ classifier head
@pytest.mark.parametrize("N,V,C", [(256, 1000, 64), (384, 50304, 768), (130, 50257, 768)])
def test_classifier_head_forward_backward(N, V, C, gemm_pairs):
    """lm_head + softmax + cross-entropy: loss, lse, argmax, dh and dW."""
    h = bf16_round(_randn((N, C), 61))
    W = bf16_round(_randn((V, C), 62, scale=0.02))
    tg = S.uniform_targets(63, N, V)
    tg[S.ignore_mask(64, N, 0.05)] = -1
    tgt = torch.from_numpy(tg.astype(np.int64))
    logits = h @ W.T
    loss_ref, lse_ref, count = O.cross_entropy_forward(logits, tgt)
    dz = O.cross_entropy_backward(logits, tgt, lse_ref, count, 1.0)
    dh_ref = dz @ W
    dW_ref = dz.T @ h
    ldl = pad8(V)
    logits_ws = torch.empty(N, ldl, dtype=torch.bfloat16, device="cuda")
    aux = torch.empty(BD.classifier_aux_floats(N, V), dtype=torch.float32, device="cuda")
    loss = torch.zeros(1, device="cuda")
    lse = torch.zeros(N, device="cuda")
    am = torch.zeros(N, dtype=torch.int32, device="cuda")
    dh = torch.zeros(N, C, device="cuda")
    dW = torch.zeros(V, C, device="cuda")
    BD.classifier_fwd_bwd(h.to(torch.bfloat16).cuda(), W.to(torch.bfloat16).cuda(),
                          torch.from_numpy(tg).cuda(), N, V, C, logits_ws, ldl, aux, loss, lse, am, dh, dW)
    torch.cuda.synchronize()
    assert BD.device_error() == 0
    assert abs(float(loss) - float(loss_ref)) < 1e-4
    assert torch.allclose(lse.cpu().double(), lse_ref, atol=1e-4)
    # argmax: bit-exact wherever the reference top-2 gap exceeds the fp32 accumulation error
    top2 = torch.topk(logits, 2, dim=1).values
    clear = (top2[:, 0] - top2[:, 1]) > 1e-4
    am_ref = O.argmax_lowest(logits)
    assert torch.equal(am.cpu()[clear], am_ref[clear])
    assert int(clear.sum()) > 0.9 * N
    assert rel_l2(dh.cpu(), dh_ref) < 2e-2
    assert rel_l2(dW.cpu(), dW_ref) < 2e-2
