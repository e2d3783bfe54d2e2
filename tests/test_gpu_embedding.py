"""Embedding forward and backward kernels (gpt2op_embedding_*) against the oracle.

The backward's sort keys must equal the stable (token, position) order bit for bit; the
sums are fp32 in a fixed order, so dwte and dwpe are compared with the fp64 oracle within
a bound on fp32 summation error and must repeat bit for bit from call to call."""
import numpy as np
import pytest
import torch

import oracle as O
from decoder_only_transformer_train_b200 import binding as BD
from decoder_only_transformer_train_b200 import synthetic as S
from gpu_common import cuda_i32, rel_l2, require_gpu

V = 50257


def _tokens(kind, B, T, seed):
    n = B * T
    if kind == "zipf":        # heavy head: token 0 holds about a ninth of the positions
        return S.zipf_tokens(seed, n, V).reshape(B, T)
    if kind == "same":        # one run over every chunk
        return np.full((B, T), 17, dtype=np.int32)
    if kind == "uniform":
        return S.uniform_targets(seed, n, V).reshape(B, T)
    if kind == "clamped":     # ids outside [0, V) are clamped by the backward
        t = S.zipf_tokens(seed, n, V).reshape(B, T).copy()
        t.reshape(-1)[::7] = -3
        t.reshape(-1)[3::11] = V + 5
        return t
    raise ValueError(kind)


def _run_bwd(tok, dx0, dwte0, dwpe0, B, T, C):
    tok_d = cuda_i32(tok.reshape(-1))
    dx_d = dx0.float().cuda()
    dwte = dwte0.float().cuda()
    dwpe = dwpe0.float().cuda()
    ws = torch.zeros(BD.embedding_bwd_ws_bytes(B * T, C), dtype=torch.uint8, device="cuda")
    BD.embedding_bwd(tok_d, dx_d, dwte, dwpe, B, T, C, V, ws)
    torch.cuda.synchronize()
    assert BD.device_error() == 0
    keys = ws[: 8 * B * T].view(torch.int64).cpu().numpy().view(np.uint64)
    return dwte.cpu(), dwpe.cpu(), keys


CASES = [
    ("zipf", 16, 1024, 768),     # the training step's shape: 512 chunks, runs over ~60 chunks
    ("zipf", 3, 77, 64),         # ragged: a partial last chunk, one thread per 4 channels
    ("zipf", 1, 1, 32),          # a single position
    ("uniform", 2, 513, 128),    # 1026 keys: the two-keys-per-thread sort
    ("same", 4, 1024, 96),       # one run through all 128 chunks (several ballot rounds)
    ("clamped", 5, 700, 1032),   # C above 1024: two column blocks
    ("zipf", 32, 1024, 64),      # 32768 keys: eight sorted segments merged
    ("uniform", 3, 5001, 32),    # a ragged last segment (15003 keys, 4 segments)
    ("zipf", 32, 2048, 64),      # 65536 keys: the GPT-3 context at B = 32, sixteen segments
]


@pytest.mark.gpu
@pytest.mark.parametrize("kind,B,T,C", CASES)
def test_embedding_bwd_matches_oracle(kind, B, T, C):
    require_gpu()
    tok = _tokens(kind, B, T, seed=40 + B + T)
    g = torch.Generator().manual_seed(B * 1000 + T)
    dx0 = torch.randn(B, T, C, generator=g, dtype=torch.float64).float().double()
    dwte0 = torch.randn(V, C, generator=g, dtype=torch.float64).float().double() * 0.01
    dwpe0 = torch.randn(T + 3, C, generator=g, dtype=torch.float64).float().double() * 0.01
    dwte, dwpe, keys = _run_bwd(tok, dx0, dwte0, dwpe0, B, T, C)

    # keys: the stable order of the clamped ids, bit for bit
    clamped = np.clip(tok.reshape(-1).astype(np.int64), 0, V - 1)
    order = np.argsort(clamped, kind="stable")
    want = ((clamped[order].astype(np.uint64) << np.uint64(32)) | order.astype(np.uint64))
    assert np.array_equal(keys, want)

    grads = {"wte": dwte0.clone(), "wpe": dwpe0.clone()}
    O.encoder_backward(grads, torch.from_numpy(clamped.reshape(B, T)), dx0)
    # fp32 sums of up to n terms: |error| <= n * 2^-24 * sum |terms| (plus the initial value)
    counts = np.bincount(clamped, minlength=V)
    abs_wte = torch.zeros(V, C, dtype=torch.float64)
    abs_wte.index_add_(0, torch.from_numpy(clamped), dx0.abs().reshape(B * T, C))
    bound_wte = (torch.from_numpy(counts).double()[:, None] + 1) * 2.0 ** -24 * (abs_wte + dwte0.abs()) + 1e-30
    assert bool(((dwte.double() - grads["wte"]).abs() <= bound_wte).all())
    bound_wpe = (B + 1) * 2.0 ** -24 * (dx0.abs().sum(0) + dwpe0[:T].abs()) + 1e-30
    assert bool(((dwpe[:T].double() - grads["wpe"][:T]).abs() <= bound_wpe).all())
    assert torch.equal(dwpe[T:], dwpe0[T:].float()), "rows of wpe past T must not change"
    untouched = torch.from_numpy(counts == 0)
    assert torch.equal(dwte[untouched], dwte0[untouched].float())
    assert rel_l2(dwte, grads["wte"]) < 1e-6

    # bit-for-bit repeat
    dwte2, dwpe2, keys2 = _run_bwd(tok, dx0, dwte0, dwpe0, B, T, C)
    assert torch.equal(dwte2, dwte) and torch.equal(dwpe2, dwpe) and np.array_equal(keys2, keys)


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,C", [(16, 1024, 768), (3, 77, 64), (2, 5, 1032)])
def test_embedding_fwd_matches_oracle(B, T, C):
    require_gpu()
    tok = _tokens("zipf", B, T, seed=90 + T)
    g = torch.Generator().manual_seed(T)
    wte = torch.randn(V, C, generator=g).float()
    wpe = torch.randn(T + 2, C, generator=g).float()
    x = torch.empty(B * T, C, dtype=torch.float32, device="cuda")
    BD.embedding_fwd(cuda_i32(tok.reshape(-1)), wte.cuda(), wpe.cuda(), x, B, T, C, V)
    torch.cuda.synchronize()
    assert BD.device_error() == 0
    want = O.encoder_forward(wte.double(), wpe.double(), torch.from_numpy(tok)).reshape(B * T, C)
    # one fp32 addition: the result is the exact sum rounded once
    assert torch.equal(x.cpu(), want.float())


@pytest.mark.gpu
def test_embedding_fwd_reports_bad_ids_and_writes_zero_rows():
    require_gpu()
    B, T, C = 2, 40, 64
    tok = _tokens("zipf", B, T, seed=5)
    tok.reshape(-1)[[3, 50]] = [-1, V]
    wte = torch.randn(V, C).float().cuda()
    wpe = torch.randn(T, C).float().cuda()
    x = torch.full((B * T, C), 7.0, device="cuda")
    BD.device_error()   # clear
    BD.embedding_fwd(cuda_i32(tok.reshape(-1)), wte, wpe, x, B, T, C, V)
    torch.cuda.synchronize()
    assert BD.device_error() == -5   # GPT2_ERR_TOKEN
    xc = x.cpu()
    assert float(xc[[3, 50]].abs().sum()) == 0.0
    good = [i for i in range(B * T) if i not in (3, 50)]
    assert bool(torch.isfinite(xc[good]).all()) and float(xc[good].abs().sum()) > 0


def test_embedding_entry_points_reject_bad_shapes_before_any_cuda_call():
    lib = BD.lib()
    buf = np.zeros(64, dtype=np.float32)
    p = (buf.ctypes.data + 15) // 16 * 16
    err_shape, err_arg = -4, -1
    assert lib.gpt2op_embedding_bwd(None, p, p, p, p, 64, 2049, 64, V, p) == err_shape   # > 131072 positions
    assert lib.gpt2op_embedding_bwd(None, p, p, p, p, 2, 8, 66, V, p) == err_shape       # C % 4
    assert lib.gpt2op_embedding_bwd(None, p, p, p, p, 0, 8, 64, V, p) == err_shape
    assert lib.gpt2op_embedding_bwd(None, p, p, p, p, 2, 8, 64, V, None) == err_arg
    assert lib.gpt2op_embedding_fwd(None, p, p, p, p, 2, 8, 62, V) == err_shape
    assert lib.gpt2op_embedding_fwd(None, None, p, p, p, 2, 8, 64, V) == err_arg
    # sorted keys (uint64), segment keys (uint32), chunk partials: each on a 256-byte boundary
    assert BD.embedding_bwd_ws_bytes(16384, 768) == 16384 * 8 + 16384 * 4 + 512 * 2 * 768 * 4
    assert BD.embedding_bwd_ws_bytes(77, 64) == 768 + 512 + 3 * 2 * 64 * 4
    # 16-byte accesses: a misaligned table, output or gradient is refused before any launch
    q = p + 4
    assert lib.gpt2op_embedding_fwd(None, p, q, p, p, 2, 8, 64, V) == err_arg
    assert lib.gpt2op_embedding_fwd(None, p, p, p, q, 2, 8, 64, V) == err_arg
    assert lib.gpt2op_embedding_bwd(None, p, q, p, p, 2, 8, 64, V, p) == err_arg
    assert lib.gpt2op_embedding_bwd(None, p, p, p, p, 2, 8, 64, V, q) == err_arg
