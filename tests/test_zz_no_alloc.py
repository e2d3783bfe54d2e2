"""gpt2op_attention_bwd_noalloc (row sums in the library's fixed array) against the
caller-scratch gpt2op_attention_bwd: the same kernels run on the same inputs, so the
gradients must agree bit for bit, call after call, while the fixed array is reused."""
import numpy as np
import pytest
import torch

from decoder_only_transformer_train_b200 import binding as BD
from decoder_only_transformer_train_b200 import synthetic as S
from gpu_common import bf16_round, require_gpu

ERR = {name: code for code, name in BD.ERRORS.items()}


def _inputs(B, T, H, hd, prec, seed):
    C = H * hd
    n = B * T
    qkv = torch.from_numpy(S.normal(seed, 11, n * 3 * C).reshape(n, 3 * C))
    dout = torch.from_numpy(S.normal(seed + 1, 11, n * C).reshape(n, C))
    if prec == BD.GPT2_BF16:
        qkv, dout = bf16_round(qkv), bf16_round(dout)
    dt = torch.bfloat16 if prec == BD.GPT2_BF16 else torch.float32
    qkv_d, dout_d = qkv.to(dt).cuda(), dout.to(dt).cuda()
    out_d = torch.zeros(n, C, dtype=dt, device="cuda")
    lse_d = torch.zeros(B * H * T, dtype=torch.float32, device="cuda")
    BD.attention_fwd(qkv_d, out_d, lse_d, B, T, H, hd, prec)
    return qkv_d, out_d, dout_d, lse_d


def _both(B, T, H, hd, prec, seed):
    """dqkv from the caller-scratch entry point, then from the no-allocation one; also
    the device's free memory just before and after the no-allocation call."""
    qkv_d, out_d, dout_d, lse_d = _inputs(B, T, H, hd, prec, seed)
    dqkv_ref = torch.zeros_like(qkv_d)
    Dbuf = torch.zeros(B * H * T, dtype=torch.float32, device="cuda")
    BD.attention_bwd(qkv_d, out_d, dout_d, lse_d, Dbuf, dqkv_ref, B, T, H, hd, prec)
    dqkv = torch.zeros_like(qkv_d)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    BD.attention_bwd_noalloc(qkv_d, out_d, dout_d, lse_d, dqkv, B, T, H, hd, prec)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert BD.device_error() == 0
    return dqkv_ref, dqkv, free_before, free_after


# Each sequence runs back to back in one test: the second call finds the fixed array
# holding the first call's row sums, and a larger second call covers rows the first
# never wrote.
SEQUENCES = [
    (BD.GPT2_BF16, [(3, 200, 4, 64), (2, 384, 12, 64)]),
    (BD.GPT2_FP32, [(1, 130, 3, 32), (2, 256, 2, 64)]),
    # the full training-step shape (B=16, T=1024, 12 heads of 64), then exactly the maximum
    (BD.GPT2_BF16, [(16, 1024, 12, 64), (16, 1024, 16, 64)]),
]


@pytest.mark.gpu
@pytest.mark.parametrize("prec,cases", SEQUENCES)
def test_noalloc_matches_scratch_entry_point_twice(prec, cases):
    require_gpu()
    for i, (B, T, H, hd) in enumerate(cases):
        assert B * H * T <= BD.NOALLOC_ATTN_MAX_ROWS
        ref, got, free_before, free_after = _both(B, T, H, hd, prec, seed=700 + 10 * i + T)
        assert torch.equal(got, ref), f"call {i + 1} of {cases} differs from the caller-scratch entry point"
        assert bool(torch.isfinite(got.float()).all())
        if i > 0:   # the address lookup of a device's first call is done by then
            assert free_after == free_before, "the no-allocation entry point changed the device's free memory"


def test_noalloc_rejects_before_any_cuda_call():
    """Argument and size errors come back before any CUDA call, so this needs no GPU:
    the pointers are host addresses that are never dereferenced."""
    lib = BD.lib()
    buf = np.zeros(16, dtype=np.float32)
    p = buf.ctypes.data
    max_rows = BD.NOALLOC_ATTN_MAX_ROWS

    def call(prec=BD.GPT2_BF16, B=1, T=64, H=1, hd=64, ptrs=(p, p, p, p, p)):
        return lib.gpt2op_attention_bwd_noalloc(None, prec, *ptrs, B, T, H, hd)

    # one row past the maximum, in several factorings
    assert call(B=1, T=max_rows + 1, H=1) == ERR["GPT2_ERR_SHAPE"]
    assert call(B=16, T=1024, H=17) == ERR["GPT2_ERR_SHAPE"]
    assert call(B=max_rows, T=2, H=1) == ERR["GPT2_ERR_SHAPE"]
    # B*H*T overflowing 32 bits must not wrap into range
    assert call(B=65536, T=65536, H=1) == ERR["GPT2_ERR_SHAPE"]
    for bad in (dict(B=0), dict(T=0), dict(H=0), dict(hd=0), dict(B=-1)):
        assert call(**bad) == ERR["GPT2_ERR_SHAPE"]
    assert call(prec=7) == ERR["GPT2_ERR_ARG"]
    for k in range(5):
        ptrs = [p] * 5
        ptrs[k] = None
        assert call(ptrs=tuple(ptrs)) == ERR["GPT2_ERR_ARG"]
    with pytest.raises(BD.Gpt2Error, match="exceeds the fixed scratch"):
        BD.attention_bwd_noalloc(buf, buf, buf, buf, buf, 16, 1024, 17, 64, BD.GPT2_BF16, stream=0)
