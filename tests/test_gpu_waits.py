"""The bounded waits inside the pipelined kernels, made to run out on purpose.

Every mbarrier wait of the GEMM and attention kernels gives up after a time limit, records
GPT2_ERR_TIMEOUT in the device error word and ends the kernel in order, so that a broken
pipeline reports an error instead of hanging the GPU.  Here one self-test kernel waits, with a
1 ms limit, on barriers that nothing completes: a single lane, then a whole warp (whose lanes
must leave together).  No GPU fault, trap or endless loop is involved."""
import pytest
import torch

from decoder_only_transformer_train_b200 import binding as BD
from gpu_common import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_a_wait_nothing_ends_gives_up_and_reports_a_timeout():
    assert BD.device_error() == BD.GPT2_OK            # a clean error word to start from
    src = torch.arange(4, dtype=torch.int32, device="cuda")
    status = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    BD.bounded_wait_selftest(1_000_000, src, status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]                   # both the lane and the warp gave up
    assert BD.device_error() == -7                      # GPT2_ERR_TIMEOUT, read and cleared
    assert BD.device_error() == BD.GPT2_OK
    # the context is still usable: a tensor-core GEMM right after gives the right answer
    M = N = K = 128
    a = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    b = torch.randn(N, K, device="cuda").to(torch.bfloat16)
    c = torch.zeros(M, N, device="cuda", dtype=torch.float32)
    BD.gemm_bf16(a, b, c, M, N, K, K, K, N, epilogue=1)
    torch.cuda.synchronize()
    ref = a.double() @ b.double().T
    assert torch.allclose(c.double(), ref, rtol=1e-3, atol=1e-3)
    assert BD.device_error() == BD.GPT2_OK


def test_selftest_refuses_bad_arguments():
    src = torch.zeros(4, dtype=torch.int32, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    for limit in (0, -1, 2_000_000_000):
        with pytest.raises(BD.Gpt2Error) as e:
            BD.bounded_wait_selftest(limit, src, status)
        assert e.value.code == -1
    with pytest.raises(BD.Gpt2Error) as e:
        BD.bounded_wait_selftest(1_000_000, src[1:], status)    # not 16-byte aligned
    assert e.value.code == -1
