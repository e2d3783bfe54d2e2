"""Helpers shared by the GPU parity tests (no arithmetic of the method here)."""
import numpy as np
import torch


def rel_l2(a, b) -> float:
    a = torch.as_tensor(a).double().reshape(-1)
    b = torch.as_tensor(b).double().reshape(-1)
    nb = float(b.norm())
    return float((a - b).norm()) / (nb if nb > 0 else 1.0)


def pad8(n: int) -> int:
    return (n + 7) // 8 * 8


def bf16_round(t: torch.Tensor) -> torch.Tensor:
    """Round to bf16 (nearest even) and back to the input dtype."""
    return t.to(torch.bfloat16).to(t.dtype)


def require_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    from decoder_only_transformer_train_b200 import binding
    binding.lib()   # raises if the CUDA library is missing: no fallback


def cuda_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
