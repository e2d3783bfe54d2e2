"""ctypes binding of libgpt2_b200.so (include/gpt2_b200.h): argument marshalling only.

Every step of the training path runs in the library's CUDA kernels; PyTorch supplies
device memory (tensor data pointers) and streams.  There is no fallback: if the built
library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgpt2_b200.so")

GPT2_OK = 0
GPT2_FP32 = 0
GPT2_BF16 = 1
ERRORS = {-1: "GPT2_ERR_ARG", -2: "GPT2_ERR_OOM", -3: "GPT2_ERR_CUDA", -4: "GPT2_ERR_SHAPE",
          -5: "GPT2_ERR_TOKEN", -6: "GPT2_ERR_TARGET", -7: "GPT2_ERR_TIMEOUT", -8: "GPT2_ERR_STATE"}


class Gpt2Error(RuntimeError):
    def __init__(self, code: int, msg: str = ""):
        self.code = code
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")


class gpt2_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("n_layer", "n_embd", "n_head", "block_size", "vocab_size",
                                            "padded_vocab_size", "max_batch", "grad_accum_steps", "precision")]


_vp, _i, _i64, _f, _u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_uint64
_fp = ctypes.POINTER(ctypes.c_float)

_PROTOS = {
    "gpt2_create": (_i, [ctypes.POINTER(gpt2_config), _u64, ctypes.POINTER(_vp)]),
    "gpt2_destroy": (None, [_vp]),
    "gpt2_set_stream": (_i, [_vp, _vp]),
    "gpt2_set_graphs": (_i, [_vp, _i]),
    "gpt2_forward": (_i, [_vp, _vp, _vp, _i, _i, _fp]),
    "gpt2_forward_host": (_i, [_vp, _vp, _vp, _i, _i, _fp]),
    "gpt2_backward": (_i, [_vp]),
    "gpt2_zero_grad": (_i, [_vp]),
    "gpt2_get_grad_buffer": (_i, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_i64)]),
    "gpt2_adamw_step": (_i, [_vp, _f, _f, _f, _f, _f, _f, _fp]),
    "gpt2_num_params": (_i64, [_vp]),
    "gpt2_get_params": (_i, [_vp, _vp]),
    "gpt2_set_params": (_i, [_vp, _vp]),
    "gpt2_get_grads": (_i, [_vp, _vp]),
    "gpt2_get_optimizer_state": (_i, [_vp, _vp, _vp, ctypes.POINTER(ctypes.c_int64)]),
    "gpt2_set_optimizer_state": (_i, [_vp, _vp, _vp, _i64]),
    "gpt2_get_argmax": (_i, [_vp, _vp]),
    "gpt2_get_lse": (_i, [_vp, _vp]),
    "gpt2_get_loss": (_i, [_vp, _fp]),
    "gpt2_synchronize": (_i, [_vp]),
    "gpt2_sample_top_k": (_i, [_vp, _vp, _vp, _i, _i, _vp, _vp]),
    "gpt2_last_error": (ctypes.c_char_p, [_vp]),
    "gpt2op_gemm_bf16": (_i, [_vp, _i, _i, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, _f, _vp, _i64]),
    "gpt2op_gemm_bf16_fused": (_i, [_vp, _i, _i, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, ctypes.c_float,
                                    _vp, _i64, _vp, _i64]),
    "gpt2op_attention_fwd": (_i, [_vp, _i, _vp, _vp, _vp, _i, _i, _i, _i]),
    "gpt2op_attention_bwd": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i]),
    "gpt2op_attention_bwd_noalloc": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i]),
    "gpt2op_layernorm_fwd": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i]),
    "gpt2op_embedding_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i]),
    "gpt2op_embedding_bwd_ws_bytes": (_i64, [_i, _i]),
    "gpt2op_embedding_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "gpt2op_sample_top_k": (_i, [_vp, _i, _vp, _i64, _i, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "gpt2op_classifier_aux_floats": (_i64, [_i, _i]),
    "gpt2op_classifier_fwd_bwd": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "gpt2op_device_error": (_i, []),
    "gpt2op_bounded_wait_selftest": (_i, [_vp, _i64, _vp, _vp]),
    "gpt2_lr_cosine": (ctypes.c_double, [_i64, ctypes.c_double, _i64, _i64, ctypes.c_double]),
    "gpt2_kernel_launches": (_i64, []),
    "gpt2_profile_start": (_i, [_vp]),
    "gpt2_profile_stop": (_i, [_vp, _vp, _vp, _vp, _vp]),
}

PROF_CLASSES = ("gemm_fwd", "gemm_bwd", "lm_head_fwd", "lm_head_bwd", "attn_fwd", "attn_bwd", "layernorm_fwd",
                "layernorm_bwd", "cross_entropy", "bias_grad", "embedding", "optimizer")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m decoder_only_transformer_train_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _PROTOS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_LIB: ctypes.CDLL | None = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = load()
    return _LIB


def _check(rc: int, ctx=None):
    if rc != GPT2_OK:
        msg = lib().gpt2_last_error(ctx).decode() if ctx else ""
        raise Gpt2Error(rc, msg)


def _ptr(t) -> int | None:
    """Device (or host) address of a torch tensor / numpy array, None for None."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream)


@dataclass
class Config:
    n_layer: int = 12
    n_embd: int = 768
    n_head: int = 12
    block_size: int = 1024
    vocab_size: int = 50257
    padded_vocab_size: int = 50304
    max_batch: int = 16
    grad_accum_steps: int = 1
    precision: int = GPT2_BF16

    def c(self) -> gpt2_config:
        return gpt2_config(self.n_layer, self.n_embd, self.n_head, self.block_size, self.vocab_size,
                           self.padded_vocab_size, self.max_batch, self.grad_accum_steps, self.precision)


class GPT2:
    """One training context (parameters, gradients, AdamW state, activations) on the
    current CUDA device."""

    def __init__(self, cfg: Config, seed: int = 1, stream=None):
        self.cfg = cfg
        self._h = ctypes.c_void_p()
        c = cfg.c()
        _check(lib().gpt2_create(ctypes.byref(c), seed, ctypes.byref(self._h)))
        self.set_stream(stream)

    def close(self):
        if self._h:
            lib().gpt2_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_stream(self, stream=None):
        _check(lib().gpt2_set_stream(self._h, _stream(stream)), self._h)

    @property
    def num_params(self) -> int:
        return int(lib().gpt2_num_params(self._h))

    def set_graphs(self, enable: bool):
        """Replay the forward / backward launch sequences as CUDA graphs (default on)."""
        _check(lib().gpt2_set_graphs(self._h, int(enable)), self._h)

    def forward(self, tokens, targets=None, sync_loss: bool = True) -> float | None:
        """tokens/targets: int32 CUDA tensors [B, T]."""
        B, T = tokens.shape
        loss = ctypes.c_float()
        _check(lib().gpt2_forward(self._h, _ptr(tokens), _ptr(targets), B, T,
                                  ctypes.byref(loss) if sync_loss and targets is not None else None), self._h)
        return float(loss.value) if sync_loss and targets is not None else None

    def forward_host(self, tokens: np.ndarray, targets: np.ndarray | None = None, sync_loss: bool = True):
        """tokens/targets: int32 host arrays (numpy, or pinned torch CPU tensors) [B, T]."""
        B, T = tokens.shape
        loss = ctypes.c_float()
        _check(lib().gpt2_forward_host(self._h, _ptr(tokens), _ptr(targets), B, T,
                                       ctypes.byref(loss) if sync_loss and targets is not None else None), self._h)
        return float(loss.value) if sync_loss and targets is not None else None

    def backward(self):
        _check(lib().gpt2_backward(self._h), self._h)

    def zero_grad(self):
        _check(lib().gpt2_zero_grad(self._h), self._h)

    def adamw_step(self, lr, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, clip=1.0,
                   sync_norm: bool = True) -> float | None:
        norm = ctypes.c_float()
        _check(lib().gpt2_adamw_step(self._h, lr, beta1, beta2, eps, weight_decay, clip,
                                     ctypes.byref(norm) if sync_norm else None), self._h)
        return float(norm.value) if sync_norm else None

    def get_params(self) -> np.ndarray:
        out = np.empty(self.num_params, dtype=np.float32)
        _check(lib().gpt2_get_params(self._h, out.ctypes.data), self._h)
        return out

    def set_params(self, flat: np.ndarray):
        flat = np.ascontiguousarray(flat, dtype=np.float32)
        assert flat.size == self.num_params
        _check(lib().gpt2_set_params(self._h, flat.ctypes.data), self._h)

    def grad_tensor(self):
        """The library's flat f32 gradient buffer as a torch CUDA tensor that aliases it
        (zero-copy, through __cuda_array_interface__), e.g. for a data-parallel all-reduce
        between the last backward of a step and adamw_step.  It must not outlive the model."""
        import torch
        p, n = ctypes.c_void_p(), ctypes.c_int64()
        _check(lib().gpt2_get_grad_buffer(self._h, ctypes.byref(p), ctypes.byref(n)), self._h)

        class _DeviceBuffer:
            __cuda_array_interface__ = {"shape": (int(n.value),), "typestr": "<f4", "data": (int(p.value), False),
                                        "version": 3, "strides": None, "stream": None}

        return torch.as_tensor(_DeviceBuffer(), device="cuda")

    def get_grads(self) -> np.ndarray:
        out = np.empty(self.num_params, dtype=np.float32)
        _check(lib().gpt2_get_grads(self._h, out.ctypes.data), self._h)
        return out

    def get_optimizer_state(self):
        m = np.empty(self.num_params, dtype=np.float32)
        v = np.empty(self.num_params, dtype=np.float32)
        t = ctypes.c_int64()
        _check(lib().gpt2_get_optimizer_state(self._h, m.ctypes.data, v.ctypes.data, ctypes.byref(t)), self._h)
        return m, v, int(t.value)

    def set_optimizer_state(self, m: np.ndarray, v: np.ndarray, t: int):
        m = np.ascontiguousarray(m, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        _check(lib().gpt2_set_optimizer_state(self._h, m.ctypes.data, v.ctypes.data, t), self._h)

    def sample_top_k(self, rows, u, k: int, out, out_topk=None):
        """Top-k sampling from the last forward's logits: rows (int32), u (f32) and out
        (int32, and out_topk [n, min(k, vocab)]) are device tensors; asynchronous."""
        _check(lib().gpt2_sample_top_k(self._h, _ptr(rows), _ptr(u), int(rows.numel()), k, _ptr(out),
                                       _ptr(out_topk)), self._h)

    def get_argmax(self, n: int) -> np.ndarray:
        out = np.empty(n, dtype=np.int32)
        _check(lib().gpt2_get_argmax(self._h, out.ctypes.data), self._h)
        return out

    def get_lse(self, n: int) -> np.ndarray:
        out = np.empty(n, dtype=np.float32)
        _check(lib().gpt2_get_lse(self._h, out.ctypes.data), self._h)
        return out

    def get_loss(self) -> float:
        loss = ctypes.c_float()
        _check(lib().gpt2_get_loss(self._h, ctypes.byref(loss)), self._h)
        return float(loss.value)

    def synchronize(self):
        _check(lib().gpt2_synchronize(self._h), self._h)

    def profile_start(self):
        _check(lib().gpt2_profile_start(self._h), self._h)

    def profile_stop(self) -> dict:
        """{class: {"ms", "launches", "flops", "bytes"}} summed over the profiled launches."""
        n = len(PROF_CLASSES)
        ms, fl, by = (np.zeros(n, dtype=np.float64) for _ in range(3))
        la = np.zeros(n, dtype=np.int64)
        _check(lib().gpt2_profile_stop(self._h, ms.ctypes.data, la.ctypes.data, fl.ctypes.data, by.ctypes.data),
               self._h)
        return {c: {"ms": float(ms[i]), "launches": int(la[i]), "flops": float(fl[i]), "bytes": float(by[i])}
                for i, c in enumerate(PROF_CLASSES)}


# ------------------------------------------------------------------ single operations
def gemm_bf16(A, B, C, M, N, K, lda, ldb, ldc, a_mn=False, b_mn=False, epilogue=0, bias=None, alpha=1.0,
              workspace=None, stream=None):
    ws = workspace.numel() if workspace is not None else 0
    _check(lib().gpt2op_gemm_bf16(_stream(stream), M, N, K, _ptr(A), lda, int(a_mn), _ptr(B), ldb, int(b_mn),
                                  _ptr(C), ldc, epilogue, _ptr(bias), alpha, _ptr(workspace), ws))


def gemm_bf16_fused(A, B, C, M, N, K, lda, ldb, ldc, a_mn, b_mn, epilogue, bias=None, alpha=1.0, aux=None,
                    ld_aux=0, aux_out=None, ld_aux_out=0, stream=None):
    """Epilogue 3 (residual), 4 (GELU, keeps the pre-activation in aux_out), 5 (GELU grad)."""
    _check(lib().gpt2op_gemm_bf16_fused(_stream(stream), M, N, K, _ptr(A), lda, int(a_mn), _ptr(B), ldb, int(b_mn),
                                        _ptr(C), ldc, epilogue, _ptr(bias), alpha, _ptr(aux), ld_aux, _ptr(aux_out),
                                        ld_aux_out))


def attention_fwd(qkv, out, lse, B, T, H, head_dim, precision, stream=None):
    _check(lib().gpt2op_attention_fwd(_stream(stream), precision, _ptr(qkv), _ptr(out), _ptr(lse), B, T, H,
                                      head_dim))


def attention_bwd(qkv, out, dout, lse, Dbuf, dqkv, B, T, H, head_dim, precision, stream=None):
    _check(lib().gpt2op_attention_bwd(_stream(stream), precision, _ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse),
                                      _ptr(Dbuf), _ptr(dqkv), B, T, H, head_dim))


# Largest B*H*T gpt2op_attention_bwd_noalloc accepts (size of its fixed row-sum array).
NOALLOC_ATTN_MAX_ROWS = 262144


def attention_bwd_noalloc(qkv, out, dout, lse, dqkv, B, T, H, head_dim, precision, stream=None):
    """attention_bwd without a scratch argument: D lives in the library's fixed array."""
    rc = lib().gpt2op_attention_bwd_noalloc(_stream(stream), precision, _ptr(qkv), _ptr(out), _ptr(dout),
                                            _ptr(lse), _ptr(dqkv), B, T, H, head_dim)
    if rc != GPT2_OK and B * H * T > NOALLOC_ATTN_MAX_ROWS:
        raise Gpt2Error(rc, f"B*H*T = {B * H * T} exceeds the fixed scratch of {NOALLOC_ATTN_MAX_ROWS} rows")
    _check(rc)


def layernorm_fwd(x, w, b, y, mean, rstd, N, C, precision, stream=None):
    _check(lib().gpt2op_layernorm_fwd(_stream(stream), precision, _ptr(x), _ptr(w), _ptr(b), _ptr(y), _ptr(mean),
                                      _ptr(rstd), N, C))


def embedding_fwd(tokens, wte, wpe, x, B, T, C, V, stream=None):
    _check(lib().gpt2op_embedding_fwd(_stream(stream), _ptr(tokens), _ptr(wte), _ptr(wpe), _ptr(x), B, T, C, V))


def embedding_bwd_ws_bytes(N: int, C: int) -> int:
    return int(lib().gpt2op_embedding_bwd_ws_bytes(N, C))


def embedding_bwd(tokens, dx0, dwte, dwpe, B, T, C, V, ws, stream=None):
    """dwte, dwpe += the embedding gradients of dx0; ws (embedding_bwd_ws_bytes bytes)
    holds the ascending sort keys token << 15 | position in its first B*T uint32 words."""
    _check(lib().gpt2op_embedding_bwd(_stream(stream), _ptr(tokens), _ptr(dx0), _ptr(dwte), _ptr(dwpe), B, T, C, V,
                                      _ptr(ws)))


SAMPLE_MAX_K = 1024


def sample_top_k(logits, ld, n_rows, rows, u, n, V, k, precision, out, out_topk=None, stream=None):
    """gpt2op_sample_top_k on caller logits [n_rows, ld] (bf16 or f32 by precision)."""
    _check(lib().gpt2op_sample_top_k(_stream(stream), precision, _ptr(logits), ld, n_rows, _ptr(rows), _ptr(u), n, V,
                                     k, _ptr(out), _ptr(out_topk)))


def classifier_aux_floats(N: int, V: int) -> int:
    return int(lib().gpt2op_classifier_aux_floats(N, V))


def classifier_fwd_bwd(h, W, targets, N, V, C, logits_ws, ldl, aux_ws, loss, lse, argmax, dh, dW, stream=None):
    _check(lib().gpt2op_classifier_fwd_bwd(_stream(stream), _ptr(h), _ptr(W), _ptr(targets), N, V, C,
                                           _ptr(logits_ws), ldl, _ptr(aux_ws), _ptr(loss), _ptr(lse), _ptr(argmax),
                                           _ptr(dh), _ptr(dW)))


def device_error() -> int:
    return int(lib().gpt2op_device_error())


def bounded_wait_selftest(limit_ns: int, src16, status, stream=None):
    _check(lib().gpt2op_bounded_wait_selftest(_stream(stream), limit_ns, _ptr(src16), _ptr(status)))
