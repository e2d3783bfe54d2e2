"""CPU checks of the C-ABI library: it builds, loads without a GPU and exports every
function that include/*.h declares; the product package never imports the oracle."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "decoder_only_transformer_train_b200")


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(gpt2\w*)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def libpath():
    from decoder_only_transformer_train_b200 import build
    return build.build()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("gpt2_create", "gpt2_forward", "gpt2_backward", "gpt2_zero_grad", "gpt2_adamw_step",
                     "gpt2_destroy", "gpt2_get_params", "gpt2_set_params", "gpt2_get_grads"):
        assert required in names


def test_library_loads_and_exports_every_declared_symbol(libpath):
    lib = ctypes.CDLL(libpath)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_prototypes_cover_the_header(libpath):
    from decoder_only_transformer_train_b200 import binding
    assert set(_declared_functions()) == set(binding._PROTOS)
    binding.load(libpath)


def test_library_is_built_for_sm100a(libpath):
    from decoder_only_transformer_train_b200 import build
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)
    assert os.path.getsize(libpath) > 100_000


def test_product_code_does_not_touch_the_oracle():
    offenders = []
    for path in glob.glob(os.path.join(PKG, "**", "*"), recursive=True):
        if not os.path.isfile(path) or path.endswith((".so", ".o")):
            continue
        text = open(path, errors="ignore").read()
        if re.search(r"^\s*(from|import)\s+oracle\b", text, flags=re.M):
            offenders.append(path)
    assert not offenders, offenders


def test_no_host_api_rejects_bad_config_without_gpu(libpath):
    """gpt2_create validates the configuration before touching the device."""
    from decoder_only_transformer_train_b200 import binding
    lib = binding.load(libpath)
    bad = binding.Config(n_embd=100, n_head=3).c()
    h = ctypes.c_void_p()
    assert lib.gpt2_create(ctypes.byref(bad), 1, ctypes.byref(h)) == -4
    assert not h.value
    assert lib.gpt2_create(None, 1, ctypes.byref(h)) == -1


def test_gemm_entry_points_refuse_misaligned_epilogue_operands_without_gpu(libpath):
    """The GEMM epilogues read bias and aux and write aux_out with 16-byte accesses: a
    pointer off a 16-byte boundary is refused (GPT2_ERR_ARG) before any CUDA call."""
    import numpy as np
    from decoder_only_transformer_train_b200 import binding
    lib = binding.load(libpath)
    buf = np.zeros(256, dtype=np.float32)
    p = (buf.ctypes.data + 15) // 16 * 16
    q = p + 4
    assert lib.gpt2op_gemm_bf16(None, 128, 128, 64, p, 64, 0, p, 64, 0, p, 128, 0, q, 1.0, None, 0) == -1
    for bias, aux, aux_out in ((q, p, p), (p, q, p), (p, p, q)):
        assert lib.gpt2op_gemm_bf16_fused(None, 128, 128, 64, p, 64, 0, p, 64, 0, p, 128, 4, bias, 1.0, aux, 128,
                                          aux_out, 128) == -1


def test_lr_schedule_host_function_matches_oracle(libpath):
    import oracle as O
    from decoder_only_transformer_train_b200 import binding
    lib = binding.load(libpath)
    for it in (0, 1, 100, 714, 715, 716, 1000, 5000, 19072, 19073, 19074, 25000):
        got = lib.gpt2_lr_cosine(it, 6e-4, 715, 19073, 0.1)
        assert abs(got - O.get_lr(it)) <= 1e-15, it
