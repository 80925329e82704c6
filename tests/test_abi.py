"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every entry point include/hlta.h declares, validates arguments before touching
the device, and honours host-side failure injection."""
import ctypes
import os
import subprocess
import sys

import pytest

import hybrid_linear_temporal_b200 as hl
from hybrid_linear_temporal_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from hybrid_linear_temporal_b200 import build
    build.build()
    return hl.load_library()


def test_library_exports_every_declared_symbol(lib):
    declared = hl.header_symbols()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", hl.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared) <= exported


def test_version(lib):
    assert lib.hlta_version() >= 100


def _cfg(**kw):
    base = dict(B=1, H=2, d_k=64, d_v=64, tokens_per_frame=4, swa_window=8, dswa_window=8,
                dswa_dilation=2, chunk=64, dtype=binding.BF16, max_seq_len=128, max_stream_tokens=0,
                gdn_form=binding.GDN_DECAYED, window_mode=binding.WINDOW_CAUSAL, rope_base=0.0, attn_fp8=0)
    base.update(kw)
    return binding.Config(*[base[n] for n, _ in binding.Config._fields_])


@pytest.mark.parametrize("field,value,status", [
    ("B", 0, binding.ERR_INVALID_ARG), ("H", -1, binding.ERR_INVALID_ARG),
    ("tokens_per_frame", 0, binding.ERR_INVALID_ARG), ("swa_window", 0, binding.ERR_INVALID_ARG),
    ("dswa_dilation", 0, binding.ERR_INVALID_ARG), ("dtype", 5, binding.ERR_INVALID_ARG),
    ("max_seq_len", 0, binding.ERR_INVALID_ARG), ("max_stream_tokens", -2, binding.ERR_INVALID_ARG),
    ("gdn_form", 2, binding.ERR_INVALID_ARG), ("gdn_form", -1, binding.ERR_INVALID_ARG),
    ("d_k", 96, binding.ERR_UNSUPPORTED), ("chunk", 32, binding.ERR_UNSUPPORTED),
])
def test_create_rejects_bad_config_before_device(lib, field, value, status):
    h = ctypes.c_void_p()
    st = lib.hlta_create(ctypes.byref(_cfg(**{field: value})), ctypes.byref(h))
    assert st == status
    assert h.value is None
    assert lib.hlta_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(window_mode=2), binding.ERR_INVALID_ARG),
    (dict(window_mode=-1), binding.ERR_INVALID_ARG),
    (dict(window_mode=binding.WINDOW_CENTRED, rope_base=-1.0), binding.ERR_INVALID_ARG),
    (dict(window_mode=binding.WINDOW_CENTRED, rope_base=float("nan")), binding.ERR_INVALID_ARG),
    (dict(window_mode=binding.WINDOW_CENTRED, rope_base=float("inf")), binding.ERR_INVALID_ARG),
    # the rotary embedding is offered with the centred (in-clip) window only
    (dict(window_mode=binding.WINDOW_CAUSAL, rope_base=10000.0), binding.ERR_UNSUPPORTED),
    # a centred window reaches keys after the query: not available token by token
    (dict(window_mode=binding.WINDOW_CENTRED, max_stream_tokens=16), binding.ERR_UNSUPPORTED),
    (dict(attn_fp8=2), binding.ERR_INVALID_ARG),
    # the FP8 logits path exists for the bf16 tensor-core kernel (d = 128) only
    (dict(attn_fp8=1), binding.ERR_UNSUPPORTED),
    (dict(attn_fp8=1, dtype=binding.FP32, d_k=128, d_v=128), binding.ERR_UNSUPPORTED),
])
def test_create_rejects_bad_window_config(lib, over, status):
    h = ctypes.c_void_p()
    st = lib.hlta_create(ctypes.byref(_cfg(**over)), ctypes.byref(h))
    assert st == status
    assert h.value is None
    assert lib.hlta_last_error().decode()


def test_null_arguments(lib):
    h = ctypes.c_void_p()
    assert lib.hlta_create(None, ctypes.byref(h)) == binding.ERR_INVALID_ARG
    assert lib.hlta_create(ctypes.byref(_cfg()), None) == binding.ERR_INVALID_ARG
    assert lib.hlta_forward(None, 1, *[None] * 9, 7, None) == binding.ERR_INVALID_ARG
    assert lib.hlta_stream_step(None, 1, *[None] * 7, 7, None) == binding.ERR_INVALID_ARG
    assert lib.hlta_state_get(None, None, None, None) == binding.ERR_INVALID_ARG
    assert lib.hlta_destroy(None) == binding.OK
    assert lib.hlta_stream_checkpoint_bytes(None) == 0


def test_failure_injection_in_subprocess():
    """HLTA_INJECT_FAIL makes the named entry point fail before doing anything."""
    code = ("import ctypes, hybrid_linear_temporal_b200 as hl\n"
            "from hybrid_linear_temporal_b200 import binding\n"
            "lib = hl.load_library()\n"
            "h = ctypes.c_void_p()\n"
            "c = binding.Config(1,2,64,64,4,8,8,2,64,0,128,0)\n"
            "print(lib.hlta_create(ctypes.byref(c), ctypes.byref(h)), lib.hlta_last_error().decode())\n"
            "print(lib.hlta_forward(None, 1, *[None]*9, 7, None))\n")
    env = dict(os.environ, HLTA_INJECT_FAIL="hlta_create", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         check=True).stdout.split("\n")
    assert out[0].startswith(f"{binding.ERR_INJECTED} hlta_create: injected")
    assert out[1] == str(binding.ERR_INVALID_ARG)
    env["HLTA_INJECT_FAIL"] = "all"
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         check=True).stdout.split("\n")
    assert out[1] == str(binding.ERR_INJECTED)


def test_create_without_usable_gpu_reports_cuda_error(lib):
    """On a machine without an sm_100 GPU a valid config fails with a CUDA
    status and a message (never a crash)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    st = lib.hlta_create(ctypes.byref(_cfg()), ctypes.byref(h))
    assert st == binding.ERR_CUDA
    assert "cuda" in lib.hlta_last_error().decode().lower()


def test_product_path_never_imports_oracle():
    """The package and its sources reference neither the oracle nor a CPU path."""
    pkg = os.path.join(ROOT, "hybrid_linear_temporal_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "hlta_oracle" not in txt, f
