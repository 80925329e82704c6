"""Thin ctypes binding of ``libhlta.so`` (the C ABI in ``include/hlta.h``).

Argument marshalling only: every step of the layer runs in the CUDA library.
Device tensors are ``torch.Tensor`` objects on the handle's GPU (PyTorch is
used for device memory and streams); host tensors for ``forward_host`` are
NumPy arrays.  If the library is missing this module raises on use -- there
is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhlta.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "hlta.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_OOM, ERR_DEVICE_TIMEOUT, ERR_INJECTED = range(7)
BF16, FP32 = 0, 1
GDN_DECAYED, GDN_PAGES = 0, 1
WINDOW_CAUSAL, WINDOW_CENTRED = 0, 1
BRANCH_SWA, BRANCH_DSWA, BRANCH_GDN, BRANCH_ALL = 1, 2, 4, 7


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "B", "H", "d_k", "d_v", "tokens_per_frame", "swa_window", "dswa_window",
        "dswa_dilation", "chunk", "dtype", "max_seq_len", "max_stream_tokens", "gdn_form",
        "window_mode")] + [("rope_base", ctypes.c_float), ("attn_fp8", ctypes.c_int)]


class ProfileData(ctypes.Structure):
    _fields_ = [("count", ctypes.c_int), ("name", (ctypes.c_char * 16) * 4),
                ("total_ms", ctypes.c_double * 4), ("passes", ctypes.c_longlong * 4),
                ("kernel_launches", ctypes.c_longlong)]


class HltaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"hlta status {status}: {msg}")
        self.status = status


_lib = None


def load_library(path: str | None = None):
    """Load libhlta.so and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m hybrid_linear_temporal_b200.build`")
    lib = ctypes.CDLL(p)
    vp, fp, i, u = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    st = ctypes.c_int
    sig = {
        "hlta_create": ([ctypes.POINTER(Config), ctypes.POINTER(vp)], st),
        "hlta_destroy": ([vp], st),
        "hlta_forward": ([vp, i, vp, vp, vp, fp, fp, fp, fp, fp, vp, u, vp], st),
        "hlta_forward_host": ([vp, i, vp, vp, vp, fp, fp, fp, fp, fp, vp, u, vp], st),
        "hlta_backward": ([vp, i, vp, vp, vp, fp, fp, fp, fp, vp, fp, vp, vp, vp, fp, fp, fp, fp, u, vp], st),
        "hlta_stream_step": ([vp, i, vp, vp, vp, fp, fp, fp, vp, u, vp], st),
        "hlta_state_get": ([vp, fp, ctypes.POINTER(ctypes.c_longlong), vp], st),
        "hlta_stream_reset": ([vp, vp], st),
        "hlta_stream_checkpoint_bytes": ([vp], ctypes.c_longlong),
        "hlta_stream_save": ([vp, vp, vp], st),
        "hlta_stream_load": ([vp, vp, vp], st),
        "hlta_device_status": ([vp], st),
        "hlta_profile_enable": ([vp, i], st),
        "hlta_profile_read": ([vp, ctypes.POINTER(ProfileData)], st),
        "hlta_gdn_forward_noalloc": ([i, i, i, vp, vp, vp, fp, fp, fp, fp, fp, vp, vp], st),
        "hlta_last_error": ([], ctypes.c_char_p),
        "hlta_version": ([], i),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    if path is None:
        _lib = lib
    return lib


def header_symbols(header: str = HEADER) -> list[str]:
    """Entry points declared in include/hlta.h."""
    txt = open(header).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(hlta_[a-z_0-9]+)\s*\(", txt)))


def _check(lib, status: int):
    if status != OK:
        raise HltaError(status, lib.hlta_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def gdn_forward_noalloc(q, k, v, alpha, beta, gates, S0=None, S_out=None, out=None, stream=None):
    """Memory branch without device allocation (hlta_gdn_forward_noalloc).

    For callers that must not allocate device memory while running; the scratch
    is a static array in the library.  Tensors as for HLTA.forward with
    d_k = d_v = 128, bf16; returns out = g[h,2] * o_t."""
    import torch
    lib = load_library()
    B, L, H, _ = q.shape
    if out is None:
        out = torch.empty_like(v)
    _check(lib, lib.hlta_gdn_forward_noalloc(B, L, H, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                             _ptr(gates), _ptr(S0), _ptr(S_out), _ptr(out), _stream(stream)))
    return out


class HLTA:
    """One configured layer (a handle of the C library) on the current GPU."""

    def __init__(self, B, H, d_k, d_v, tokens_per_frame, swa_window, dswa_window, dilation,
                 chunk=64, dtype="bf16", max_seq_len=1, max_stream_tokens=0, gdn_form=0,
                 window_mode=0, rope_base=0.0, attn_fp8=0):
        self.lib = load_library()
        self.cfg = Config(B, H, d_k, d_v, tokens_per_frame, swa_window, dswa_window, dilation,
                          chunk, BF16 if dtype == "bf16" else FP32, max_seq_len, max_stream_tokens,
                          gdn_form, window_mode, rope_base, attn_fp8)
        self.dtype = dtype
        h = ctypes.c_void_p()
        _check(self.lib, self.lib.hlta_create(ctypes.byref(self.cfg), ctypes.byref(h)))
        self.h = h

    @classmethod
    def for_workload(cls, wl, max_seq_len=None, max_stream_tokens=0, gdn_form=0, window_mode=0,
                     rope_base=0.0, attn_fp8=0):
        return cls(wl.B, wl.H, wl.d_k, wl.d_v, wl.P, wl.swa_window, wl.dswa_window, wl.dilation,
                   wl.chunk, wl.dtype, max_seq_len or wl.L, max_stream_tokens, gdn_form, window_mode,
                   rope_base, attn_fp8)

    def close(self):
        if getattr(self, "h", None):
            self.lib.hlta_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- marshalling helpers ------------------------------------------------
    def _torch_dtype(self):
        import torch
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def _check_tensor(self, t, name, shape, dtype):
        if t is None:
            raise ValueError(f"{name} is required")
        if not t.is_cuda or not t.is_contiguous() or t.dtype != dtype or tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                             f"{t.dtype} {tuple(t.shape)} cuda={t.is_cuda}")

    def _check_inputs(self, n, q, k, v, alpha, beta, gates):
        import torch
        c = self.cfg
        dt = self._torch_dtype()
        self._check_tensor(q, "q", (c.B, n, c.H, c.d_k), dt)
        self._check_tensor(k, "k", (c.B, n, c.H, c.d_k), dt)
        self._check_tensor(v, "v", (c.B, n, c.H, c.d_v), dt)
        self._check_tensor(alpha, "alpha", (c.B, n, c.H), torch.float32)
        self._check_tensor(beta, "beta", (c.B, n, c.H), torch.float32)
        self._check_tensor(gates, "gates", (c.H, 3), torch.float32)

    # -- entry points -------------------------------------------------------
    def forward(self, q, k, v, alpha, beta, gates, S0=None, S_out=None, out=None,
                branches=BRANCH_ALL, stream=None):
        import torch
        c = self.cfg
        L = q.shape[1]
        self._check_inputs(L, q, k, v, alpha, beta, gates)
        if out is None:
            out = torch.empty((c.B, L, c.H, c.d_v), dtype=self._torch_dtype(), device=q.device)
        self._check_tensor(out, "out", (c.B, L, c.H, c.d_v), self._torch_dtype())
        for name, s in (("S0", S0), ("S_out", S_out)):
            if s is not None:
                self._check_tensor(s, name, (c.B, c.H, c.d_v, c.d_k), torch.float32)
        _check(self.lib, self.lib.hlta_forward(
            self.h, L, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(gates),
            _ptr(S0), _ptr(S_out), _ptr(out), branches, _stream(stream)))
        return out

    def backward(self, q, k, v, alpha, beta, gates, dout, S0=None, dS_final=None, want_dS0=False,
                 branches=BRANCH_ALL, stream=None):
        """Gradients of ``forward`` (hlta_backward).  Returns a dict of tensors:
        dq, dk, dv (cfg dtype), dalpha, dbeta, dgates and dS0 (float32; dS0 only
        when want_dS0)."""
        import torch
        c = self.cfg
        L = q.shape[1]
        self._check_inputs(L, q, k, v, alpha, beta, gates)
        dt = self._torch_dtype()
        self._check_tensor(dout, "dout", (c.B, L, c.H, c.d_v), dt)
        for name, s in (("S0", S0), ("dS_final", dS_final)):
            if s is not None:
                self._check_tensor(s, name, (c.B, c.H, c.d_v, c.d_k), torch.float32)
        dev = q.device
        r = {"dq": torch.empty((c.B, L, c.H, c.d_k), dtype=dt, device=dev),
             "dk": torch.empty((c.B, L, c.H, c.d_k), dtype=dt, device=dev),
             "dv": torch.empty((c.B, L, c.H, c.d_v), dtype=dt, device=dev),
             "dalpha": torch.empty((c.B, L, c.H), dtype=torch.float32, device=dev),
             "dbeta": torch.empty((c.B, L, c.H), dtype=torch.float32, device=dev),
             "dgates": torch.empty((c.H, 3), dtype=torch.float32, device=dev),
             "dS0": torch.empty((c.B, c.H, c.d_v, c.d_k), dtype=torch.float32, device=dev)
             if want_dS0 else None}
        _check(self.lib, self.lib.hlta_backward(
            self.h, L, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(gates), _ptr(S0),
            _ptr(dout), _ptr(dS_final), _ptr(r["dq"]), _ptr(r["dk"]), _ptr(r["dv"]), _ptr(r["dalpha"]),
            _ptr(r["dbeta"]), _ptr(r["dgates"]), _ptr(r["dS0"]), branches, _stream(stream)))
        return r

    def forward_host(self, q, k, v, alpha, beta, gates, S0=None, S_out=None, out=None,
                     branches=BRANCH_ALL, stream=None):
        """Host-buffer variant (NumPy arrays; bf16 as uint16 bits).  Synchronous."""
        c = self.cfg
        L = q.shape[1]
        edt = np.uint16 if self.dtype == "bf16" else np.float32
        arrs = []
        for name, a, dt in (("q", q, edt), ("k", k, edt), ("v", v, edt), ("alpha", alpha, np.float32),
                            ("beta", beta, np.float32), ("gates", gates, np.float32)):
            if a.dtype != dt or not a.flags.c_contiguous:
                raise ValueError(f"{name}: expected contiguous {dt}")
            arrs.append(a)
        if out is None:
            out = np.empty((c.B, L, c.H, c.d_v), dtype=edt)
        hp = lambda a: None if a is None else ctypes.c_void_p(a.ctypes.data)
        _check(self.lib, self.lib.hlta_forward_host(
            self.h, L, *[hp(a) for a in arrs], hp(S0), hp(S_out), hp(out), branches, _stream(stream)))
        return out

    def stream_step(self, q, k, v, alpha, beta, gates, out=None, branches=BRANCH_ALL, stream=None):
        import torch
        c = self.cfg
        n = q.shape[1]
        self._check_inputs(n, q, k, v, alpha, beta, gates)
        if out is None:
            out = torch.empty((c.B, n, c.H, c.d_v), dtype=self._torch_dtype(), device=q.device)
        self._check_tensor(out, "out", (c.B, n, c.H, c.d_v), self._torch_dtype())
        _check(self.lib, self.lib.hlta_stream_step(
            self.h, n, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(gates), _ptr(out),
            branches, _stream(stream)))
        return out

    def state_get(self, S_dst=None, stream=None):
        import torch
        c = self.cfg
        if S_dst is None:
            S_dst = torch.empty((c.B, c.H, c.d_v, c.d_k), dtype=torch.float32, device="cuda")
        pos = ctypes.c_longlong()
        _check(self.lib, self.lib.hlta_state_get(self.h, _ptr(S_dst), ctypes.byref(pos), _stream(stream)))
        return S_dst, pos.value

    def stream_reset(self, stream=None):
        _check(self.lib, self.lib.hlta_stream_reset(self.h, _stream(stream)))

    def checkpoint_bytes(self) -> int:
        return int(self.lib.hlta_stream_checkpoint_bytes(self.h))

    def stream_save(self, dst=None, stream=None):
        import torch
        if dst is None:
            dst = torch.empty(self.checkpoint_bytes(), dtype=torch.uint8, device="cuda")
        _check(self.lib, self.lib.hlta_stream_save(self.h, _ptr(dst), _stream(stream)))
        return dst

    def stream_load(self, src, stream=None):
        _check(self.lib, self.lib.hlta_stream_load(self.h, _ptr(src), _stream(stream)))

    def profile_enable(self, enable=True):
        _check(self.lib, self.lib.hlta_profile_enable(self.h, int(enable)))

    def profile_read(self) -> dict:
        """Per-branch device time recorded since profile_enable (synchronises)."""
        d = ProfileData()
        _check(self.lib, self.lib.hlta_profile_read(self.h, ctypes.byref(d)))
        res = {"kernel_launches": int(d.kernel_launches)}
        for i in range(d.count):
            res[d.name[i].value.decode()] = {"total_ms": float(d.total_ms[i]),
                                             "passes": int(d.passes[i])}
        return res

    def device_status(self):
        return self.lib.hlta_device_status(self.h)
