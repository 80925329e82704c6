"""hlta_gdn_forward_noalloc -- the memory branch for callers that must not
allocate device memory while running (fixed-budget control loops, code under an
allocator that forbids cudaMalloc).  Its scratch is a static array in the
library, so it needs no handle.  Checked here through the C ABI against the
handle path (hlta_forward with only the memory branch) on two calls in a row,
within the bf16 tolerance the parity tests use.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest

from workloads import WORKLOADS, make_inputs
from parity_util import to_device, to_numpy64, assert_close

pytestmark = pytest.mark.gpu


def test_noalloc_matches_handle_path_twice():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_linear_temporal_b200 import build
    build.build()
    import hybrid_linear_temporal_b200 as hl
    from hybrid_linear_temporal_b200 import binding
    wl = WORKLOADS["clip_4k"].with_(B=2, H=4, L=1000, P=100, swa_window=100, dswa_window=100, dilation=2)
    inp = make_inputs(wl, seed=7)
    dev = to_device(inp)
    S0 = torch.from_numpy(np.random.default_rng(1).standard_normal((2, 4, 128, 128)).astype(np.float32) * 0.1).cuda()
    layer = hl.HLTA.for_workload(wl)
    S_ref = torch.empty_like(S0)
    ref = layer.forward(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], dev["gates"], S0=S0,
                        S_out=S_ref, branches=hl.BRANCH_GDN)
    torch.cuda.synchronize()
    lib = hl.load_library()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    for call in range(2):
        out = torch.full_like(dev["v"], float("nan"))
        S_out = torch.full_like(S0, float("nan"))
        st = lib.hlta_gdn_forward_noalloc(wl.B, wl.L, wl.H, p(dev["q"]), p(dev["k"]), p(dev["v"]),
                                          p(dev["alpha"]), p(dev["beta"]), p(dev["gates"]), p(S0), p(S_out),
                                          p(out), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == binding.OK, lib.hlta_last_error().decode()
        torch.cuda.synchronize()
        assert_close(to_numpy64(out), to_numpy64(ref), "bf16", f"call {call}: output")
        assert_close(to_numpy64(S_out), to_numpy64(S_ref), "bf16", f"call {call}: final state")
    # sizes beyond the static scratch are refused with a message, nothing enqueued
    st = lib.hlta_gdn_forward_noalloc(1, 64 * 1200, 1, p(dev["q"]), p(dev["k"]), p(dev["v"]), p(dev["alpha"]),
                                      p(dev["beta"]), p(dev["gates"]), None, None, p(dev["v"]), None)
    assert st == binding.ERR_UNSUPPORTED and b"1110" in lib.hlta_last_error()
    layer.close()
