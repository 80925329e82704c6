"""GPU parity of the layer backward (hlta_backward through the C ABI) against
the oracle's reverse-mode derivatives on the same seeded inputs.

Tolerances: gradients returned in bf16 (dq, dk, dv of a bf16 layer) -- relative
L2 <= 5e-3 and max-abs <= 2e-2 * max(1, max |ref|) (one bf16 rounding of each
element on top of the arithmetic); gradients returned in fp32 (dalpha, dbeta,
dS0, and everything of an fp32 layer) -- relative L2 <= 1e-3 for bf16 layers
(fp32 arithmetic from bf16 inputs) and 1e-4 for fp32 layers.  dgates = dout . o
takes the branch outputs of the forward, whose bf16 tensor-core path rounds the
softmax weights to bf16, so for bf16 layers it carries the forward's relative
L2 bound of 5e-3.
"""
import numpy as np
import pytest

import oracle
from workloads import WORKLOADS, make_inputs, bf16_bits, bf16_to_float32
from parity_util import to_device, to_numpy64, errors

pytestmark = pytest.mark.gpu

BRANCHES = ("swa", "dswa", "gdn")


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from hybrid_linear_temporal_b200 import build
    build.build()
    return torch


def _dout(wl, seed):
    x = np.random.default_rng(1000 + seed).standard_normal((wl.B, wl.L, wl.H, wl.d_v))
    return bf16_bits(x) if wl.dtype == "bf16" else x.astype(np.float32)


def _check(got, ref, what, returned_bf16, layer_bf16, tol_bf16_layer=1e-3):
    e = errors(got, ref)
    if returned_bf16:
        lim = 2e-2 * max(1.0, float(np.abs(ref).max()))
        assert e["rel_l2"] <= 5e-3 and e["max_abs"] <= lim, f"{what}: {e}"
    else:
        tol = tol_bf16_layer if layer_bf16 else 1e-4
        assert e["rel_l2"] <= tol, f"{what}: {e} vs {tol}"
    return e


def backward_compare(torch, wl, seed=0, branches=BRANCHES, S0=False, dS_final=False, window_mode=0,
                     rope_base=0.0, q_scale=1.0):
    from hybrid_linear_temporal_b200 import HLTA
    inp = make_inputs(wl, seed=seed, q_scale=q_scale)
    dout = _dout(wl, seed)
    dout64 = bf16_to_float32(dout).astype(np.float64) if wl.dtype == "bf16" else dout.astype(np.float64)
    rng = np.random.default_rng(2000 + seed)
    S0_np = rng.standard_normal((wl.B, wl.H, wl.d_v, wl.d_k)).astype(np.float32) * 0.1 if S0 else None
    dSf_np = rng.standard_normal((wl.B, wl.H, wl.d_v, wl.d_k)).astype(np.float32) if dS_final else None
    ref = oracle.backward(inp, dout64, S0=None if S0_np is None else S0_np.astype(np.float64),
                          dS_final=None if dSf_np is None else dSf_np.astype(np.float64),
                          branches=branches, centred=window_mode == 1, rope_base=rope_base)
    layer = HLTA.for_workload(wl, window_mode=window_mode, rope_base=rope_base)
    dev = to_device(inp)
    t = lambda a: None if a is None else torch.from_numpy(a).cuda()
    dout_t = (torch.from_numpy(dout.view(np.int16)).view(torch.bfloat16) if wl.dtype == "bf16"
              else torch.from_numpy(dout)).cuda()
    mask = sum(1 << i for i, n in enumerate(BRANCHES) if n in branches)
    got = layer.backward(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], dev["gates"], dout_t,
                         S0=t(S0_np), dS_final=t(dSf_np), want_dS0="gdn" in branches, branches=mask)
    torch.cuda.synchronize()
    layer.close()
    bf = wl.dtype == "bf16"
    res = {}
    for n in ("dq", "dk", "dv"):
        res[n] = _check(to_numpy64(got[n]), ref[n], f"{wl.name} {n}", bf, bf)
    cols = [i for i, n in enumerate(BRANCHES) if n in branches]
    res["dgates"] = _check(to_numpy64(got["dgates"])[:, cols], ref["dgates"][:, cols], f"{wl.name} dgates",
                           False, bf, tol_bf16_layer=5e-3)
    assert np.abs(to_numpy64(got["dgates"])[:, [i for i in range(3) if i not in cols]]).max(initial=0) == 0
    if "gdn" in branches:
        for n in ("dalpha", "dbeta", "dS0"):
            res[n] = _check(to_numpy64(got[n]), ref[n], f"{wl.name} {n}", False, bf)
    else:
        assert np.abs(to_numpy64(got["dalpha"])).max() == 0 and np.abs(to_numpy64(got["dbeta"])).max() == 0
    return res


def test_backward_tiny_fp32(torch_cuda):
    backward_compare(torch_cuda, WORKLOADS["tiny_fp32"])


def test_backward_tiny_fp32_state_gradients(torch_cuda):
    backward_compare(torch_cuda, WORKLOADS["tiny_fp32"].with_(L=200), seed=1, S0=True, dS_final=True)


def test_backward_clip_4k_bf16(torch_cuda):
    backward_compare(torch_cuda, WORKLOADS["clip_4k"])


@pytest.mark.parametrize("branches", [("swa",), ("dswa",), ("gdn",), ("swa", "gdn")])
def test_backward_branch_subsets(torch_cuda, branches):
    wl = WORKLOADS["clip_4k"].with_(H=2, L=640, P=64, swa_window=100, dswa_window=80, dilation=3)
    backward_compare(torch_cuda, wl, branches=branches)


@pytest.mark.parametrize("case", [
    dict(L=1), dict(L=65), dict(L=333, P=50), dict(L=256, swa_window=1, dswa_window=1),
    dict(L=300, swa_window=1000, dswa_window=1000), dict(L=384, P=8, dilation=5, dswa_window=41),
    dict(L=512, d_k=64, d_v=64), dict(B=2, L=192, H=3), dict(L=200, d_k=128, d_v=64),
])
def test_backward_edge_cases_bf16(torch_cuda, case):
    base = WORKLOADS["clip_4k"].with_(H=2, L=256, P=32, swa_window=48, dswa_window=40, dilation=3)
    backward_compare(torch_cuda, base.with_(**case), S0=True, dS_final=True)


@pytest.mark.parametrize("rope_base", [0.0, 10000.0])
def test_backward_centred_window(torch_cuda, rope_base):
    wl = WORKLOADS["clip_4k"].with_(H=2, L=700, P=50, swa_window=64, dswa_window=40, dilation=3)
    backward_compare(torch_cuda, wl, window_mode=1, rope_base=rope_base, q_scale=16.0,
                     branches=("swa", "dswa"))
    backward_compare(torch_cuda, WORKLOADS["tiny_fp32"], window_mode=1, rope_base=rope_base)


def test_backward_slow_decay_and_sharp_softmax(torch_cuda):
    wl = WORKLOADS["clip_4k"].with_(H=2, L=1000, P=64, swa_window=100, dswa_window=80, dilation=4)
    inp_kw = dict(seed=3)
    backward_compare(torch_cuda, wl, q_scale=64.0, branches=("swa", "dswa"), **inp_kw)


def test_backward_rejects_printed_update_form(torch_cuda):
    import torch
    from hybrid_linear_temporal_b200 import HLTA, HltaError
    from hybrid_linear_temporal_b200.binding import ERR_UNSUPPORTED
    wl = WORKLOADS["tiny_fp32"]
    inp = make_inputs(wl)
    dev = to_device(inp)
    layer = HLTA.for_workload(wl, gdn_form=1)
    dout = torch.zeros((wl.B, wl.L, wl.H, wl.d_v), dtype=torch.float32, device="cuda")
    with pytest.raises(HltaError) as ei:
        layer.backward(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], dev["gates"], dout)
    assert ei.value.status == ERR_UNSUPPORTED
    # the attention branches alone are fine with either update form
    layer.backward(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], dev["gates"], dout, branches=3)
    layer.close()


def test_backward_rollout_shaped_bf16(torch_cuda):
    """Frames of the 480P rollout (1560 tokens, windows 1560), fewer frames and
    heads so that the oracle runs in seconds; both branches on the tensor cores."""
    wl = WORKLOADS["rollout_480p"].with_(H=2, L=1560 * 5, dilation=2)
    backward_compare(torch_cuda, wl, S0=True, dS_final=True)
