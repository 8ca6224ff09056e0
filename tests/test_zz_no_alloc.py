"""gdn_prefill_noalloc: the prefill entry point for callers that cannot give
the library scratch device memory (for example a runtime whose device memory
belongs to another allocator, or code that must not call cudaMalloc because it
can synchronise the device).  It uses the library's built-in scratch array
instead of a workspace.  Checked through the C ABI against gdn_prefill, on two
calls in a row (different problems, so the second call starts from the first
call's leftover scratch contents).  This file is collected last."""

import numpy as np
import pytest
import torch

import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi
from linear_attention_recurrence_deltanet_b200.device import DeviceProblem, io_float, io_numpy

pytestmark = pytest.mark.gpu

TOL_O, TOL_S, U_BF16 = 2e-3, 1e-3, 2.0 ** -8


def _maxrel(x, ref, u=0.0):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    err = np.maximum(np.abs(x - ref) - u * np.abs(ref), 0.0)
    return float(err.max() / max(np.abs(ref).max(), 1e-30))


def _noalloc(dp, flags=0):
    gdn.prefill_noalloc(dp.cfg, dp.params, dp.qkv, dp.z, dp.a, dp.b, dp.cu_dev, dp.cu_host, dp.chunk_size, flags,
                        dp.conv_state, dp.state, dp.o)


def test_prefill_noalloc_matches_prefill_on_two_calls():
    assert torch.cuda.is_available()
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    problems = [gi.make_prefill_inputs(geo, [70, 5, 129, 0, 33], seed=41, zero_init=False),
                gi.make_prefill_inputs(geo, [200, 1, 64], seed=42, zero_init=False)]
    for inp in problems:  # call 1 and call 2 of the no-alloc entry point
        ref = DeviceProblem(inp, 64)
        ref.prefill()
        got = DeviceProblem(inp, 64)
        got.workspace = None  # the no-alloc call receives no workspace
        _noalloc(got)
        torch.cuda.synchronize()
        assert _maxrel(io_float(got.o), io_float(ref.o), U_BF16) <= TOL_O
        assert _maxrel(got.state.cpu().numpy(), ref.state.cpu().numpy()) <= TOL_S
        assert np.array_equal(io_numpy(got.conv_state), io_numpy(ref.conv_state))
    assert gdn.device_status() == 0


def test_prefill_noalloc_fp32_chunk16_matches_prefill_on_two_calls():
    """fp32 io at chunk 16 takes the token-recurrent kernel, with the varlen
    schedule of several sequences written into the built-in scratch array."""
    geo = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32, io_dtype="f32")
    problems = [gi.make_prefill_inputs(geo, [64, 3, 0, 17, 40], seed=43, zero_init=False),
                gi.make_prefill_inputs(geo, [5, 64, 1], seed=44, zero_init=False)]
    for inp in problems:
        ref = DeviceProblem(inp, 16)
        ref.prefill()
        got = DeviceProblem(inp, 16)
        got.workspace = None
        _noalloc(got)
        torch.cuda.synchronize()
        assert _maxrel(io_float(got.o), io_float(ref.o), 2.0 ** -24) <= 1e-5
        assert _maxrel(got.state.cpu().numpy(), ref.state.cpu().numpy()) <= 1e-5
        assert np.array_equal(io_numpy(got.conv_state), io_numpy(ref.conv_state))
    assert gdn.device_status() == 0


def test_prefill_noalloc_rejects_oversized_problem():
    geo = gi.Geometry(num_k_heads=1, num_v_heads=1, head_k_dim=32, head_v_dim=32)
    cfg = gdn.make_config(geo)
    T = 64 * 1024 * 1024  # chunk map alone exceeds the built-in scratch
    need = gdn.prefill_workspace_size(cfg, T, 1, 16)
    assert need > 4 * 1024 * 1024
    cu = np.array([0, T], np.int32)
    dummy = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill_noalloc(cfg, (dummy,) * 4, dummy, dummy, dummy, dummy, dummy, cu, 16, 0, dummy, dummy, dummy)
    assert e.value.name == "GDN_E_WORKSPACE" and "scratch" in str(e.value)
