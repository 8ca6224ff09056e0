"""Failure handling on the GPU without a fault: a bounded wait that runs out
reports through the device status word and leaves the context usable, and
no entry point writes outside the buffers it is given (guard bands of a known
byte pattern around every output, checked byte for byte after the call)."""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi
from linear_attention_recurrence_deltanet_b200.device import DeviceProblem, io_float, io_tensor
from gpu_common import TOL_O_BF16, TOL_S_BF16, compare_prefill

pytestmark = pytest.mark.gpu

GUARD_BYTES = 4096
PATTERN = 0xA5


def test_wait_expiry_reports_status_and_next_launch_runs_clean():
    assert torch.cuda.is_available()
    assert gdn.device_status() == 0
    gdn.debug_wait_expiry(100)  # an mbarrier nothing arrives on, 100 us limit
    assert gdn.device_status() == 1  # kStatusWaitTimeout, read and cleared
    assert gdn.device_status() == 0
    # the context is intact: an ordinary prefill right after matches the oracle
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [70, 5, 129], seed=51, zero_init=False)
    o_ref, st_ref, _ = oracle.prefill_inputs(inp)
    dp = DeviceProblem(inp, 64)
    dp.prefill()
    torch.cuda.synchronize()
    compare_prefill(inp, io_float(dp.o), dp.state.cpu().numpy(), o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    assert gdn.device_status() == 0


def _guarded(t: torch.Tensor):
    """A copy of `t` placed between two guard bands of PATTERN bytes inside one
    allocation; returns (view, raw)."""
    nbytes = t.numel() * t.element_size()
    raw = torch.full((GUARD_BYTES + nbytes + GUARD_BYTES,), PATTERN, dtype=torch.uint8, device=t.device)
    view = raw[GUARD_BYTES:GUARD_BYTES + nbytes].view(t.dtype).view(t.shape)
    view.copy_(t)
    return view, raw


def _guards_intact(raw: torch.Tensor) -> bool:
    g = torch.cat([raw[:GUARD_BYTES], raw[-GUARD_BYTES:]])
    return bool((g == PATTERN).all())


@pytest.mark.parametrize("chunk,flags", [(64, 0), (64, gdn.PREFILL_AFFINE), (64, gdn.PREFILL_FUSED),
                                         (64, gdn.PREFILL_RECURRENT), (16, 0), (32, 0), (128, 0)])
def test_prefill_writes_nothing_outside_its_buffers(chunk, flags):
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [1, 63, 64, 65, 130, 0, 3], seed=52, zero_init=False)
    o_ref, st_ref, _ = oracle.prefill_inputs(inp)
    dp = DeviceProblem(inp, chunk)
    dp.o, o_raw = _guarded(dp.o)
    dp.state, st_raw = _guarded(dp.state)
    dp.conv_state, cv_raw = _guarded(dp.conv_state)
    ws = dp.workspace
    if ws is not None:
        dp.workspace, ws_raw = _guarded(ws)
    dp.prefill(flags)
    torch.cuda.synchronize()
    for raw in (o_raw, st_raw, cv_raw) + ((ws_raw,) if ws is not None else ()):
        assert _guards_intact(raw)
    compare_prefill(inp, io_float(dp.o), dp.state.cpu().numpy(), o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    assert gdn.device_status() == 0


def test_decode_writes_nothing_outside_its_buffers():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [4, 4, 4], seed=53, zero_init=False)
    dp = DeviceProblem(inp, 64)
    N = 3
    o, o_raw = _guarded(torch.empty((N, geo.value_dim), dtype=torch.bfloat16, device="cuda"))
    st, st_raw = _guarded(dp.state)
    cv, cv_raw = _guarded(dp.conv_state)
    for t in range(4):  # token t of every sequence
        qkv = torch.cat([dp.qkv[4 * n + t:4 * n + t + 1] for n in range(N)])
        z = torch.cat([dp.z[4 * n + t:4 * n + t + 1] for n in range(N)])
        a = torch.cat([dp.a[4 * n + t:4 * n + t + 1] for n in range(N)])
        b = torch.cat([dp.b[4 * n + t:4 * n + t + 1] for n in range(N)])
        gdn.decode_step(dp.cfg, dp.params, qkv, z, a, b, N, cv, st, o)
    torch.cuda.synchronize()
    for raw in (o_raw, st_raw, cv_raw):
        assert _guards_intact(raw)
    assert gdn.device_status() == 0
