"""The sequence-parallel prefill of one long sequence (gdn_prefill_seqpar)
through the C ABI: against the float64 oracle and against gdn_prefill of the
same sequence.

The segmented carry reassociates the state products, so it agrees with
gdn_prefill within rounding, not bit for bit; both must meet the oracle
tolerances (bf16: o <= 2e-3, state <= 1e-3).  The conv history comes from
the same conv/prep kernels and must match gdn_prefill's bit for bit.
Few value heads per GPU (2 key / 6 value heads, an eighth of the Qwen
layer's heads) is the configuration this path is for.
"""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi
from linear_attention_recurrence_deltanet_b200.device import DeviceProblem, io_float, io_numpy
from gpu_common import TOL_O_BF16, TOL_S_BF16, U_BF16, compare_prefill, maxrel, ref_hist_bits

pytestmark = pytest.mark.gpu

SHARD = gi.Geometry(num_k_heads=2, num_v_heads=6)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.lib()
    yield
    assert gdn.device_status() == 0


def run_seqpar(inp, segments, flags=0):
    dp = DeviceProblem(inp, 64)
    T = inp.total_tokens
    ws = torch.empty(gdn.prefill_seqpar_workspace_size(dp.cfg, T, segments), dtype=torch.uint8, device="cuda")
    used = gdn.prefill_seqpar(dp.cfg, dp.params, dp.qkv, dp.z, dp.a, dp.b, T, segments, flags, dp.conv_state,
                              dp.state, dp.o, ws)
    torch.cuda.synchronize()
    return used, io_float(dp.o), dp.state.cpu().numpy().astype(np.float64), io_numpy(dp.conv_state)


def close_to_plain(o, st, o_p, st_p):
    """Both outputs are rounded to bf16 independently: allow one rounding on
    each side (2 x 2^-8 |ref|) before the o tolerance."""
    assert maxrel(o, o_p, 2 * U_BF16) <= TOL_O_BF16
    assert maxrel(st, st_p) <= TOL_S_BF16


def run_plain(inp, flags=0):
    dp = DeviceProblem(inp, 64)
    dp.prefill(flags)
    torch.cuda.synchronize()
    return io_float(dp.o), dp.state.cpu().numpy().astype(np.float64), io_numpy(dp.conv_state)


@pytest.mark.parametrize("T,segments,zero_init", [
    (2577, 1, True),    # one segment: the two chain passes around a trivial composition
    (2577, 2, True),
    (2577, 7, False),   # 41 chunks in segments of 6 (the last one short and ragged), non-zero start
    (2577, 0, False),   # segment count from the SM count
    (64 * 40, 40, True),  # one chunk per segment
    (100, 3, False),    # two chunks: at most two segments
])
def test_seqpar_matches_oracle_and_prefill(T, segments, zero_init):
    inp = gi.make_prefill_inputs(SHARD, [T], seed=31 + T + segments, zero_init=zero_init)
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    used, o, st, hist = run_seqpar(inp, segments)
    nchunks = -(-T // 64)
    assert 1 <= used <= nchunks
    if segments:
        seg = -(-nchunks // min(segments, nchunks))
        assert used == -(-nchunks // seg)
    compare_prefill(inp, o, st, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    assert np.array_equal(hist, ref_hist_bits(inp, hist_ref))
    o_p, st_p, hist_p = run_plain(inp)
    assert np.array_equal(hist, hist_p)
    close_to_plain(o, st, o_p, st_p)


def test_seqpar_long_context_matches_oracle():
    """16384 tokens (256 chunks) in 16 segments, non-zero start."""
    inp = gi.make_prefill_inputs(SHARD, [16384], seed=41, zero_init=False)
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    used, o, st, hist = run_seqpar(inp, 16)
    assert used == 16
    compare_prefill(inp, o, st, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    assert np.array_equal(hist, ref_hist_bits(inp, hist_ref))


def test_seqpar_flags_zero_state_and_history():
    """GDN_ZERO_INIT_STATE / GDN_ZERO_INIT_CONV ignore the incoming caches,
    as gdn_prefill's do."""
    inp = gi.make_prefill_inputs(SHARD, [1000], seed=43, zero_init=False)
    flags = gdn.ZERO_INIT_STATE | gdn.ZERO_INIT_CONV
    _, o, st, hist = run_seqpar(inp, 4, flags)
    o_p, st_p, hist_p = run_plain(inp, flags)
    assert np.array_equal(hist, hist_p)
    close_to_plain(o, st, o_p, st_p)


def test_seqpar_qwen_heads_sampled():
    """All 48 value heads (where the path brings no speed-up) still compute
    the same result: oracle on 4 sampled heads."""
    inp = gi.make_prefill_inputs(gi.QWEN_GEO, [3000], seed=44, zero_init=False)
    heads = [0, 17, 30, 47]
    o_ref, st_ref, _ = oracle.prefill_inputs(inp, heads=heads)
    _, o, st, _ = run_seqpar(inp, 3)
    compare_prefill(inp, o, st, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16, heads=heads)


def test_seqpar_rejects_unsupported_and_empty():
    geo64 = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=64, head_v_dim=64)
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill_seqpar_workspace_size(gdn.make_config(geo64), 1000, 0)
    assert e.value.name == "GDN_E_UNSUPPORTED"
    inp = gi.make_prefill_inputs(SHARD, [0], seed=45, zero_init=False)
    dp = DeviceProblem(inp, 64)
    st0 = dp.state.clone()
    ws = torch.empty(gdn.prefill_seqpar_workspace_size(dp.cfg, 0, 0), dtype=torch.uint8, device="cuda")
    gdn.prefill_seqpar(dp.cfg, dp.params, dp.qkv, dp.z, dp.a, dp.b, 0, 0, 0, dp.conv_state, dp.state, dp.o, ws)
    torch.cuda.synchronize()
    assert torch.equal(dp.state, st0)
