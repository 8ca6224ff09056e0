"""Shared helpers of the GPU parity tests (CUDA path through the C ABI vs the
float64 oracle)."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from linear_attention_recurrence_deltanet_b200 import inputs as gi
from linear_attention_recurrence_deltanet_b200.device import DeviceProblem, io_float, io_numpy, io_tensor

# Tolerances: max |x - ref| / max |ref|, per sequence and per tensor.
TOL_O_BF16 = 2e-3
TOL_S_BF16 = 1e-3
TOL_F32 = 1e-5


# Unit roundoff of the io dtypes: an output stored in bf16 carries one final
# rounding of up to U_BF16 * |value| that no kernel can avoid.
U_BF16 = 2.0 ** -8
U_F32 = 2.0 ** -24


def maxrel(x: np.ndarray, ref: np.ndarray, round_u: float = 0.0) -> float:
    """max |x - ref| / max |ref|.  With round_u > 0, each element's error is
    first reduced by the final rounding allowance round_u * |ref| (outputs
    stored in a narrower dtype than the float64 reference)."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    if not ref.size:
        return 0.0
    err = np.abs(x - ref)
    if round_u:
        err = np.maximum(err - round_u * np.abs(ref), 0.0)
    den = float(np.max(np.abs(ref)))
    num = float(np.max(err))
    return num if den == 0.0 else num / den


def io_round(geo) -> float:
    return U_BF16 if geo.io_dtype == "bf16" else U_F32


def head_cols(geo, heads):
    dv = geo.head_v_dim
    return np.concatenate([np.arange(h * dv, (h + 1) * dv) for h in heads])


def compare_prefill(inp, o_gpu, st_gpu, o_ref, st_ref, tol_o, tol_s, heads=None):
    """Per-sequence max-relative errors; returns (worst_o, worst_s)."""
    geo = inp.geo
    heads = list(range(geo.num_v_heads)) if heads is None else list(heads)
    cols = head_cols(geo, heads)
    cu = inp.cu_seqlens
    worst_o = worst_s = 0.0
    for n in range(inp.num_seqs):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        if t1 > t0:
            e = maxrel(o_gpu[t0:t1][:, cols], o_ref[t0:t1][:, cols], io_round(geo))
            worst_o = max(worst_o, e)
            assert e <= tol_o, f"seq {n}: o max-rel error {e:.3e} > {tol_o}"
        e = maxrel(st_gpu[n, heads], st_ref[n, heads])
        worst_s = max(worst_s, e)
        assert e <= tol_s, f"seq {n}: state max-rel error {e:.3e} > {tol_s}"
    return worst_o, worst_s


def run_gpu_prefill(inp, chunk, flags=0):
    dp = DeviceProblem(inp, chunk)
    dp.prefill(flags)
    torch.cuda.synchronize()
    return dp, io_float(dp.o), dp.state.cpu().numpy().astype(np.float64), io_numpy(dp.conv_state)


def ref_hist_bits(inp, hist_f32):
    """Oracle conv history (float32 exact values) in the io dtype's encoding."""
    if inp.geo.io_dtype == "bf16":
        return gi.bf16_bits_from_f32(hist_f32)
    return np.asarray(hist_f32, np.float32)
