"""The bf16 projection GEMM (gdn_gemm_bf16, gdn_project_in, gdn_project_out)
through the C ABI against the float64 oracle.  The shapes reach all three
kernels: one CTA per 128-row tile, a CTA pair per 256-row tile, and (up to
128 rows) a cluster of CTAs per tile splitting K and reducing through
distributed shared memory.

Inputs are bf16; the kernel accumulates in fp32 and rounds once to bf16.
After taking off that final rounding (U_BF16 * |ref| per element), the error
left is the fp32 accumulation of K <= 6144 products.  Each bf16 x bf16
product is exact in fp32, and summing K of them loses a few units of 2^-24
of the partial sums, far below TOL_GEMM = 1e-4 of max |ref|.
"""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi
from linear_attention_recurrence_deltanet_b200.device import io_float, io_tensor
from gpu_common import U_BF16, maxrel

pytestmark = pytest.mark.gpu

TOL_GEMM = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.lib()
    yield
    assert gdn.device_status() == 0


def operands(M, K, N, seed):
    x = gi.make_hidden_states(M, K, seed)
    w = gi.make_hidden_states(N, K, seed + 1)
    return x, w


def check(y_gpu, x_bits, w_bits, rows=None):
    ref = oracle.project(gi.f32_from_bf16_bits(x_bits), gi.f32_from_bf16_bits(w_bits), rows=rows)
    got = io_float(y_gpu) if rows is None else io_float(y_gpu)[rows]
    e = maxrel(got, ref, U_BF16)
    assert e <= TOL_GEMM, f"max-rel error {e:.3e} > {TOL_GEMM}"
    return e


@pytest.mark.parametrize("M,K,N,tile_n", [
    (1, 8, 1, 0),          # one element; K below one stage, N below one 8-column group
    (130, 72, 200, 64),    # ragged M tile, K not a multiple of 64, ragged 64-wide N tile
    (257, 520, 1000, 128),
    (300, 1024, 1030, 256),  # row pitch not a multiple of 8: every group takes the element path
    (200, 256, 512, 256),  # fewer than 256 rows: one CTA per tile at the widest tile
    (256, 128, 384, 0),    # exactly one 256-row tile for a CTA pair
    (64, 5120, 16480, 0),  # decode-sized input projection: K split over a cluster of 2
    (33, 640, 1000, 0),    # ragged rows, one CTA per tile
    (40, 6144, 5120, 128),  # K split over a cluster of 3, partial rows padded to 64
    (128, 6144, 5120, 0),  # decode-sized output projection shape at 128 rows: K split over 3
    (512, 6144, 5120, 0),
])
def test_gemm_matches_oracle(M, K, N, tile_n):
    x, w = operands(M, K, N, seed=M + K + N)
    xt, wt = io_tensor(x), io_tensor(w)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    gdn.gemm_bf16(xt, wt, y, tile_n=tile_n)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any()
    check(y, x, w)


@pytest.mark.parametrize("tile_n", [32, 64, 96, 128, 160, 224, 256])
def test_every_tile_width(tile_n):
    M, K, N = 384, 640, 704
    x, w = operands(M, K, N, seed=7)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    gdn.gemm_bf16(io_tensor(x), io_tensor(w), y, tile_n=tile_n)
    torch.cuda.synchronize()
    check(y, x, w)


def test_empty_problem_writes_nothing():
    x, w = operands(4, 64, 8, seed=3)
    y = torch.full((4, 8), 7.0, dtype=torch.bfloat16, device="cuda")
    gdn.lib().gdn_gemm_bf16(io_tensor(x).data_ptr(), 0, 64, io_tensor(w).data_ptr(), 8, y.data_ptr(), 0,
                            torch.cuda.current_stream().cuda_stream)
    gdn.lib().gdn_gemm_bf16(io_tensor(x).data_ptr(), 4, 64, io_tensor(w).data_ptr(), 0, y.data_ptr(), 0,
                            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())


def project_in_case(geo, T, hidden, seed, rows=None):
    w_in, _ = gi.make_projection_weights(geo, hidden, seed)
    x = gi.make_hidden_states(T, hidden, seed)
    out = dict(qkv=torch.full((T, geo.conv_dim), float("nan"), dtype=torch.bfloat16, device="cuda"),
               z=torch.full((T, geo.value_dim), float("nan"), dtype=torch.bfloat16, device="cuda"),
               a=torch.full((T, geo.num_v_heads), float("nan"), dtype=torch.bfloat16, device="cuda"),
               b=torch.full((T, geo.num_v_heads), float("nan"), dtype=torch.bfloat16, device="cuda"))
    gdn.project_in(gdn.make_config(geo), io_tensor(x), io_tensor(w_in), out["qkv"], out["z"], out["a"], out["b"])
    torch.cuda.synchronize()
    ref = oracle.project(gi.f32_from_bf16_bits(x), gi.f32_from_bf16_bits(w_in), rows=rows)
    refs = oracle.split_projection(geo, ref)
    for name, r in zip(("qkv", "z", "a", "b"), refs):
        got = io_float(out[name]) if rows is None else io_float(out[name])[rows]
        assert not np.isnan(io_float(out[name])).any(), name
        # the tolerance is relative to the whole projection's scale
        e = float(np.max(np.maximum(np.abs(got - r) - U_BF16 * np.abs(r), 0.0))) / float(np.max(np.abs(ref)))
        assert e <= TOL_GEMM, f"{name}: {e:.3e}"


def test_project_in_small_heads_route_every_column():
    """Hv = 4: a and b are 4 columns wide, so 8-column groups straddle z, a
    and b and take the element path."""
    project_in_case(gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32), 70, 96, seed=21)


def test_project_in_qwen_decode_batch():
    project_in_case(gi.QWEN_GEO, 64, gi.QWEN_HIDDEN, seed=22)


def test_project_in_qwen_prefill_sampled_rows():
    """The full T=4096 input projection (16480 output columns); the oracle
    checks 24 rows, among them the first and last of the first, a middle and
    the last 128-row tile."""
    rows = sorted({0, 127, 128, 2047, 2048, 4095} | set(np.random.default_rng(23).integers(0, 4096, 18).tolist()))
    project_in_case(gi.QWEN_GEO, 4096, gi.QWEN_HIDDEN, seed=23, rows=rows)


def test_project_out_qwen_prefill_sampled_rows():
    geo = gi.QWEN_GEO
    T = 4096
    _, w_out = gi.make_projection_weights(geo, gi.QWEN_HIDDEN, 24)
    o = gi.make_hidden_states(T, geo.value_dim, 24)
    y = torch.full((T, gi.QWEN_HIDDEN), float("nan"), dtype=torch.bfloat16, device="cuda")
    gdn.project_out(gdn.make_config(geo), io_tensor(o), io_tensor(w_out), y)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any()
    rows = sorted({0, 127, 128, 255, 256, 4095} | set(np.random.default_rng(24).integers(0, T, 21).tolist()))
    check(y, o, w_out, rows=rows)


def test_project_out_qwen_decode_batch():
    """64 tokens through the output projection (6144 -> 5120): the K-split
    cluster path, every row against the oracle."""
    geo = gi.QWEN_GEO
    _, w_out = gi.make_projection_weights(geo, gi.QWEN_HIDDEN, 25)
    o = gi.make_hidden_states(64, geo.value_dim, 25)
    y = torch.full((64, gi.QWEN_HIDDEN), float("nan"), dtype=torch.bfloat16, device="cuda")
    gdn.project_out(gdn.make_config(geo), io_tensor(o), io_tensor(w_out), y)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any()
    check(y, o, w_out)
