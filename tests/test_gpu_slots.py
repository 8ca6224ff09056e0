"""Slot-indexed state pools through the C ABI (continuous batching).

Row n of a batch reads and writes pool slot state_indices[n].  The indexed
calls run the same arithmetic as the unindexed ones, so against an unindexed
call on a pool holding the batch's slots in batch order they must agree bit
for bit; slots outside the batch must not change at all; padding rows
(negative slots) write zero outputs (decode) or run from a zero state without
storing it (prefill).  A batch that mixes prefill sequences with length-1
decode steps is checked against the float64 oracle.
"""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi
from linear_attention_recurrence_deltanet_b200.device import io_float, io_numpy, io_tensor
from gpu_common import TOL_F32, TOL_O_BF16, TOL_S_BF16, U_BF16, U_F32, maxrel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.lib()
    yield
    assert gdn.device_status() == 0


def pool(geo, slots, seed):
    conv, st = gi.make_initial_state(geo, slots, seed, zero=False)
    return conv, st


def i32(x):
    return torch.tensor(list(x), dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("io,Hk,Hv,d", [("bf16", 2, 6, 128), ("f32", 2, 6, 128), ("bf16", 2, 4, 64),
                                        ("f32", 1, 2, 32)])
def test_indexed_decode_step_equals_unindexed_on_gathered_slots(io, Hk, Hv, d):
    geo = gi.Geometry(num_k_heads=Hk, num_v_heads=Hv, head_k_dim=d, head_v_dim=d, io_dtype=io)
    cfg = gdn.make_config(geo)
    params = tuple(torch.from_numpy(p).cuda() for p in gi.make_params(geo, 5))
    P, idx = 6, [4, 0, 5, 2]
    N = len(idx)
    conv0, st0 = pool(geo, P, 6)
    toks = [io_tensor(x) for x in gi.make_decode_step_tokens(geo, N, 7, 0)]
    # indexed, on the pool
    conv, st = io_tensor(conv0), torch.from_numpy(st0).cuda()
    o = torch.full((N, geo.value_dim), 3.0, dtype=toks[0].dtype, device="cuda")
    gdn.decode_step_indexed(cfg, params, *toks, N, i32(idx), P, conv, st, o)
    # unindexed, on the gathered slots
    convg, stg = io_tensor(conv0[idx]), torch.from_numpy(np.ascontiguousarray(st0[idx])).cuda()
    og = torch.empty_like(o)
    gdn.decode_step(cfg, params, *toks, N, convg, stg, og)
    torch.cuda.synchronize()
    assert np.array_equal(io_numpy(o), io_numpy(og))
    convn, stn = io_numpy(conv), st.cpu().numpy()
    assert np.array_equal(convn[idx], io_numpy(convg)) and np.array_equal(stn[idx], stg.cpu().numpy())
    others = [s for s in range(P) if s not in idx]
    assert np.array_equal(convn[others], io_numpy(io_tensor(conv0))[others])
    assert np.array_equal(stn[others], st0[others])


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_indexed_decode_padding_and_out_of_pool_rows(io):
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, io_dtype=io)
    cfg = gdn.make_config(geo)
    params = tuple(torch.from_numpy(p).cuda() for p in gi.make_params(geo, 8))
    P = 3
    conv0, st0 = pool(geo, P, 9)
    toks = [io_tensor(x) for x in gi.make_decode_step_tokens(geo, 3, 10, 0)]
    conv, st = io_tensor(conv0), torch.from_numpy(st0).cuda()
    o = torch.full((3, geo.value_dim), 3.0, dtype=toks[0].dtype, device="cuda")
    gdn.decode_step_indexed(cfg, params, *toks, 3, i32([2, -1, 0]), P, conv, st, o)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    on = io_float(o)
    assert np.all(on[1] == 0.0) and np.all(np.isfinite(on)) and not np.all(on[0] == 0.0)
    assert np.array_equal(io_numpy(conv)[1], io_numpy(io_tensor(conv0))[1])
    assert np.array_equal(st.cpu().numpy()[1], st0[1])
    # a slot past the pool: the row is skipped and the status word says so
    conv, st = io_tensor(conv0), torch.from_numpy(st0).cuda()
    gdn.decode_step_indexed(cfg, params, *toks, 3, i32([1, 7, -3]), P, conv, st, o)
    torch.cuda.synchronize()
    assert gdn.device_status() == 3
    assert gdn.device_status() == 0
    assert np.all(io_float(o)[1:] == 0.0)
    sn = st.cpu().numpy()
    assert np.array_equal(sn[[0, 2]], st0[[0, 2]]) and not np.array_equal(sn[1], st0[1])


@pytest.mark.parametrize("K", [2, 3])
def test_indexed_multi_decode_equals_unindexed(K):
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, io_dtype="bf16")
    cfg = gdn.make_config(geo)
    params = tuple(torch.from_numpy(p).cuda() for p in gi.make_params(geo, 11))
    P, idx = 5, [3, -1, 1]
    N = len(idx)
    conv0, st0 = pool(geo, P, 12)
    toks = [gi.make_decode_step_tokens(geo, N, 13, s) for s in range(K)]
    multi = [io_tensor(np.ascontiguousarray(np.stack([t[i] for t in toks], axis=1))) for i in range(4)]
    accept = i32([K, 1, 1])
    # indexed verify then commit
    conv, st = io_tensor(conv0), torch.from_numpy(st0).cuda()
    ov = torch.empty((N, K, geo.value_dim), dtype=multi[0].dtype, device="cuda")
    oc = torch.full_like(ov, 2.0)
    gdn.decode_multi_indexed(cfg, params, *multi, N, K, False, None, i32(idx), P, conv, st, ov)
    gdn.decode_multi_indexed(cfg, params, *multi, N, K, True, accept, i32(idx), P, conv, st, oc)
    # unindexed on the real rows (0 and 2 of the batch)
    real = [0, 2]
    mr = [t[real].contiguous() for t in multi]
    convg = io_tensor(conv0[[idx[n] for n in real]])
    stg = torch.from_numpy(np.ascontiguousarray(st0[[idx[n] for n in real]])).cuda()
    ovg = torch.empty((2, K, geo.value_dim), dtype=multi[0].dtype, device="cuda")
    ocg = torch.full_like(ovg, 2.0)
    gdn.decode_multi(cfg, params, *mr, 2, K, False, None, convg, stg, ovg)
    gdn.decode_multi(cfg, params, *mr, 2, K, True, i32([K, 1]), convg, stg, ocg)
    torch.cuda.synchronize()
    assert np.array_equal(io_numpy(ov)[real], io_numpy(ovg))
    assert np.array_equal(io_numpy(oc)[real], io_numpy(ocg))
    assert np.all(io_float(ov)[1] == 0.0) and np.all(io_float(oc)[1] == 0.0)
    stn, convn = st.cpu().numpy(), io_numpy(conv)
    assert np.array_equal(stn[[3, 1]], stg.cpu().numpy()) and np.array_equal(convn[[3, 1]], io_numpy(convg))
    for s in (0, 2, 4):
        assert np.array_equal(stn[s], st0[s]) and np.array_equal(convn[s], io_numpy(io_tensor(conv0))[s])


def prefill_bufs(geo, lengths, seed):
    inp = gi.make_prefill_inputs(geo, lengths, seed, zero_init=False)
    toks = [io_tensor(x) for x in (inp.qkv, inp.z, inp.a, inp.b)]
    params = tuple(torch.from_numpy(np.ascontiguousarray(p, np.float32)).cuda()
                   for p in (inp.conv_w, inp.A_log, inp.dt_bias, inp.norm_w))
    cu = np.ascontiguousarray(inp.cu_seqlens, np.int32)
    return inp, toks, params, cu, torch.from_numpy(cu).cuda()


@pytest.mark.parametrize("chunk,flags", [(64, 0), (64, gdn.PREFILL_FUSED), (16, 0), (64, gdn.ZERO_INIT_STATE)])
def test_indexed_prefill_equals_unindexed_on_gathered_slots(chunk, flags):
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, io_dtype="bf16")
    cfg = gdn.make_config(geo)
    lengths = [150, 1, 64, 0, 77]
    idx = [5, 0, 2, 6, 3]
    N, P = len(lengths), 7
    inp, toks, params, cu, cu_dev = prefill_bufs(geo, lengths, 21)
    conv0, st0 = pool(geo, P, 22)
    T = int(cu[-1])
    # indexed
    conv, st = io_tensor(conv0), torch.from_numpy(st0).cuda()
    o = torch.empty((T, geo.value_dim), dtype=toks[0].dtype, device="cuda")
    ws = torch.empty(gdn.prefill_indexed_workspace_size(cfg, T, N, chunk), dtype=torch.uint8, device="cuda")
    gdn.prefill_indexed(cfg, params, *toks, cu_dev, cu, i32(idx), P, chunk, flags, conv, st, o, ws)
    # unindexed on the gathered slots
    convg, stg = io_tensor(conv0[idx]), torch.from_numpy(np.ascontiguousarray(st0[idx])).cuda()
    og = torch.empty_like(o)
    wsg = torch.empty(max(gdn.prefill_workspace_size(cfg, T, N, chunk), 256), dtype=torch.uint8, device="cuda")
    gdn.prefill(cfg, params, *toks, cu_dev, cu, chunk, flags, convg, stg, og, wsg)
    torch.cuda.synchronize()
    assert np.array_equal(io_numpy(o), io_numpy(og))
    stn, convn = st.cpu().numpy(), io_numpy(conv)
    assert np.array_equal(stn[idx], stg.cpu().numpy()) and np.array_equal(convn[idx], io_numpy(convg))
    assert np.array_equal(stn[[1, 4]], st0[[1, 4]])
    assert np.array_equal(convn[[1, 4]], io_numpy(io_tensor(conv0))[[1, 4]])


def test_indexed_prefill_padding_row_runs_from_zero_and_is_not_stored():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, io_dtype="bf16")
    cfg = gdn.make_config(geo)
    lengths = [90, 40]
    inp, toks, params, cu, cu_dev = prefill_bufs(geo, lengths, 31)
    conv0, st0 = pool(geo, 2, 32)
    T = int(cu[-1])
    conv, st = io_tensor(conv0), torch.from_numpy(st0).cuda()
    o = torch.empty((T, geo.value_dim), dtype=toks[0].dtype, device="cuda")
    ws = torch.empty(gdn.prefill_indexed_workspace_size(cfg, T, 2, 64), dtype=torch.uint8, device="cuda")
    gdn.prefill_indexed(cfg, params, *toks, cu_dev, cu, i32([-1, 1]), 2, 64, 0, conv, st, o, ws)
    # reference: the padding row from zeros, the other from slot 1
    convg = io_tensor(np.stack([np.zeros_like(conv0[0]), conv0[1]]))
    stg = torch.from_numpy(np.stack([np.zeros_like(st0[0]), st0[1]])).cuda()
    og = torch.empty_like(o)
    wsg = torch.empty(gdn.prefill_workspace_size(cfg, T, 2, 64), dtype=torch.uint8, device="cuda")
    gdn.prefill(cfg, params, *toks, cu_dev, cu, 64, 0, convg, stg, og, wsg)
    torch.cuda.synchronize()
    assert np.array_equal(io_numpy(o), io_numpy(og))
    stn = st.cpu().numpy()
    assert np.array_equal(stn[0], st0[0]) and np.array_equal(stn[1], stg.cpu().numpy()[1])


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_mixed_prefill_and_decode_batch_matches_oracle(io):
    """One indexed call over prefill sequences and length-1 decode steps;
    every row against the float64 oracle on its own slot."""
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, io_dtype=io)
    cfg = gdn.make_config(geo)
    lengths = [1, 200, 1, 1, 67, 1]
    idx = [4, 1, 0, 6, 2, 5]
    N, P = len(lengths), 7
    inp, toks, params, cu, cu_dev = prefill_bufs(geo, lengths, 41)
    conv0, st0 = pool(geo, P, 42)
    T = int(cu[-1])
    conv, st = io_tensor(conv0), torch.from_numpy(st0).cuda()
    o = torch.empty((T, geo.value_dim), dtype=toks[0].dtype, device="cuda")
    ws = torch.empty(gdn.prefill_indexed_workspace_size(cfg, T, N, 64), dtype=torch.uint8, device="cuda")
    gdn.prefill_indexed(cfg, params, *toks, cu_dev, cu, i32(idx), P, 64, 0, conv, st, o, ws)
    torch.cuda.synchronize()
    f = (lambda x: gi.f32_from_bf16_bits(x)) if io == "bf16" else (lambda x: np.asarray(x, np.float32))
    o_ref, st_ref, h_ref = oracle.prefill(geo, (inp.conv_w, inp.A_log, inp.dt_bias, inp.norm_w), f(inp.qkv),
                                          f(inp.z), f(inp.a), f(inp.b), cu, f(conv0[idx]), st0[idx])
    tol_o, tol_s, u = (TOL_O_BF16, TOL_S_BF16, U_BF16) if io == "bf16" else (TOL_F32, TOL_F32, U_F32)
    on, stn, convn = io_float(o), st.cpu().numpy(), io_numpy(conv)
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        assert maxrel(on[t0:t1], o_ref[t0:t1], u) <= tol_o, n
        assert maxrel(stn[idx[n]], st_ref[n]) <= tol_s, n
        want = gi.bf16_bits_from_f32(h_ref[n]) if io == "bf16" else np.asarray(h_ref[n], np.float32)
        assert np.array_equal(convn[idx[n]], want), n
    assert np.array_equal(stn[3], st0[3])
