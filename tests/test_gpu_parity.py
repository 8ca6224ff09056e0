"""GPU parity: the CUDA path, called through the C ABI, against the float64
oracle on the same seeded inputs.

Tolerances (max |x - ref| / max |ref| per sequence and tensor): bf16 inputs
o <= 2e-3 and final state <= 1e-3; fp32 inputs <= 1e-5.  Conv histories,
varlen boundaries and the schedule are compared bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrence_deltanet_b200 as gdn
from linear_attention_recurrence_deltanet_b200 import inputs as gi
from linear_attention_recurrence_deltanet_b200.device import DeviceProblem, io_float, io_numpy, io_tensor
from gpu_common import (TOL_F32, TOL_O_BF16, TOL_S_BF16, U_BF16, U_F32, compare_prefill, maxrel, ref_hist_bits,
                        run_gpu_prefill)

pytestmark = pytest.mark.gpu

RECURRENT = gdn.PREFILL_RECURRENT
FUSED = gdn.PREFILL_FUSED
FACTORED = gdn.PREFILL_FACTORED
AFFINE = gdn.PREFILL_AFFINE


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    gdn.lib()
    yield
    assert gdn.device_status() == 0


def _tol(geo):
    return (TOL_F32, TOL_F32) if geo.io_dtype == "f32" else (TOL_O_BF16, TOL_S_BF16)


# ------------------------------------------------------------------ tiny fp32 mixer


def test_tiny_fp32_prefill_matches_oracle():
    inp = gi.workload_inputs("tiny_fp32_t64")
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    _, o, st, hist = run_gpu_prefill(inp, 16)
    compare_prefill(inp, o, st, o_ref, st_ref, TOL_F32, TOL_F32)
    assert np.array_equal(hist, ref_hist_bits(inp, hist_ref))


def test_tiny_fp32_decode_steps_match_oracle():
    inp = gi.workload_inputs("tiny_fp32_t64")
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    dp = DeviceProblem(inp, 16)
    o = torch.empty((1, inp.geo.value_dim), dtype=dp.qkv.dtype, device="cuda")
    for t in range(64):
        dp.decode(dp.qkv[t:t + 1], dp.z[t:t + 1], dp.a[t:t + 1], dp.b[t:t + 1], o)
        assert maxrel(io_float(o)[0], o_ref[t], U_F32) <= TOL_F32, t
    assert maxrel(dp.state.cpu().numpy(), st_ref) <= TOL_F32
    assert np.array_equal(io_numpy(dp.conv_state), ref_hist_bits(inp, hist_ref))


# ------------------------------------------------------------------ small shapes, edge cases


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("d,Hk,Hv", [(32, 2, 4), (64, 2, 6), (128, 1, 3)])
@pytest.mark.parametrize("zero_init", [True, False])
def test_small_varlen_prefill(io, d, Hk, Hv, zero_init):
    geo = gi.Geometry(num_k_heads=Hk, num_v_heads=Hv, head_k_dim=d, head_v_dim=d, io_dtype=io)
    lengths = [0, 1, 2, 3, 5, 17, 70, 33]
    inp = gi.make_prefill_inputs(geo, lengths, seed=21, zero_init=zero_init)
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    _, o, st, hist = run_gpu_prefill(inp, 16)
    compare_prefill(inp, o, st, o_ref, st_ref, *_tol(geo))
    assert np.array_equal(hist, ref_hist_bits(inp, hist_ref))


def test_zero_init_flags_ignore_buffers():
    geo = gi.Geometry(num_k_heads=1, num_v_heads=2, head_k_dim=64, head_v_dim=64)
    inp = gi.make_prefill_inputs(geo, [9, 40], seed=22, zero_init=True)
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    dp = DeviceProblem(inp, 16)
    dp.state.normal_()
    dp.conv_state.normal_()
    dp.prefill(gdn.ZERO_INIT_STATE | gdn.ZERO_INIT_CONV)
    torch.cuda.synchronize()
    compare_prefill(inp, io_float(dp.o), dp.state.cpu().numpy(), o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    assert np.array_equal(io_numpy(dp.conv_state), ref_hist_bits(inp, hist_ref))


def test_alpha1_beta0_leaves_state_bit_exact():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [37, 5], seed=23, zero_init=False)
    inp.a[:] = gi.bf16_bits_from_f32(np.full(inp.a.shape, -1e4, np.float32))
    inp.b[:] = gi.bf16_bits_from_f32(np.full(inp.b.shape, -1e4, np.float32))
    _, _, st, _ = run_gpu_prefill(inp, 64)
    assert np.array_equal(st.astype(np.float32), inp.state)
    # and one decode step
    dp = DeviceProblem(inp, 64)
    o = torch.empty((2, geo.value_dim), dtype=torch.bfloat16, device="cuda")
    dp.decode(dp.qkv[:2], dp.z[:2], dp.a[:2], dp.b[:2], o)
    torch.cuda.synchronize()
    assert np.array_equal(dp.state.cpu().numpy(), inp.state)


def test_varlen_boundaries_are_isolated_bit_exact():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    lengths = [50, 3, 130, 1, 77]
    inp = gi.make_prefill_inputs(geo, lengths, seed=24, zero_init=False)
    _, o1, st1, h1 = run_gpu_prefill(inp, 64)
    cu = inp.cu_seqlens
    inp.qkv[cu[2]:cu[3]] ^= np.uint16(0x0040)  # perturb every input of sequence 2
    inp.z[cu[2]:cu[3]] ^= np.uint16(0x0040)
    _, o2, st2, h2 = run_gpu_prefill(inp, 64)
    for n in range(len(lengths)):
        same = n != 2
        sl = slice(cu[n], cu[n + 1])
        assert np.array_equal(o1[sl], o2[sl]) == same, n
        assert np.array_equal(st1[n], st2[n]) == same, n
        assert np.array_equal(h1[n], h2[n]) == same, n


@pytest.mark.parametrize("chunk,flags", [(64, 0), (64, AFFINE), (16, 0), (32, 0), (128, 0), (64, FUSED)])
def test_deterministic(chunk, flags):
    """Repeated prefills give the same bits.  Every head of the 16K/48V geometry runs, so the chain kernels
    refill their operand buffers while the other clusters load memory: a buffer refilled before its last
    reader (an MMA still in flight) is done changes output bits from run to run, even when the difference is
    far inside the oracle tolerance."""
    inp = gi.make_prefill_inputs(gi.QWEN_GEO, [1, 63, 65, 130, 7, 200, 16, 17, 1000], seed=25, zero_init=False)
    dp = DeviceProblem(inp, chunk)
    ref = None
    for run in range(4):
        dp.reset_states()
        dp.o.zero_()
        dp.prefill(flags)
        torch.cuda.synchronize()
        out = (io_numpy(dp.o).copy(), dp.state.cpu().numpy().view(np.int32).copy(), io_numpy(dp.conv_state).copy())
        if ref is None:
            ref = out
            continue
        diff = [int(np.count_nonzero(x != y)) for x, y in zip(ref, out)]
        assert diff == [0, 0, 0], f"run {run}: (o, state, history) elements that differ from run 0: {diff}"


def test_schedule_matches_host_reference():
    geo = gi.Geometry(num_k_heads=1, num_v_heads=1, head_k_dim=32, head_v_dim=32)
    lengths = [5, 0, 64, 65, 5, 1, 128, 200, 0, 64]
    inp = gi.make_prefill_inputs(geo, lengths, seed=26)
    for C in (16, 64, 128):
        dp = DeviceProblem(inp, C)
        dp.workspace.zero_()
        dp.prefill()
        torch.cuda.synchronize()
        ws = dp.workspace.cpu().numpy()
        N = len(lengths)
        order = np.frombuffer(ws[:4 * N].tobytes(), np.int32)
        ref_order = sorted(range(N), key=lambda n: (-lengths[n], n))
        assert list(order) == ref_order
        off0 = ((4 * N + 255) // 256) * 256
        chunk_off = np.frombuffer(ws[off0:off0 + 4 * (N + 1)].tobytes(), np.int32)
        counts = [(L + C - 1) // C for L in lengths]
        assert list(chunk_off) == list(np.concatenate([[0], np.cumsum(counts)]))
        off1 = off0 + ((4 * (N + 1) + 255) // 256) * 256
        total = sum(counts)
        cmap = np.frombuffer(ws[off1:off1 + 16 * total].tobytes(), np.int32).reshape(total, 4)
        ref = []
        for n, L in enumerate(lengths):
            for k in range(counts[n]):
                ref.append([n, inp.cu_seqlens[n] + k * C, min(C, L - k * C), k])
        assert np.array_equal(cmap, np.array(ref, np.int32).reshape(-1, 4))


# ------------------------------------------------------------------ conv entry points


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_conv_prefill_and_step(io):
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=64, head_v_dim=64, io_dtype=io)
    lengths = [7, 0, 1, 2, 40]
    inp = gi.make_prefill_inputs(geo, lengths, seed=27, zero_init=False)
    cfg = gdn.make_config(geo)
    x = io_tensor(inp.qkv)
    w = torch.from_numpy(inp.conv_w).cuda()
    hist = io_tensor(inp.conv_state)
    y = torch.empty_like(x)
    cu = torch.from_numpy(inp.cu_seqlens).cuda()
    gdn.conv_prefill(cfg, x, w, cu, inp.cu_seqlens, hist, y)
    torch.cuda.synchronize()
    y_ref, h_ref = oracle.conv_prefill(inp.f32("qkv"), inp.conv_w, inp.cu_seqlens, inp.f32("conv_state"))
    u = U_F32 if io == "f32" else U_BF16  # one rounding of y to the io dtype
    assert maxrel(io_float(y), y_ref, u) <= 1e-6
    assert np.array_equal(io_numpy(hist), ref_hist_bits(inp, h_ref))
    # conv step: one token per sequence, from the current history
    N = len(lengths)
    xs = io_tensor(inp.qkv[:N])
    ys = torch.empty_like(xs)
    h_before = io_numpy(hist).copy()
    gdn.conv_step(cfg, xs, w, N, hist, ys)
    torch.cuda.synchronize()
    ys_ref, hs_ref = oracle.conv_prefill(inp.f32("qkv")[:N], inp.conv_w, np.arange(N + 1), h_ref)
    assert maxrel(io_float(ys), ys_ref, u) <= 1e-6
    assert np.array_equal(io_numpy(hist), ref_hist_bits(inp, hs_ref))
    assert not np.array_equal(io_numpy(hist), h_before)


# ------------------------------------------------------------------ Qwen-shaped workloads


def test_prefill_t4096_matches_oracle():
    inp = gi.workload_inputs("prefill_t4096")
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    for flags in (0, AFFINE, FUSED, RECURRENT):
        _, o, st, hist = run_gpu_prefill(inp, 64, flags | gdn.ZERO_INIT_STATE)
        eo, es = compare_prefill(inp, o, st, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
        print(f"prefill T=4096 flags={flags}: o max-rel {eo:.2e}, state max-rel {es:.2e}")
        assert np.array_equal(hist, ref_hist_bits(inp, hist_ref))


def _decode_run(steps):
    """`steps` decode steps of the B=64 workload; every output of every value
    head is compared with the oracle at every step, and every final state."""
    w = gi.WORKLOADS["decode_b64"]
    geo, seed, N = w["geo"], w["seed"], 64
    params = gi.make_params(geo, seed)
    conv0, st0 = gi.make_initial_state(geo, N, seed, zero=False)
    cfg = gdn.make_config(geo)
    dparams = tuple(torch.from_numpy(p).cuda() for p in params)
    conv = io_tensor(conv0)
    st = torch.from_numpy(st0).cuda()
    o = torch.empty((N, geo.value_dim), dtype=torch.bfloat16, device="cuda")
    ref_st, ref_hist = st0.astype(np.float64), gi.f32_from_bf16_bits(conv0)
    worst_o = worst_s = 0.0
    for s in range(steps):
        qkv, z, a, b = gi.make_decode_step_tokens(geo, N, seed, s)
        gdn.decode_step(cfg, dparams, io_tensor(qkv), io_tensor(z), io_tensor(a), io_tensor(b), N, conv, st, o)
        o_ref, ref_st, ref_hist = oracle.decode_step(geo, params, gi.f32_from_bf16_bits(qkv), gi.f32_from_bf16_bits(z),
                                                     gi.f32_from_bf16_bits(a), gi.f32_from_bf16_bits(b), ref_hist,
                                                     ref_st)
        og = io_float(o)
        for n in range(N):
            e = maxrel(og[n], o_ref[n], U_BF16)
            worst_o = max(worst_o, e)
            assert e <= TOL_O_BF16, (s, n, e)
    torch.cuda.synchronize()
    stg = st.cpu().numpy()
    for n in range(N):
        e = maxrel(stg[n], ref_st[n])
        worst_s = max(worst_s, e)
        assert e <= TOL_S_BF16, (n, e)
    assert np.array_equal(io_numpy(conv), gi.bf16_bits_from_f32(ref_hist))
    return worst_o, worst_s


def test_decode_b64_first_steps_all_heads():
    _decode_run(16)


@pytest.mark.slow
def test_decode_b64_1000_steps_all_heads():
    eo, es = _decode_run(1000)
    print(f"decode B=64, 1000 steps, all 48 value heads: worst o max-rel {eo:.2e}, worst state max-rel {es:.2e}")


@pytest.mark.slow
def test_varlen16_chunk_sizes():
    inp = gi.workload_inputs("varlen_16")
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    outs = []
    for C in (16, 64, 128):
        _, o, st, hist = run_gpu_prefill(inp, C)
        eo, es = compare_prefill(inp, o, st, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
        print(f"varlen-16 chunk {C}, all 48 value heads: worst o max-rel {eo:.2e}, worst state max-rel {es:.2e}")
        assert np.array_equal(hist, ref_hist_bits(inp, hist_ref))
        outs.append((o, st, hist))
    for o, st, hist in outs[1:]:  # chunk-size equivalence, all heads
        for n in range(inp.num_seqs):
            sl = slice(inp.cu_seqlens[n], inp.cu_seqlens[n + 1])
            assert maxrel(o[sl], outs[0][0][sl], 2 * U_BF16) <= TOL_O_BF16
            assert maxrel(st[n], outs[0][1][n]) <= TOL_S_BF16
        assert np.array_equal(hist, outs[0][2])


@pytest.mark.slow
def test_long_t65536_split_save_restore_decode():
    w = gi.WORKLOADS["prefill_t65536"]
    inp = gi.workload_inputs("prefill_t65536")
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    # run A: one pass
    _, oA, stA, hA = run_gpu_prefill(inp, 64)
    eo, es = compare_prefill(inp, oA, stA, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    print(f"T=65536 one pass, all 48 value heads: o max-rel {eo:.2e}, state max-rel {es:.2e}")
    assert np.array_equal(hA, ref_hist_bits(inp, hist_ref))
    # run B: prefill [0, 40961), save, restore into fresh buffers, prefill to 65280, decode the last 256
    split, tail = w["split"], w["decode_tail"]
    geo, cfg = inp.geo, gdn.make_config(inp.geo)
    dp = DeviceProblem(inp, 64)
    params = dp.params

    def prefill_range(t0, t1, conv, st):
        o = torch.empty((t1 - t0, geo.value_dim), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(gdn.prefill_workspace_size(cfg, t1 - t0, 1, 64) + 256, dtype=torch.uint8, device="cuda")
        cu_h = np.array([0, t1 - t0], np.int32)
        gdn.prefill(cfg, params, dp.qkv[t0:t1], dp.z[t0:t1], dp.a[t0:t1], dp.b[t0:t1], torch.from_numpy(cu_h).cuda(),
                    cu_h, 64, 0, conv, st, o, ws)
        return o

    conv1, st1 = dp.conv_state.clone(), dp.state.clone()
    o1 = prefill_range(0, split, conv1, st1)
    blob = torch.empty(gdn.state_blob_size(cfg), dtype=torch.uint8, device="cuda")
    gdn.state_save(cfg, conv1, st1, 0, blob)
    conv2 = torch.full_like(conv1, 7.0)
    st2 = torch.full_like(st1, -3.0)
    gdn.state_restore(cfg, blob, 0, conv2, st2)
    assert torch.equal(conv2.view(torch.uint16), conv1.view(torch.uint16)) and torch.equal(st2, st1)
    T = inp.total_tokens
    o2 = prefill_range(split, T - tail, conv2, st2)
    od = torch.empty((tail, geo.value_dim), dtype=torch.bfloat16, device="cuda")
    for t in range(T - tail, T):
        gdn.decode_step(cfg, params, dp.qkv[t:t + 1], dp.z[t:t + 1], dp.a[t:t + 1], dp.b[t:t + 1], 1, conv2, st2,
                        od[t - (T - tail):t - (T - tail) + 1])
    torch.cuda.synchronize()
    oB = np.concatenate([io_float(o1), io_float(o2), io_float(od)])
    stB = st2.cpu().numpy().astype(np.float64)
    eo, es = compare_prefill(inp, oB, stB, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    print(f"T=65536 split/save/restore/decode, all 48 value heads: o max-rel {eo:.2e}, state max-rel {es:.2e}")
    assert maxrel(oB, oA, 2 * U_BF16) <= TOL_O_BF16 and maxrel(stB, stA) <= TOL_S_BF16
    assert np.array_equal(io_numpy(conv2), hA)


# ------------------------------------------------------------------ checkpoint / resume


@pytest.mark.parametrize("where", ["device", "host"])
def test_save_restore_continuation_is_bit_exact(where):
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [40, 40], seed=28, zero_init=False)
    cfg = gdn.make_config(geo)
    dp = DeviceProblem(inp, 64)
    dp.prefill()
    nbytes = gdn.state_blob_size(cfg)
    blob = torch.empty(nbytes, dtype=torch.uint8, device="cuda") if where == "device" else \
        torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    gdn.state_save(cfg, dp.conv_state, dp.state, 1, blob)
    torch.cuda.synchronize()
    conv_live, st_live = dp.conv_state.clone(), dp.state.clone()
    conv_r = torch.zeros_like(conv_live)
    st_r = torch.zeros_like(st_live)
    gdn.state_restore(cfg, blob, 1, conv_r, st_r)
    torch.cuda.synchronize()
    assert torch.equal(conv_r[1].view(torch.uint16), conv_live[1].view(torch.uint16))
    assert torch.equal(st_r[1], st_live[1])
    # continue both by 5 decode steps: identical bytes
    o1 = torch.empty((1, geo.value_dim), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    c_live, s_live = conv_live[1:2].clone(), st_live[1:2].clone()
    c_res, s_res = conv_r[1:2].clone(), st_r[1:2].clone()
    for t in range(5):
        sl = slice(t, t + 1)
        gdn.decode_step(cfg, dp.params, dp.qkv[sl], dp.z[sl], dp.a[sl], dp.b[sl], 1, c_live, s_live, o1)
        gdn.decode_step(cfg, dp.params, dp.qkv[sl], dp.z[sl], dp.a[sl], dp.b[sl], 1, c_res, s_res, o2)
        assert torch.equal(o1.view(torch.uint16), o2.view(torch.uint16))
    assert torch.equal(s_live, s_res) and torch.equal(c_live.view(torch.uint16), c_res.view(torch.uint16))


def test_corrupt_device_blob_rejected_without_writes():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=64, head_v_dim=64)
    inp = gi.make_prefill_inputs(geo, [20], seed=29, zero_init=False)
    cfg = gdn.make_config(geo)
    dp = DeviceProblem(inp, 64)
    blob = torch.empty(gdn.state_blob_size(cfg), dtype=torch.uint8, device="cuda")
    gdn.state_save(cfg, dp.conv_state, dp.state, 0, blob)
    torch.cuda.synchronize()
    target_c = torch.full_like(dp.conv_state, 1.5)
    target_s = torch.full_like(dp.state, 2.5)
    for pos, status in ((1000, "GDN_E_BLOB_CHECKSUM"), (2, "GDN_E_BLOB_FORMAT"), (8, "GDN_E_BLOB_VERSION")):
        bad = blob.clone()
        bad[pos] ^= 1
        with pytest.raises(gdn.GdnError) as e:
            gdn.state_restore(cfg, bad, 0, target_c, target_s)
        assert e.value.name == status
        torch.cuda.synchronize()
        assert bool((target_c.float() == 1.5).all()) and bool((target_s == 2.5).all())
    other = gdn.make_config(gi.Geometry(num_k_heads=1, num_v_heads=4, head_k_dim=64, head_v_dim=64))
    with pytest.raises(gdn.GdnError) as e:
        gdn.state_restore(other, blob, 0, target_c, target_s)
    assert e.value.name in ("GDN_E_BLOB_GEOMETRY", "GDN_E_BLOB_FORMAT")


# ------------------------------------------------------------------ diagnostics


def test_launch_count_and_profiler():
    geo = gi.Geometry(num_k_heads=1, num_v_heads=2, head_k_dim=32, head_v_dim=32)
    inp = gi.make_prefill_inputs(geo, [10, 20], seed=30)
    dp = DeviceProblem(inp, 16)
    gdn.profiler_reset()
    gdn.profiler_enable(True)
    gdn.launch_count_reset()
    dp.prefill()
    dp.prefill()
    torch.cuda.synchronize()
    gdn.profiler_enable(False)
    n = gdn.launch_count()
    assert n >= 4  # per call: schedule (N > 1), mixer kernel, history update
    total = 0
    for k in range(gdn.K.COUNT):
        cnt, ms = gdn.profiler_read(k)
        total += cnt
        assert ms >= 0
    assert total == n
    assert gdn.device_status() == 0


# ------------------------------------------------------------------ chunked tensor-core prefill


@pytest.mark.parametrize("chunk,flags", [(16, 0), (32, 0), (64, 0), (128, 0), (64, AFFINE), (64, FUSED)])
@pytest.mark.parametrize("zero_init", [True, False])
def test_chunked_partial_chunks_match_oracle(zero_init, chunk, flags):
    # lengths around chunk and 64-row tile boundaries: partial first/last chunks, exact multiples, short sequences
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    lengths = [1, 15, 16, 17, 31, 33, 63, 64, 65, 127, 128, 129, 200, 257, 2, 3]
    inp = gi.make_prefill_inputs(geo, lengths, seed=31, zero_init=zero_init)
    o_ref, st_ref, hist_ref = oracle.prefill_inputs(inp)
    _, o, st, hist = run_gpu_prefill(inp, chunk, flags)
    eo, es = compare_prefill(inp, o, st, o_ref, st_ref, TOL_O_BF16, TOL_S_BF16)
    print(f"chunked partial chunks (chunk {chunk}, flags {flags}): o {eo:.2e} state {es:.2e}")
    assert np.array_equal(hist, ref_hist_bits(inp, hist_ref))


@pytest.mark.parametrize("chunk,flags,kernels", [
    (16, 0, "wy"), (32, 0, "wy"), (128, 0, "wy"), (64, AFFINE, "wy"), (64, 0, "split"), (64, FACTORED, "split")])
def test_chunked_paths_run_their_tensor_core_kernels(chunk, flags, kernels):
    """bf16 d=128 runs a three-kernel tensor-core path at every chunk size (the
    affine form at 16, 32, 128, the factored form by default at 64), never the
    token-recurrent kernel, so the chunk-size comparisons compare different
    chunkwise computations."""
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [100, 37], seed=34, zero_init=False)
    dp = DeviceProblem(inp, chunk)
    gdn.profiler_reset()
    gdn.profiler_enable(True)
    dp.prefill(flags)
    torch.cuda.synchronize()
    gdn.profiler_enable(False)
    ran = {k for k in range(gdn.K.COUNT) if gdn.profiler_read(k)[0] > 0}
    want = {gdn.K.WY_CONV, gdn.K.WY_PREP, gdn.K.WY_CHAIN} if kernels == "wy" else \
        {gdn.K.SPLIT_CONV, gdn.K.SPLIT_PREP, gdn.K.SPLIT_CHAIN}
    assert want <= ran
    assert gdn.K.PREFILL_RECURRENT not in ran and gdn.K.PREFILL_CHUNKED not in ran


def test_more_than_one_path_flag_is_rejected():
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [10], seed=35, zero_init=False)
    dp = DeviceProblem(inp, 64)
    with pytest.raises(gdn.GdnError) as e:
        dp.prefill(AFFINE | FUSED)
    assert e.value.name == "GDN_E_INVAL"


@pytest.mark.parametrize("flags", [0, AFFINE, FUSED])
def test_chunked_matches_recurrent_kernel(flags):
    geo = gi.Geometry(num_k_heads=4, num_v_heads=12, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [300, 64, 1, 517], seed=32, zero_init=False)
    _, o1, st1, h1 = run_gpu_prefill(inp, 64, flags)
    _, o2, st2, h2 = run_gpu_prefill(inp, 64, RECURRENT)
    for n in range(inp.num_seqs):
        sl = slice(inp.cu_seqlens[n], inp.cu_seqlens[n + 1])
        assert maxrel(o1[sl], o2[sl], 2 * U_BF16) <= TOL_O_BF16
        assert maxrel(st1[n], st2[n]) <= TOL_S_BF16
    assert np.array_equal(h1, h2)


def test_split_path_workspace_and_fused_workspace():
    """The three-kernel path needs its intermediates; GDN_PREFILL_FUSED runs
    with the schedule alone and rejects nothing that fits it."""
    geo = gi.Geometry(num_k_heads=2, num_v_heads=6, head_k_dim=128, head_v_dim=128)
    inp = gi.make_prefill_inputs(geo, [130, 70], seed=33, zero_init=False)
    dp = DeviceProblem(inp, 64)
    full = gdn.prefill_workspace_size(dp.cfg, inp.total_tokens, inp.num_seqs, 64)
    assert full > 4 * 65664 * geo.num_v_heads  # records of at least four chunks
    small = torch.empty(8192, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill(dp.cfg, dp.params, dp.qkv, dp.z, dp.a, dp.b, dp.cu_dev, dp.cu_host, 64, 0, dp.conv_state,
                    dp.state, dp.o, small)
    assert e.value.name == "GDN_E_WORKSPACE"
    gdn.prefill(dp.cfg, dp.params, dp.qkv, dp.z, dp.a, dp.b, dp.cu_dev, dp.cu_host, 64, FUSED, dp.conv_state,
                dp.state, dp.o, small)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
