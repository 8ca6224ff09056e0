"""Pins of the float64 CPU oracle against things other than itself.

Each test checks the oracle against a hand-derived value, a closed form, an
invariant, a library routine or an independent brute-force expansion, chosen
so that a dropped term, a wrong sign or index or a transposed operand in the
oracle fails at least one of them.  No GPU is needed.
"""

import json
import os

import numpy as np
import pytest

import brute
import oracle
from linear_attention_recurrence_deltanet_b200 import inputs as gi

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))


def tiny_geo(Hk=2, Hv=4, d=4, eps=1e-6):
    return gi.Geometry(num_k_heads=Hk, num_v_heads=Hv, head_k_dim=d, head_v_dim=d, l2_eps=eps, norm_eps=eps,
                       io_dtype="f32")


# ---------------------------------------------------------------- gates / norms


@pytest.mark.parametrize("case", GOLD["gates"])
def test_gates_closed_form(case):
    g, al, be = oracle.gates(case["a"], case["dt_bias"], case["A_log"], case["b"])
    if case.get("exact"):
        assert al == case["alpha"] and be == case["beta"] and g == case["g"]
    else:
        assert g == pytest.approx(case["g"], rel=1e-14, abs=1e-15)
        assert al == pytest.approx(case["alpha"], rel=1e-14)
        assert be == pytest.approx(case["beta"], rel=1e-14)


def test_gates_match_library_softplus_and_sigmoid():
    rng = np.random.default_rng(7)
    for _ in range(200):
        a, dtb, Al, b = rng.normal(size=4) * np.array([3, 2, 1.5, 4])
        g, al, be = oracle.gates(a, dtb, Al, b)
        g2, al2, be2 = brute.gates(a, dtb, Al, b)
        assert g == pytest.approx(g2, rel=1e-13, abs=1e-300)
        assert al == pytest.approx(al2, rel=1e-13)
        assert be == pytest.approx(be2, rel=1e-13)
        assert al <= 1.0 and g <= 0.0  # decay never amplifies


@pytest.mark.parametrize("case", GOLD["l2norm"])
def test_l2norm_closed_form(case):
    out = oracle.l2norm(case["x"], case["eps"])
    np.testing.assert_allclose(out, case["out"], rtol=1e-14)


def test_l2norm_norm_identity():
    # |x_hat|^2 = s / (s + eps) with s = sum x^2: the epsilon sits inside the sqrt of the sum.
    rng = np.random.default_rng(1)
    for scale in (1e-4, 1e-3, 1.0, 30.0):
        x = rng.normal(size=128) * scale
        s = float(np.sum(x * x))
        out = oracle.l2norm(x, 1e-6)
        assert float(np.sum(out * out)) == pytest.approx(s / (s + 1e-6), rel=1e-13)
        np.testing.assert_allclose(oracle.l2norm(x, 1e-6, scale=0.25), 0.25 * out, rtol=1e-15)


@pytest.mark.parametrize("case", GOLD["output"])
def test_output_closed_form(case):
    out = oracle.output_norm_gate(case["o"], case["z"], case["w"], case["eps"])
    np.testing.assert_allclose(out, case["out"], rtol=1e-14, atol=1e-15)


def test_output_reduces_to_textbook_rmsnorm():
    rng = np.random.default_rng(2)
    o = rng.normal(size=64) * 3
    # w = 0 and a saturated gate (z = 50, sigmoid = 1 to 1e-21): plain RMSNorm
    out = oracle.output_norm_gate(o, np.full(64, 50.0), np.zeros(64), 1e-6)
    np.testing.assert_allclose(out, o / np.sqrt(np.mean(o * o) + 1e-6), rtol=1e-14)
    # gate and weight act per element
    z, w = rng.normal(size=64), rng.normal(size=64) * 0.3
    out2 = oracle.output_norm_gate(o, z, w, 1e-6)
    np.testing.assert_allclose(out2, brute.rmsnorm_gate(o, z, w, 1e-6), rtol=1e-13)


# ---------------------------------------------------------------- delta rule


@pytest.mark.parametrize("case", GOLD["delta_step"])
def test_delta_step_hand_values(case):
    S, o = oracle.delta_step(np.array(case["S0"]), case["k"], case["v"], case["q"], case["alpha"], case["beta"])
    np.testing.assert_allclose(S, case["S1"], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(o, case["o"], rtol=1e-14, atol=1e-15)


def test_delta_step_single_token_closed_form():
    # S1 = alpha (I - beta k k^T) S0 + beta k v^T ; o = S1^T q
    rng = np.random.default_rng(3)
    for dk, dv in ((4, 4), (8, 3), (32, 32)):
        S0 = rng.normal(size=(dk, dv))
        k = brute.l2n(rng.normal(size=dk), 1e-6)
        q = brute.l2n(rng.normal(size=dk), 1e-6)
        v = rng.normal(size=dv)
        alpha, beta = 0.7, 0.35
        S1, o = oracle.delta_step(S0, k, v, q, alpha, beta)
        S1_ref = alpha * (np.eye(dk) - beta * np.outer(k, k)) @ S0 + beta * np.outer(k, v)
        np.testing.assert_allclose(S1, S1_ref, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(o, S1_ref.T @ q, rtol=1e-13, atol=1e-14)


def test_delta_step_identity_when_alpha1_beta0():
    rng = np.random.default_rng(4)
    S0 = rng.normal(size=(16, 16))
    S1, _ = oracle.delta_step(S0, rng.normal(size=16), rng.normal(size=16), rng.normal(size=16), 1.0, 0.0)
    assert np.array_equal(S1, S0)  # bit-exact


def test_retrieval_beta1_q_equals_k():
    # beta = 1, q = k: S1^T k = alpha (1 - |k|^2) S0^T k + |k|^2 v
    rng = np.random.default_rng(5)
    S0 = rng.normal(size=(8, 6))
    k = brute.l2n(rng.normal(size=8), 1e-6)
    v = rng.normal(size=6)
    S1, o = oracle.delta_step(S0, k, v, k, 0.8, 1.0)
    kk = float(k @ k)
    np.testing.assert_allclose(o, 0.8 * (1 - kk) * (S0.T @ k) + kk * v, rtol=1e-12, atol=1e-13)


def test_superposition_in_state_and_values():
    # o(S0, V) = o(S0, 0) + o(0, V) at fixed q, k, g, beta (before the output norm)
    rng = np.random.default_rng(6)
    dk, dv, L = 6, 5, 7
    S0 = rng.normal(size=(dk, dv))
    ks = [brute.l2n(x, 1e-6) for x in rng.normal(size=(L, dk))]
    qs = [brute.l2n(x, 1e-6) for x in rng.normal(size=(L, dk))]
    vs = rng.normal(size=(L, dv))
    al, be = rng.uniform(0.3, 1.0, L), rng.uniform(0.0, 1.0, L)

    def run(S, V):
        out = []
        for t in range(L):
            S, o = oracle.delta_step(S, ks[t], V[t], qs[t], al[t], be[t])
            out.append(o)
        return np.array(out), S

    o_full, S_full = run(S0, vs)
    o_s, S_s = run(S0, np.zeros_like(vs))
    o_v, S_v = run(np.zeros_like(S0), vs)
    np.testing.assert_allclose(o_full, o_s + o_v, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S_full, S_s + S_v, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- conv


def test_conv_tap_impulse_shifts_input():
    rng = np.random.default_rng(8)
    C, W, L = 6, 4, 9
    x = rng.normal(size=(L, C)).astype(np.float32)
    hist = rng.normal(size=(1, W - 1, C)).astype(np.float32)
    full = np.concatenate([hist[0], x], 0).astype(np.float64)
    for j in range(W):
        w = np.zeros((C, W), np.float32)
        w[:, j] = 1.0
        y, _ = oracle.conv_prefill(x, w, [0, L], hist)
        shifted = full[j:j + L]  # tap j reads position p + j - (W-1) of the sequence
        np.testing.assert_allclose(y, shifted / (1 + np.exp(-shifted)), rtol=1e-15)


def test_conv_matches_np_convolve_and_history_is_raw_copy():
    rng = np.random.default_rng(9)
    C, W = 5, 4
    lengths = [7, 1, 2, 0, 3, 5]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    x = rng.normal(size=(cu[-1], C)).astype(np.float32)
    w = rng.normal(size=(C, W)).astype(np.float32) * 0.5
    hist = rng.normal(size=(len(lengths), W - 1, C)).astype(np.float32)
    y, hout = oracle.conv_prefill(x, w, cu, hist)
    for n, L in enumerate(lengths):
        if L:
            np.testing.assert_allclose(y[cu[n]:cu[n + 1]], brute.conv_silu(x[cu[n]:cu[n + 1]], hist[n], w), rtol=1e-13)
        full = np.concatenate([hist[n], x[cu[n]:cu[n + 1]]], 0)
        assert np.array_equal(hout[n], full[-(W - 1):])  # byte copy of the last W-1 raw inputs


# ---------------------------------------------------------------- whole mixer


def _tiny_problem(lengths, seed, zero_init=False, Hk=2, Hv=4, d=4):
    geo = tiny_geo(Hk, Hv, d)
    return gi.make_prefill_inputs(geo, lengths, seed, zero_init=zero_init)


def _params(inp):
    return (inp.conv_w, inp.A_log, inp.dt_bias, inp.norm_w)


@pytest.mark.parametrize("lengths,Hk,Hv,d", [([5], 2, 4, 4), ([3, 1, 6, 0, 2], 1, 3, 4), ([8], 2, 2, 8),
                                                ([4, 4], 2, 6, 3)])
def test_prefill_matches_outer_product_expansion(lengths, Hk, Hv, d):
    inp = _tiny_problem(lengths, seed=11, Hk=Hk, Hv=Hv, d=d)
    o, st, _ = oracle.prefill_inputs(inp)
    o_b, st_b = brute.prefill(inp.geo, _params(inp), inp.qkv, inp.z, inp.a, inp.b, inp.cu_seqlens, inp.conv_state,
                              inp.state)
    np.testing.assert_allclose(o, o_b, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(st, st_b, rtol=1e-11, atol=1e-12)


def test_beta_zero_only_decays_state():
    inp = _tiny_problem([6], seed=12)
    inp.b[:] = -1e4  # beta = 0 exactly
    o, st, _ = oracle.prefill_inputs(inp)
    for h in range(inp.geo.num_v_heads):
        g = np.array([oracle.gates(inp.a[t, h], inp.dt_bias[h], inp.A_log[h], inp.b[t, h])[0] for t in range(6)])
        np.testing.assert_allclose(st[0, h], np.exp(g.sum()) * inp.state[0, h], rtol=1e-13)


def test_alpha1_beta0_prefill_leaves_state_bit_exact():
    inp = _tiny_problem([7], seed=13)
    inp.a[:] = -1e4
    inp.b[:] = -1e4
    _, st, _ = oracle.prefill_inputs(inp)
    assert np.array_equal(st, inp.state.astype(np.float64))


def test_varlen_packing_equals_separate_runs():
    lengths = [5, 0, 1, 9, 2]
    inp = _tiny_problem(lengths, seed=14)
    o, st, hist = oracle.prefill_inputs(inp)
    cu = inp.cu_seqlens
    for n in range(len(lengths)):
        sl = slice(cu[n], cu[n + 1])
        o1, st1, h1 = oracle.prefill(inp.geo, _params(inp), inp.qkv[sl], inp.z[sl], inp.a[sl], inp.b[sl],
                                     [0, lengths[n]], inp.conv_state[n:n + 1], inp.state[n:n + 1])
        assert np.array_equal(o[sl], o1)
        assert np.array_equal(st[n], st1[0])
        assert np.array_equal(hist[n], h1[0])


def test_prefill_equals_decode_steps_and_split_resume():
    inp = _tiny_problem([11], seed=15)
    o, st, hist = oracle.prefill_inputs(inp)
    # token-by-token decode
    S, H = inp.state.astype(np.float64), inp.conv_state
    for t in range(11):
        sl = slice(t, t + 1)
        ot, S, H = oracle.decode_step(inp.geo, _params(inp), inp.qkv[sl], inp.z[sl], inp.a[sl], inp.b[sl], H, S)
        assert np.array_equal(ot, o[sl])
    assert np.array_equal(S, st) and np.array_equal(H, hist)
    # split at 4 and resume from the saved state and history
    o1, S1, H1 = oracle.prefill(inp.geo, _params(inp), inp.qkv[:4], inp.z[:4], inp.a[:4], inp.b[:4], [0, 4],
                                inp.conv_state, inp.state)
    o2, S2, H2 = oracle.prefill(inp.geo, _params(inp), inp.qkv[4:], inp.z[4:], inp.a[4:], inp.b[4:], [0, 7], H1, S1)
    assert np.array_equal(np.concatenate([o1, o2]), o) and np.array_equal(S2, st) and np.array_equal(H2, hist)


def test_key_head_sharing_groups_are_contiguous():
    # value heads G*kh .. G*kh+G-1 read key head kh: perturbing key head 1's q/k
    # channels changes value heads 2,3 (G=2) and leaves heads 0,1 bit-identical.
    inp = _tiny_problem([6], seed=16)
    o, st, _ = oracle.prefill_inputs(inp)
    d = inp.geo.head_k_dim
    inp.qkv[:, d:2 * d] += 0.5  # q of key head 1
    o2, st2, _ = oracle.prefill_inputs(inp)
    dv = inp.geo.head_v_dim
    assert np.array_equal(o[:, :2 * dv], o2[:, :2 * dv])
    assert not np.allclose(o[:, 2 * dv:], o2[:, 2 * dv:])


def test_head_mask_samples_heads():
    inp = _tiny_problem([9, 3], seed=17)
    o, st, _ = oracle.prefill_inputs(inp)
    o2, st2, _ = oracle.prefill_inputs(inp, heads=[1, 3])
    dv = inp.geo.head_v_dim
    for h in (1, 3):
        assert np.array_equal(o[:, h * dv:(h + 1) * dv], o2[:, h * dv:(h + 1) * dv])
        assert np.array_equal(st[:, h], st2[:, h])


@pytest.mark.parametrize("C", [1, 3, 4, 16])
def test_chunked_form_equals_oracle(C):
    # the chunkwise WY/UT algebra the GPU prefill uses reproduces the oracle
    inp = _tiny_problem([13], seed=18, d=6)
    o_ref, st_ref, _ = oracle.prefill_inputs(inp)
    geo = inp.geo
    dv = geo.head_v_dim
    for h in range(geo.num_v_heads):
        qh, kh, v = brute.head_inputs(geo, _params(inp), inp.qkv.astype(np.float64), inp.conv_state[0], h)
        g, _, beta = brute.gates(inp.a[:, h].astype(np.float64), inp.dt_bias[h], inp.A_log[h],
                                 inp.b[:, h].astype(np.float64))
        o_pre, S = brute.chunked_head(inp.state[0, h].T.astype(np.float64), qh, kh, v, g, beta, C)
        o = np.stack([brute.rmsnorm_gate(o_pre[t], inp.z[t, h * dv:(h + 1) * dv], inp.norm_w, geo.norm_eps)
                      for t in range(13)])
        np.testing.assert_allclose(o, o_ref[:, h * dv:(h + 1) * dv], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S.T, st_ref[0, h], rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("C,base", [(4, 2), (16, 4), (13, 4), (32, 16)])
def test_affine_form_equals_oracle(C, base):
    # the affine chunk maps (M' = -K~^T W, Q' = e^gamma Q - P W) with T by recursive doubling, as the
    # affine GPU prefill computes them, reproduce the oracle
    inp = _tiny_problem([37], seed=19, d=6)
    o_ref, st_ref, _ = oracle.prefill_inputs(inp)
    geo = inp.geo
    dv = geo.head_v_dim
    for h in range(geo.num_v_heads):
        qh, kh, v = brute.head_inputs(geo, _params(inp), inp.qkv.astype(np.float64), inp.conv_state[0], h)
        g, _, beta = brute.gates(inp.a[:, h].astype(np.float64), inp.dt_bias[h], inp.A_log[h],
                                 inp.b[:, h].astype(np.float64))
        o_pre, S = brute.affine_head(inp.state[0, h].T.astype(np.float64), qh, kh, v, g, beta, C, base)
        o = np.stack([brute.rmsnorm_gate(o_pre[t], inp.z[t, h * dv:(h + 1) * dv], inp.norm_w, geo.norm_eps)
                      for t in range(37)])
        np.testing.assert_allclose(o, o_ref[:, h * dv:(h + 1) * dv], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S.T, st_ref[0, h], rtol=1e-11, atol=1e-12)


def test_doubling_inverse_is_the_inverse():
    rng = np.random.default_rng(7)
    for n, base in ((16, 4), (23, 4), (64, 16), (128, 16)):
        A = np.tril(rng.normal(0, 0.3, (n, n)), -1)
        T = brute.doubling_inverse(A, base)
        np.testing.assert_allclose(T @ (np.eye(n) + A), np.eye(n), atol=1e-10)
        assert np.array_equal(np.triu(T, 1), np.zeros((n, n)))  # lower triangular, like (I + A)^-1


def test_workload_tiny_fp32_runs_and_is_finite():
    inp = gi.workload_inputs("tiny_fp32_t64")
    o, st, hist = oracle.prefill_inputs(inp)
    assert o.shape == (64, 128) and np.isfinite(o).all() and np.isfinite(st).all()
    assert np.array_equal(hist[0], inp.qkv[-3:])
