"""Multi-token decode (draft-and-verify) through the C ABI.

A verify pass computes the outputs of K draft tokens per sequence and leaves
the caches untouched; a commit applies each sequence's accepted prefix.  Both
must agree bit for bit with K single decode steps (the same kernel arithmetic,
token after token), and the single steps are themselves checked against the
float64 oracle here and in the parity suite.
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


class Round:
    """One draft-and-verify round: N sequences, K draft tokens each."""

    def __init__(self, io, N, K, seed, Hk=2, Hv=6):
        self.geo = geo = gi.Geometry(num_k_heads=Hk, num_v_heads=Hv, io_dtype=io)
        self.N, self.K = N, K
        self.params = gi.make_params(geo, seed)
        self.conv0, self.st0 = gi.make_initial_state(geo, N, seed, zero=False)
        self.toks = [gi.make_decode_step_tokens(geo, N, seed, s) for s in range(K)]  # K x (qkv, z, a, b)
        self.cfg = gdn.make_config(geo)
        self.dparams = tuple(torch.from_numpy(p).cuda() for p in self.params)
        # token-major inside a sequence: [N, K, ...]
        self.multi = [io_tensor(np.ascontiguousarray(np.stack([t[i] for t in self.toks], axis=1)))
                      for i in range(4)]
        self.odt = self.multi[0].dtype

    def caches(self):
        return io_tensor(self.conv0), torch.from_numpy(self.st0).cuda()

    def singles(self):
        """K single decode steps; outputs and cache snapshots after each step."""
        conv, st = self.caches()
        outs, convs, sts = [], [io_numpy(conv)], [st.cpu().numpy()]
        for s in range(self.K):
            o = torch.empty((self.N, self.geo.value_dim), dtype=self.odt, device="cuda")
            qkv, z, a, b = (io_tensor(x) for x in self.toks[s])
            gdn.decode_step(self.cfg, self.dparams, qkv, z, a, b, self.N, conv, st, o)
            outs.append(io_numpy(o))
            convs.append(io_numpy(conv))
            sts.append(st.cpu().numpy())
        return outs, convs, sts

    def run_multi(self, commit, accept=None, conv=None, st=None):
        if conv is None:
            conv, st = self.caches()
        o = torch.full((self.N, self.K, self.geo.value_dim), 7.0, dtype=self.odt, device="cuda")
        acc = None if accept is None else torch.tensor(accept, dtype=torch.int32, device="cuda")
        gdn.decode_multi(self.cfg, self.dparams, *self.multi, self.N, self.K, commit, acc, conv, st, o)
        torch.cuda.synchronize()
        return io_numpy(o), io_numpy(conv), st.cpu().numpy()


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_verify_matches_single_steps_and_leaves_caches(io, K):
    r = Round(io, N=5, K=K, seed=31 + K)
    outs, _, _ = r.singles()
    o, conv, st = r.run_multi(commit=False)
    for t in range(K):
        assert np.array_equal(o[:, t], outs[t]), f"token {t}"
    assert np.array_equal(conv, io_numpy(io_tensor(r.conv0)))
    assert np.array_equal(st, r.st0)


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("K", [2, 4])
def test_commit_accepted_prefix_equals_single_steps(io, K):
    N = 7
    r = Round(io, N=N, K=K, seed=41 + K)
    outs, convs, sts = r.singles()
    accept = [(n * 3 + 1) % (K + 1) for n in range(N)]
    accept[0], accept[1] = 0, K
    raw = list(accept)
    raw[2] = K + 5       # clamped to K
    raw[3] = -2          # clamped to 0
    accept[2], accept[3] = K, 0
    o, conv, st = r.run_multi(commit=True, accept=raw)
    sentinel = io_numpy(torch.full((1,), 7.0, dtype=r.odt))[0]
    for n in range(N):
        a = accept[n]
        assert np.array_equal(conv[n], convs[a][n]), (n, a)
        assert np.array_equal(st[n], sts[a][n]), (n, a)
        for t in range(K):
            if t < a:
                assert np.array_equal(o[n, t], outs[t][n]), (n, t)
            else:
                assert np.all(o[n, t] == sentinel), (n, t)


def test_commit_all_equals_verify_then_commit():
    r = Round("bf16", N=4, K=3, seed=51)
    o_all, conv_all, st_all = r.run_multi(commit=True)
    o_v, conv_v, st_v = r.run_multi(commit=False)
    assert np.array_equal(o_all, o_v)
    conv, st = r.caches()
    o_c, conv_c, st_c = r.run_multi(commit=True, accept=[3, 3, 3, 3], conv=conv, st=st)
    assert np.array_equal(o_c, o_all) and np.array_equal(conv_c, conv_all) and np.array_equal(st_c, st_all)


def test_round_trip_matches_oracle():
    """Verify outputs and a commit of two of three tokens against the oracle."""
    r = Round("bf16", N=3, K=3, seed=61)
    o, _, _ = r.run_multi(commit=False)
    hist = gi.f32_from_bf16_bits(r.conv0)
    st = r.st0.astype(np.float64)
    o_ref = []
    for s in range(3):
        f = [gi.f32_from_bf16_bits(x) for x in r.toks[s]]
        on, st, hist = oracle.decode_step(r.geo, r.params, *f, hist, st)
        o_ref.append(on)
        if s == 1:
            st2, hist2 = st.copy(), hist.copy()
    for n in range(3):
        for t in range(3):
            assert maxrel(gi.f32_from_bf16_bits(o[n, t]), o_ref[t][n], U_BF16) <= TOL_O_BF16, (n, t)
    _, conv, stc = r.run_multi(commit=True, accept=[2, 2, 2])
    for n in range(3):
        assert maxrel(stc[n], st2[n]) <= TOL_S_BF16
    assert np.array_equal(conv, gi.bf16_bits_from_f32(hist2))


def test_f32_round_matches_oracle():
    r = Round("f32", N=2, K=4, seed=71, Hk=1, Hv=3)
    o, conv, st = r.run_multi(commit=True)
    hist = np.asarray(r.conv0, np.float32)
    stf = r.st0.astype(np.float64)
    for s in range(4):
        on, stf, hist = oracle.decode_step(r.geo, r.params, *r.toks[s], hist, stf)
        for n in range(2):
            assert maxrel(o[n, s], on[n], U_F32) <= TOL_F32, (n, s)
    for n in range(2):
        assert maxrel(st[n], stf[n]) <= TOL_F32
    assert np.array_equal(conv, np.asarray(hist, np.float32))


def test_rejects_bad_arguments_without_launch():
    r = Round("bf16", N=2, K=2, seed=81)
    conv, st = r.caches()
    o = torch.empty((2, 2, r.geo.value_dim), dtype=r.odt, device="cuda")
    acc = torch.tensor([1, 1], dtype=torch.int32, device="cuda")
    before = gdn.launch_count()
    for K, commit, a in [(0, True, None), (5, True, None), (2, False, acc)]:
        with pytest.raises(gdn.GdnError) as ei:
            gdn.decode_multi(r.cfg, r.dparams, *r.multi, 2, K, commit, a, conv, st, o)
        assert ei.value.name == "GDN_E_INVAL"
    assert gdn.launch_count() == before
