"""Pins of the algebra the sequence-parallel prefill rests on, checked with
the float64 oracle's own delta-rule step (no CUDA code involved).

Over a run of tokens the gated delta rule is affine in the state it starts
from: S_L = A S_0 + B, where A (d_k x d_k) depends only on keys and gates and
B is the run's final state from S_0 = 0.  With d_k = d_v, A is the final
state of the same run started from S_0 = I with every value set to zero.
In the stored (transposed) layout the composition is T_L = T_0 A^T + B^T.
"""

import numpy as np
import pytest

import oracle


def run(S0, ks, vs, qs, alphas, betas):
    S = np.array(S0, dtype=np.float64)
    for k, v, q, al, be in zip(ks, vs, qs, alphas, betas):
        S, _ = oracle.delta_step(S, k, v, q, al, be)
    return S


def tokens(rng, n, d):
    ks = rng.standard_normal((n, d))
    ks /= np.linalg.norm(ks, axis=1, keepdims=True)
    qs = rng.standard_normal((n, d))
    vs = rng.standard_normal((n, d))
    alphas = rng.uniform(0.5, 1.0, n)
    betas = rng.uniform(0.0, 1.0, n)
    return ks, vs, qs, alphas, betas


@pytest.mark.parametrize("n,d", [(1, 4), (7, 8), (33, 16)])
def test_segment_is_affine_in_its_starting_state(n, d):
    rng = np.random.default_rng(100 + n)
    ks, vs, qs, alphas, betas = tokens(rng, n, d)
    S0 = rng.standard_normal((d, d))
    A = run(np.eye(d), ks, np.zeros_like(vs), qs, alphas, betas)
    B = run(np.zeros((d, d)), ks, vs, qs, alphas, betas)
    direct = run(S0, ks, vs, qs, alphas, betas)
    assert np.allclose(direct, A @ S0 + B, rtol=0, atol=1e-12 * max(1.0, np.abs(direct).max()))
    # stored layout: T = S^T, T_L = T_0 A^T + B^T
    assert np.allclose(direct.T, S0.T @ A.T + B.T, rtol=0, atol=1e-12 * max(1.0, np.abs(direct).max()))
    # A acts on the key index: it is the product of the tokens' alpha (I - beta k k^T), last token leftmost
    P = np.eye(d)
    for k, al, be in zip(ks, alphas, betas):
        P = al * (np.eye(d) - be * np.outer(k, k)) @ P
    assert np.allclose(A, P, rtol=0, atol=1e-12)


def test_segments_compose_in_order():
    """Three segments walked as S_{j+1} = A_j S_j + B_j equal one run."""
    rng = np.random.default_rng(7)
    d, lens = 8, [5, 9, 4]
    ks, vs, qs, alphas, betas = tokens(rng, sum(lens), d)
    S0 = rng.standard_normal((d, d))
    S, t = S0.copy(), 0
    for L in lens:
        sl = slice(t, t + L)
        A = run(np.eye(d), ks[sl], np.zeros_like(vs[sl]), qs[sl], alphas[sl], betas[sl])
        B = run(np.zeros((d, d)), ks[sl], vs[sl], qs[sl], alphas[sl], betas[sl])
        S = A @ S + B
        t += L
    assert np.allclose(S, run(S0, ks, vs, qs, alphas, betas), rtol=0, atol=1e-11)
