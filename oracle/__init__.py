"""CPU oracle for the Gated DeltaNet token mixer (float64, token by token).

TEST INFRASTRUCTURE ONLY: tests/, the smoke check and the benchmark's CPU
baseline may import this package; the CUDA library and its Python binding
never do.  The arithmetic lives in ``gdn_oracle.cpp`` (compiled here with the
host C++ compiler into ``libgdn_oracle.so``); this module marshals numpy
arrays and nothing else.  It shares no code with the CUDA path: inputs come
from ``linear_attention_recurrence_deltanet_b200.inputs``, which only draws
numbers.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.cpp")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None


class Geometry(ctypes.Structure):
    _fields_ = [
        ("num_k_heads", ctypes.c_int32),
        ("num_v_heads", ctypes.c_int32),
        ("head_k_dim", ctypes.c_int32),
        ("head_v_dim", ctypes.c_int32),
        ("conv_width", ctypes.c_int32),
        ("l2_eps", ctypes.c_double),
        ("norm_eps", ctypes.c_double),
        ("q_scale", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain -O2, IEEE arithmetic, no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        L.gdn_ref_gates.argtypes = [ctypes.c_double] * 4 + [P, P, P]
        L.gdn_ref_l2norm.argtypes = [P, ctypes.c_int32, ctypes.c_double, ctypes.c_double, P]
        L.gdn_ref_output.argtypes = [P, P, P, ctypes.c_int32, ctypes.c_double, P]
        L.gdn_ref_delta_step.argtypes = [P, P, P, P, ctypes.c_double, ctypes.c_double, ctypes.c_int32,
                                         ctypes.c_int32, P]
        L.gdn_ref_conv_prefill.argtypes = [ctypes.c_int64, ctypes.c_int32, P, P, P, ctypes.c_int32, P, P, P]
        L.gdn_ref_conv_prefill.restype = ctypes.c_int32
        L.gdn_ref_prefill.argtypes = [P] + [P] * 8 + [P, ctypes.c_int32, P, P, P, P, P, ctypes.c_int32]
        L.gdn_ref_prefill.restype = ctypes.c_int32
        L.gdn_ref_decode_step.argtypes = [P] + [P] * 8 + [ctypes.c_int32, P, P, P, P, P, ctypes.c_int32]
        L.gdn_ref_decode_step.restype = ctypes.c_int32
        L.gdn_ref_project.argtypes = [P, ctypes.c_int64, P, ctypes.c_int64, P, ctypes.c_int64, P, ctypes.c_int32]
        L.gdn_ref_project.restype = None
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def default_threads() -> int:
    return os.cpu_count() or 1


def gates(a: float, dt_bias: float, A_log: float, b: float):
    """(g, alpha, beta) of one token and value head."""
    g, al, be = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    lib().gdn_ref_gates(a, dt_bias, A_log, b, ctypes.byref(g), ctypes.byref(al), ctypes.byref(be))
    return g.value, al.value, be.value


def l2norm(x, eps: float, scale: float = 1.0) -> np.ndarray:
    x = _f64(x)
    out = np.empty_like(x)
    lib().gdn_ref_l2norm(_ptr(x), x.size, eps, scale, _ptr(out))
    return out


def output_norm_gate(o, z, w, eps: float) -> np.ndarray:
    o, z, w = _f64(o), _f64(z), _f64(w)
    out = np.empty_like(o)
    lib().gdn_ref_output(_ptr(o), _ptr(z), _ptr(w), o.size, eps, _ptr(out))
    return out


def delta_step(S, k, v, q, alpha: float, beta: float):
    """One gated delta-rule step on a [dk, dv] state; returns (S_new, o)."""
    S = _f64(S).copy()
    k, v, q = _f64(k), _f64(v), _f64(q)
    o = np.empty(S.shape[1], np.float64)
    lib().gdn_ref_delta_step(_ptr(S), _ptr(k), _ptr(v), _ptr(q), alpha, beta, S.shape[0], S.shape[1], _ptr(o))
    return S, o


def conv_prefill(x, conv_w, cu_seqlens, hist):
    """SiLU(causal depthwise conv) of every channel; returns (y float64, new history float32)."""
    x, conv_w, hist = _f32(x), _f32(conv_w), _f32(hist)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    C, W = conv_w.shape
    y = np.zeros((x.shape[0], C), np.float64)
    hout = np.empty_like(hist)
    lib().gdn_ref_conv_prefill(C, W, _ptr(conv_w), _ptr(x), _ptr(cu), cu.size - 1, _ptr(hist), _ptr(y), _ptr(hout))
    return y, hout


def _geometry(geo) -> Geometry:
    return Geometry(geo.num_k_heads, geo.num_v_heads, geo.head_k_dim, geo.head_v_dim, geo.conv_width,
                    geo.l2_eps, geo.norm_eps, geo.q_scale)


def prefill(geo, params, qkv, z, a, b, cu_seqlens, hist, state, heads=None, threads: Optional[int] = None):
    """Prefill over packed sequences.

    params = (conv_w, A_log, dt_bias, norm_w); qkv/z/a/b are float arrays of
    the stored values; hist [N, W-1, C] and state [N, Hv, dv, dk] are the
    starting conv history and recurrent state.  ``heads`` optionally lists the
    value heads to compute (others: outputs NaN, state unchanged).
    Returns (o float64 [T, Hv*dv], state float64, new history float32).
    """
    conv_w, A_log, dt_bias, norm_w = (_f32(p) for p in params)
    qkv, z, a, b, hist = _f32(qkv), _f32(z), _f32(a), _f32(b), _f32(hist)
    st = _f64(state).copy()
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    o = np.full((T, geo.num_v_heads * geo.head_v_dim), np.nan, np.float64)
    hout = np.empty_like(hist)
    mask = None
    if heads is not None:
        mask = np.zeros(geo.num_v_heads, np.uint8)
        mask[list(heads)] = 1
    g = _geometry(geo)
    rc = lib().gdn_ref_prefill(ctypes.byref(g), _ptr(conv_w), _ptr(A_log), _ptr(dt_bias), _ptr(norm_w), _ptr(qkv),
                               _ptr(z), _ptr(a), _ptr(b), _ptr(cu), cu.size - 1, _ptr(mask), _ptr(hist), _ptr(st),
                               _ptr(o), _ptr(hout), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the geometry")
    return o, st, hout


def decode_step(geo, params, qkv, z, a, b, hist, state, heads=None, threads: Optional[int] = None):
    """One decode step (one token per sequence).  Same conventions as prefill."""
    conv_w, A_log, dt_bias, norm_w = (_f32(p) for p in params)
    qkv, z, a, b, hist = _f32(qkv), _f32(z), _f32(a), _f32(b), _f32(hist)
    st = _f64(state).copy()
    N = qkv.shape[0]
    o = np.full((N, geo.num_v_heads * geo.head_v_dim), np.nan, np.float64)
    hout = np.empty_like(hist)
    mask = None
    if heads is not None:
        mask = np.zeros(geo.num_v_heads, np.uint8)
        mask[list(heads)] = 1
    g = _geometry(geo)
    rc = lib().gdn_ref_decode_step(ctypes.byref(g), _ptr(conv_w), _ptr(A_log), _ptr(dt_bias), _ptr(norm_w),
                                   _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), N, _ptr(mask), _ptr(hist), _ptr(st),
                                   _ptr(o), _ptr(hout), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle rejected the geometry")
    return o, st, hout


def prefill_inputs(inp, heads=None, threads=None):
    """Run the oracle on a ``GdnInputs`` problem (from the inputs module)."""
    params = (inp.conv_w, inp.A_log, inp.dt_bias, inp.norm_w)
    return prefill(inp.geo, params, inp.f32("qkv"), inp.f32("z"), inp.f32("a"), inp.f32("b"), inp.cu_seqlens,
                   inp.f32("conv_state"), inp.state, heads=heads, threads=threads)


def project(x, w, rows=None, threads: Optional[int] = None) -> np.ndarray:
    """Linear layer y = x w^T in float64 for the listed rows of x (all rows by
    default).  x [M, K] and w [N, K] are float arrays holding the exact values
    of their stored dtype; returns float64 [len(rows), N]."""
    x, w = _f32(x), _f32(w)
    rows = np.arange(x.shape[0], dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    assert x.shape[1] == w.shape[1] and (rows.size == 0 or (rows.min() >= 0 and rows.max() < x.shape[0]))
    y = np.empty((rows.size, w.shape[0]), np.float64)
    lib().gdn_ref_project(_ptr(x), x.shape[1], _ptr(w), w.shape[0], _ptr(rows), rows.size, _ptr(y),
                          threads or default_threads())
    return y


def split_projection(geo, y):
    """Columns of the input projection's output, in the stacking order of its
    weight rows: (qkv [., C_conv], z [., Hv*d_v], a [., Hv], b [., Hv])."""
    C = 2 * geo.num_k_heads * geo.head_k_dim + geo.num_v_heads * geo.head_v_dim
    V = geo.num_v_heads * geo.head_v_dim
    H = geo.num_v_heads
    assert y.shape[1] == C + V + 2 * H
    return y[:, :C], y[:, C:C + V], y[:, C + V:C + V + H], y[:, C + V + H:]
