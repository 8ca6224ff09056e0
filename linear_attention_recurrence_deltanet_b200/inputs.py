"""Seeded synthetic inputs for the Gated DeltaNet (GDN) token mixer.

This module only draws numbers.  It holds none of the mixer's arithmetic and
is shared by the tests, the benchmark and the CPU oracle's callers, so that
the CUDA path and the oracle always see exactly the same inputs.

The workloads follow the shapes the reference pages give for Qwen3.8's GDN
layers ("16-key/48-value-head GDN geometry, convolution width 4, fp32
recurrent state": DS4Server issue #95, "Implement the Qwen3.8 Flash Next Rust
and Metal text core", section Implementation; "BF16 width-4 convolution
history": the implementation comment on the same page).  Head dimension 128
and the value distributions are this library's stated workload recipe.

Distributions (N(mu, var) takes the variance):
  pre-conv q/k/v channels x ~ N(0, 1); conv weights ~ N(0, 1/4);
  a, b, z ~ N(0, 1); A_log = log U[1, 16]; dt_bias = log(expm1(U[1e-3, 0.1]));
  norm offset w ~ N(0, 0.1) (applied as 1 + w);
  initial recurrent state ~ N(0, 0.02) and initial conv history ~ N(0, 1)
  where a workload asks for a non-zero start.
Draws are float32 from numpy's PCG64; bf16 tensors are the round-to-nearest-
even bf16 encodings of those draws, and every consumer uses the rounded value.

Streams: parameters come from ``default_rng([seed, 0])``, initial states from
``default_rng([seed, 1])`` and token inputs from ``default_rng([seed, 2])``
(drawn tensor by tensor: qkv, z, a, b).  Decode step ``s`` draws its token
inputs from ``default_rng([seed, 1000 + s])`` so any step can be regenerated
alone.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "Geometry",
    "GdnInputs",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
    "make_params",
    "make_initial_state",
    "make_tokens",
    "make_prefill_inputs",
    "make_decode_step_tokens",
    "varlen_lengths",
    "QWEN_HIDDEN",
    "make_projection_weights",
    "make_hidden_states",
    "WORKLOADS",
]


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def f32_from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    """Exact float32 value of bf16 bit patterns."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Geometry:
    """Head geometry and numerics of one GDN mixer layer."""

    num_k_heads: int = 16
    num_v_heads: int = 48
    head_k_dim: int = 128
    head_v_dim: int = 128
    conv_width: int = 4
    l2_eps: float = 1e-6
    norm_eps: float = 1e-6
    q_scale: float = 1.0
    io_dtype: str = "bf16"  # "bf16" or "f32"

    @property
    def group(self) -> int:
        return self.num_v_heads // self.num_k_heads

    @property
    def key_dim(self) -> int:
        return self.num_k_heads * self.head_k_dim

    @property
    def value_dim(self) -> int:
        return self.num_v_heads * self.head_v_dim

    @property
    def conv_dim(self) -> int:
        return 2 * self.key_dim + self.value_dim

    @property
    def io_bytes(self) -> int:
        return 2 if self.io_dtype == "bf16" else 4


def _io(values: np.ndarray, geo: Geometry) -> np.ndarray:
    """Store float32 draws in the io dtype: uint16 bf16 bits, or float32."""
    if geo.io_dtype == "bf16":
        return bf16_bits_from_f32(values)
    return np.ascontiguousarray(values, dtype=np.float32)


@dataclasses.dataclass
class GdnInputs:
    """One prefill (or decode) problem.  io tensors are stored in the io dtype
    (uint16 bf16 bits or float32); parameters and the recurrent state are
    float32."""

    geo: Geometry
    cu_seqlens: np.ndarray  # int32 [N+1]
    qkv: np.ndarray  # [T, conv_dim]
    z: np.ndarray  # [T, Hv*dv]
    a: np.ndarray  # [T, Hv]
    b: np.ndarray  # [T, Hv]
    conv_w: np.ndarray  # f32 [conv_dim, W]
    A_log: np.ndarray  # f32 [Hv]
    dt_bias: np.ndarray  # f32 [Hv]
    norm_w: np.ndarray  # f32 [dv]
    conv_state: np.ndarray  # io dtype [N, W-1, conv_dim]
    state: np.ndarray  # f32 [N, Hv, dv, dk]
    zero_init: bool = True

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    def f32(self, name: str) -> np.ndarray:
        """float32 values of an io-dtype tensor (exact)."""
        arr = getattr(self, name)
        if arr.dtype == np.uint16:
            return f32_from_bf16_bits(arr)
        return arr


def make_params(geo: Geometry, seed: int):
    rng = np.random.default_rng([seed, 0])
    conv_w = rng.normal(0.0, 0.5, size=(geo.conv_dim, geo.conv_width)).astype(np.float32)
    A_log = np.log(rng.uniform(1.0, 16.0, size=geo.num_v_heads)).astype(np.float32)
    dt = rng.uniform(1e-3, 0.1, size=geo.num_v_heads)
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    norm_w = rng.normal(0.0, np.sqrt(0.1), size=geo.head_v_dim).astype(np.float32)
    return conv_w, A_log, dt_bias, norm_w


def make_initial_state(geo: Geometry, num_seqs: int, seed: int, zero: bool):
    shape_c = (num_seqs, geo.conv_width - 1, geo.conv_dim)
    shape_s = (num_seqs, geo.num_v_heads, geo.head_v_dim, geo.head_k_dim)
    if zero:
        return _io(np.zeros(shape_c, np.float32), geo), np.zeros(shape_s, np.float32)
    rng = np.random.default_rng([seed, 1])
    conv = rng.standard_normal(size=shape_c, dtype=np.float32)
    state = (rng.standard_normal(size=shape_s, dtype=np.float32) * np.float32(np.sqrt(0.02))).astype(np.float32)
    return _io(conv, geo), state


def make_tokens(geo: Geometry, rng: np.random.Generator, num_tokens: int):
    qkv = rng.standard_normal(size=(num_tokens, geo.conv_dim), dtype=np.float32)
    z = rng.standard_normal(size=(num_tokens, geo.value_dim), dtype=np.float32)
    a = rng.standard_normal(size=(num_tokens, geo.num_v_heads), dtype=np.float32)
    b = rng.standard_normal(size=(num_tokens, geo.num_v_heads), dtype=np.float32)
    return _io(qkv, geo), _io(z, geo), _io(a, geo), _io(b, geo)


def make_prefill_inputs(geo: Geometry, lengths, seed: int, zero_init: bool = True) -> GdnInputs:
    lengths = [int(x) for x in lengths]
    cu = np.zeros(len(lengths) + 1, np.int32)
    cu[1:] = np.cumsum(lengths)
    conv_w, A_log, dt_bias, norm_w = make_params(geo, seed)
    conv_state, state = make_initial_state(geo, len(lengths), seed, zero_init)
    qkv, z, a, b = make_tokens(geo, np.random.default_rng([seed, 2]), int(cu[-1]))
    return GdnInputs(geo, cu, qkv, z, a, b, conv_w, A_log, dt_bias, norm_w, conv_state, state, zero_init)


def make_decode_step_tokens(geo: Geometry, num_seqs: int, seed: int, step: int):
    """Token inputs (qkv, z, a, b) of decode step ``step`` for ``num_seqs`` sequences."""
    return make_tokens(geo, np.random.default_rng([seed, 1000 + step]), num_seqs)


def varlen_lengths(seed: int = 4, num_seqs: int = 16, max_len: int = 8192) -> np.ndarray:
    """Sequence lengths drawn uniformly from 1..max_len."""
    return np.random.default_rng(seed).integers(1, max_len + 1, num_seqs)


# hidden size of the Qwen3.8-27B configuration (DS4Server issue #89, Model and reference contract)
QWEN_HIDDEN = 5120


def make_projection_weights(geo: Geometry, hidden: int, seed: int):
    """bf16 bits of a layer's two projection weights, drawn from
    ``default_rng([seed, 3])``: w_in [C_conv + Hv*d_v + 2*Hv, hidden] ~ N(0, 1/hidden)
    (rows stacked qkv, z, a, b) then w_out [hidden, Hv*d_v] ~ N(0, 1/(Hv*d_v))."""
    rng = np.random.default_rng([seed, 3])
    n_in = geo.conv_dim + geo.value_dim + 2 * geo.num_v_heads
    w_in = rng.standard_normal((n_in, hidden), dtype=np.float32) * np.float32(1.0 / np.sqrt(hidden))
    w_out = rng.standard_normal((hidden, geo.value_dim), dtype=np.float32) * np.float32(1.0 / np.sqrt(geo.value_dim))
    return bf16_bits_from_f32(w_in), bf16_bits_from_f32(w_out)


def make_hidden_states(num_tokens: int, hidden: int, seed: int) -> np.ndarray:
    """bf16 bits of a layer's input hidden states [T, hidden] ~ N(0, 1), from ``default_rng([seed, 4])``."""
    rng = np.random.default_rng([seed, 4])
    return bf16_bits_from_f32(rng.standard_normal((num_tokens, hidden), dtype=np.float32))


QWEN_GEO = Geometry()
TINY_GEO = Geometry(num_k_heads=2, num_v_heads=4, head_k_dim=32, head_v_dim=32, io_dtype="f32")

# Named workloads: (geometry, sequence lengths, seed, zero initial state, chunk sizes)
WORKLOADS = {
    # tiny fp32 mixer: 1 sequence, T=64, 2 key / 4 value heads, d=32, chunk 16
    "tiny_fp32_t64": dict(geo=TINY_GEO, lengths=[64], seed=0, zero_init=True, chunks=(16,)),
    # single-layer prefill, B=1, T=4096, 16K/48V x 128, chunk 64, bf16
    "prefill_t4096": dict(geo=QWEN_GEO, lengths=[4096], seed=1, zero_init=True, chunks=(64,)),
    # batched decode, 64 sequences, 1000 steps
    "decode_b64": dict(geo=QWEN_GEO, lengths=[1] * 64, seed=2, zero_init=False, chunks=(64,), steps=1000),
    # long-context prefill, B=1, T=65536, split-and-resume at 40961
    "prefill_t65536": dict(geo=QWEN_GEO, lengths=[65536], seed=3, zero_init=True, chunks=(64,), split=40961,
                           decode_tail=256),
    # packed varlen batch: 16 sequences, lengths uniform in 1..8192, chunk 16/64/128
    "varlen_16": dict(geo=QWEN_GEO, lengths=None, seed=4, zero_init=False, chunks=(16, 64, 128)),
}


def workload_inputs(name: str, lengths: Optional[list] = None) -> GdnInputs:
    w = WORKLOADS[name]
    if lengths is None:
        lengths = w["lengths"] if w["lengths"] is not None else list(varlen_lengths(w["seed"]))
    return make_prefill_inputs(w["geo"], lengths, w["seed"], w["zero_init"])
