"""Python binding of libgdn.so, the Gated DeltaNet token mixer for B200.

Argument marshalling only: every function here hands device pointers of
torch tensors, sizes and the current CUDA stream to one C entry point of
``libgdn.so`` (declared in ``include/gdn.h``) and raises ``GdnError`` on a
non-zero status.  There is no fallback: if the library is missing or was not
built, the first call raises.  Build it with
``python -m linear_attention_recurrence_deltanet_b200.build``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

__all__ = [
    "GdnError", "Config", "Params", "lib", "make_config", "conv_prefill", "conv_step", "prefill_workspace_size",
    "prefill", "prefill_noalloc", "decode_step", "decode_multi", "decode_step_indexed", "decode_multi_indexed",
    "prefill_indexed_workspace_size", "prefill_indexed", "gemm_bf16", "project_in", "project_out", "prefill_seqpar_workspace_size", "prefill_seqpar", "state_blob_size", "state_save", "state_restore", "device_status", "debug_wait_expiry", "last_error",
    "abi_version", "launch_count", "launch_count_reset", "profiler_enable", "profiler_reset", "profiler_read",
    "kernel_name", "EXPORTS", "ZERO_INIT_STATE", "ZERO_INIT_CONV", "PREFILL_RECURRENT", "PREFILL_FUSED", "PREFILL_FACTORED", "PREFILL_AFFINE", "K", "MAX_DRAFT_TOKENS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdn.so")

ZERO_INIT_STATE = 0x1
ZERO_INIT_CONV = 0x2
PREFILL_RECURRENT = 0x4
PREFILL_FUSED = 0x8
PREFILL_FACTORED = 0x10
PREFILL_AFFINE = 0x20
MAX_DRAFT_TOKENS = 4

F32, BF16 = 0, 1

STATUS = {0: "GDN_OK", -1: "GDN_E_INVAL", -2: "GDN_E_UNSUPPORTED", -3: "GDN_E_WORKSPACE", -4: "GDN_E_CUDA",
          -5: "GDN_E_BLOB_FORMAT", -6: "GDN_E_BLOB_VERSION", -7: "GDN_E_BLOB_GEOMETRY", -8: "GDN_E_BLOB_CHECKSUM",
          -9: "GDN_E_DEVICE"}


class K:
    """Kernel ids of the profiler (gdn_kernel_id)."""
    (CONV_PREFILL, CONV_STEP, CONV_HISTORY, SCHEDULE, PREFILL_RECURRENT, PREFILL_CHUNKED, DECODE, STATE_CHECKSUM,
     SPLIT_CONV, SPLIT_PREP, SPLIT_CHAIN, SLOT_COPY, GEMM, SEQPAR, DIAG, WY_CONV, WY_PREP, WY_CHAIN) = range(18)
    COUNT = 18


# Every symbol include/gdn.h declares.
EXPORTS = [
    "gdn_conv_prefill", "gdn_conv_step", "gdn_prefill_workspace_size", "gdn_prefill", "gdn_decode_step",
    "gdn_state_blob_size", "gdn_state_save", "gdn_state_restore", "gdn_get_device_status", "gdn_last_error",
    "gdn_abi_version", "gdn_launch_count", "gdn_launch_count_reset", "gdn_kernel_name", "gdn_profiler_enable",
    "gdn_profiler_reset", "gdn_profiler_read", "gdn_prefill_noalloc", "gdn_decode_multi",
    "gdn_decode_step_indexed", "gdn_decode_multi_indexed", "gdn_prefill_indexed_workspace_size",
    "gdn_prefill_indexed", "gdn_gemm_bf16", "gdn_project_in", "gdn_project_out",
    "gdn_prefill_seqpar_workspace_size", "gdn_prefill_seqpar", "gdn_debug_wait_expiry",
]


class GdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.name = STATUS.get(status, str(status))


class Config(ctypes.Structure):
    _fields_ = [("num_k_heads", ctypes.c_int32), ("num_v_heads", ctypes.c_int32), ("head_k_dim", ctypes.c_int32),
                ("head_v_dim", ctypes.c_int32), ("conv_width", ctypes.c_int32), ("l2_eps", ctypes.c_float),
                ("norm_eps", ctypes.c_float), ("q_scale", ctypes.c_float), ("io_dtype", ctypes.c_int32)]


class Params(ctypes.Structure):
    _fields_ = [("conv_w", ctypes.c_void_p), ("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("norm_w", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m linear_attention_recurrence_deltanet_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, U32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_size_t
        sig = {
            "gdn_conv_prefill": [P, P, P, P, P, I32, P, P, P],
            "gdn_conv_step": [P, P, P, I32, P, P, P],
            "gdn_prefill_workspace_size": [P, I64, I32, I32, P],
            "gdn_prefill": [P, P, P, P, P, P, P, P, I32, I32, U32, P, P, P, P, SZ, P],
            "gdn_prefill_noalloc": [P, P, P, P, P, P, P, P, I32, I32, U32, P, P, P, P],
            "gdn_decode_step": [P, P, P, P, P, P, I32, P, P, P, P],
            "gdn_decode_multi": [P, P, P, P, P, P, I32, I32, I32, P, P, P, P, P],
            "gdn_decode_step_indexed": [P, P, P, P, P, P, I32, P, I32, P, P, P, P],
            "gdn_decode_multi_indexed": [P, P, P, P, P, P, I32, I32, I32, P, P, I32, P, P, P, P],
            "gdn_prefill_indexed_workspace_size": [P, I64, I32, I32, P],
            "gdn_prefill_indexed": [P, P, P, P, P, P, P, P, I32, P, I32, I32, U32, P, P, P, P, SZ, P],
            "gdn_gemm_bf16": [P, I32, I32, P, I32, P, I32, P],
            "gdn_project_in": [P, P, I32, I32, P, P, P, P, P, P],
            "gdn_project_out": [P, P, I32, P, I32, P, P],
            "gdn_prefill_seqpar_workspace_size": [P, I64, I32, P],
            "gdn_prefill_seqpar": [P, P, P, P, P, P, I64, I32, U32, P, P, P, P, SZ, P, P],
            "gdn_state_blob_size": [P, P],
            "gdn_state_save": [P, P, P, I32, P, SZ, P],
            "gdn_state_restore": [P, P, SZ, I32, P, P, P],
            "gdn_get_device_status": [P, P],
            "gdn_debug_wait_expiry": [ctypes.c_uint32, P],
            "gdn_profiler_enable": [I32],
            "gdn_profiler_reset": [],
            "gdn_profiler_read": [I32, P, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = I32
        L.gdn_last_error.restype = ctypes.c_char_p
        L.gdn_kernel_name.restype = ctypes.c_char_p
        L.gdn_kernel_name.argtypes = [I32]
        L.gdn_abi_version.restype = I32
        L.gdn_launch_count.restype = I64
        L.gdn_launch_count_reset.restype = None
        _lib = L
    return _lib


def last_error() -> str:
    return lib().gdn_last_error().decode()


def _check(rc: int):
    if rc != 0:
        raise GdnError(rc, last_error())


def make_config(geo) -> Config:
    """Config from an ``inputs.Geometry`` (or any object with the same fields)."""
    return Config(geo.num_k_heads, geo.num_v_heads, geo.head_k_dim, geo.head_v_dim, geo.conv_width, geo.l2_eps,
                  geo.norm_eps, geo.q_scale, BF16 if geo.io_dtype == "bf16" else F32)


def _p(t) -> Optional[int]:
    """Data pointer of a torch tensor / numpy array (None passes NULL)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    import torch
    return torch.cuda.current_stream().cuda_stream


def _host_cu(cu_host) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(cu_host), dtype=np.int32)


def _params(conv_w, A_log, dt_bias, norm_w) -> Params:
    return Params(_p(conv_w), _p(A_log), _p(dt_bias), _p(norm_w))


def conv_prefill(cfg, x, conv_w, cu_dev, cu_host, conv_state, y, stream=None):
    cu_h = _host_cu(cu_host)
    _check(lib().gdn_conv_prefill(ctypes.byref(cfg), _p(x), _p(conv_w), _p(cu_dev), cu_h.ctypes.data,
                                  cu_h.size - 1, _p(conv_state), _p(y), _stream(stream)))


def conv_step(cfg, x, conv_w, num_seqs, conv_state, y, stream=None):
    _check(lib().gdn_conv_step(ctypes.byref(cfg), _p(x), _p(conv_w), num_seqs, _p(conv_state), _p(y),
                               _stream(stream)))


def prefill_workspace_size(cfg, total_tokens: int, num_seqs: int, chunk_size: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().gdn_prefill_workspace_size(ctypes.byref(cfg), total_tokens, num_seqs, chunk_size,
                                            ctypes.byref(out)))
    return out.value


def prefill(cfg, params, qkv, z, a, b, cu_dev, cu_host, chunk_size, flags, conv_state, state, o, workspace,
            workspace_bytes=None, stream=None):
    """gdn_prefill.  params = (conv_w, A_log, dt_bias, norm_w) device tensors."""
    cu_h = _host_cu(cu_host)
    prm = _params(*params)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().gdn_prefill(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b), _p(cu_dev),
                             cu_h.ctypes.data, cu_h.size - 1, chunk_size, flags, _p(conv_state), _p(state), _p(o),
                             _p(workspace), workspace_bytes, _stream(stream)))


def prefill_noalloc(cfg, params, qkv, z, a, b, cu_dev, cu_host, chunk_size, flags, conv_state, state, o,
                    stream=None):
    """gdn_prefill_noalloc: gdn_prefill with the library's built-in scratch
    instead of a caller workspace (for callers that cannot allocate device
    memory); calls that overlap on the GPU share that scratch and race."""
    cu_h = _host_cu(cu_host)
    prm = _params(*params)
    _check(lib().gdn_prefill_noalloc(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b), _p(cu_dev),
                                     cu_h.ctypes.data, cu_h.size - 1, chunk_size, flags, _p(conv_state), _p(state),
                                     _p(o), _stream(stream)))


def decode_step(cfg, params, qkv, z, a, b, num_seqs, conv_state, state, o, stream=None):
    prm = _params(*params)
    _check(lib().gdn_decode_step(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b), num_seqs,
                                 _p(conv_state), _p(state), _p(o), _stream(stream)))


def decode_multi(cfg, params, qkv, z, a, b, num_seqs, num_tokens, commit, accept, conv_state, state, o,
                 stream=None):
    """gdn_decode_multi: num_tokens draft tokens per sequence in one pass.
    commit=False verifies (outputs only, caches untouched, accept None);
    commit=True applies accept[n] tokens (device int32, None = all)."""
    prm = _params(*params)
    _check(lib().gdn_decode_multi(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b), num_seqs,
                                  num_tokens, 1 if commit else 0, _p(accept),
                                  _p(conv_state), _p(state), _p(o), _stream(stream)))


def decode_step_indexed(cfg, params, qkv, z, a, b, num_seqs, state_indices, num_slots, conv_state, state, o,
                        stream=None):
    """gdn_decode_step_indexed: row n of the batch uses pool slot
    state_indices[n] (device int32; negative = padding row)."""
    prm = _params(*params)
    _check(lib().gdn_decode_step_indexed(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b),
                                         num_seqs, _p(state_indices), num_slots, _p(conv_state), _p(state), _p(o),
                                         _stream(stream)))


def decode_multi_indexed(cfg, params, qkv, z, a, b, num_seqs, num_tokens, commit, accept, state_indices, num_slots,
                         conv_state, state, o, stream=None):
    """gdn_decode_multi_indexed: gdn_decode_multi over pool slots."""
    prm = _params(*params)
    _check(lib().gdn_decode_multi_indexed(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b),
                                          num_seqs, num_tokens, 1 if commit else 0, _p(accept), _p(state_indices),
                                          num_slots, _p(conv_state), _p(state), _p(o), _stream(stream)))


def prefill_indexed_workspace_size(cfg, total_tokens: int, num_seqs: int, chunk_size: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().gdn_prefill_indexed_workspace_size(ctypes.byref(cfg), total_tokens, num_seqs, chunk_size,
                                                    ctypes.byref(out)))
    return out.value


def prefill_indexed(cfg, params, qkv, z, a, b, cu_dev, cu_host, state_indices, num_slots, chunk_size, flags,
                    conv_state, state, o, workspace, workspace_bytes=None, stream=None):
    """gdn_prefill_indexed: gdn_prefill over pool slots (a batch may mix
    prefill sequences with length-1 decode steps)."""
    cu_h = _host_cu(cu_host)
    prm = _params(*params)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().gdn_prefill_indexed(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b), _p(cu_dev),
                                     cu_h.ctypes.data, cu_h.size - 1, _p(state_indices), num_slots, chunk_size, flags,
                                     _p(conv_state), _p(state), _p(o), _p(workspace), workspace_bytes,
                                     _stream(stream)))


def gemm_bf16(x, w, y, tile_n: int = 0, stream=None):
    """gdn_gemm_bf16: y [M, N] = x [M, K] @ w [N, K]^T, all bf16 (fp32 accumulation)."""
    M, K = x.shape[0], x.shape[1]
    N = w.shape[0]
    _check(lib().gdn_gemm_bf16(_p(x), M, K, _p(w), N, _p(y), tile_n, _stream(stream)))


def project_in(cfg, x, w_in, qkv, z, a, b, stream=None):
    """gdn_project_in: x [T, hidden] through w_in [C_conv + Hv*d_v + 2*Hv, hidden] into qkv, z, a, b."""
    _check(lib().gdn_project_in(ctypes.byref(cfg), _p(x), x.shape[0], x.shape[1], _p(w_in), _p(qkv), _p(z), _p(a),
                                _p(b), _stream(stream)))


def project_out(cfg, o, w_out, y, stream=None):
    """gdn_project_out: y [T, hidden] = o [T, Hv*d_v] @ w_out [hidden, Hv*d_v]^T."""
    _check(lib().gdn_project_out(ctypes.byref(cfg), _p(o), o.shape[0], _p(w_out), w_out.shape[0], _p(y),
                                 _stream(stream)))


def prefill_seqpar_workspace_size(cfg, total_tokens: int, segments: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(lib().gdn_prefill_seqpar_workspace_size(ctypes.byref(cfg), total_tokens, segments, ctypes.byref(out)))
    return out.value


def prefill_seqpar(cfg, params, qkv, z, a, b, total_tokens, segments, flags, conv_state, state, o, workspace,
                   workspace_bytes=None, stream=None) -> int:
    """gdn_prefill_seqpar: one sequence of total_tokens tokens in `segments`
    chunk-aligned segments (0 = from the SM count); returns the count used."""
    prm = _params(*params)
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    used = ctypes.c_int32(0)
    _check(lib().gdn_prefill_seqpar(ctypes.byref(cfg), ctypes.byref(prm), _p(qkv), _p(z), _p(a), _p(b), total_tokens,
                                    segments, flags, _p(conv_state), _p(state), _p(o), _p(workspace),
                                    workspace_bytes, ctypes.byref(used), _stream(stream)))
    return used.value


def state_blob_size(cfg) -> int:
    out = ctypes.c_size_t()
    _check(lib().gdn_state_blob_size(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def _nbytes(t) -> int:
    return t.nbytes if isinstance(t, np.ndarray) else t.numel() * t.element_size()


def state_save(cfg, conv_state, state, seq, blob, stream=None):
    _check(lib().gdn_state_save(ctypes.byref(cfg), _p(conv_state), _p(state), seq, _p(blob), _nbytes(blob),
                                _stream(stream)))


def state_restore(cfg, blob, seq, conv_state, state, stream=None):
    _check(lib().gdn_state_restore(ctypes.byref(cfg), _p(blob), _nbytes(blob), seq, _p(conv_state), _p(state),
                                   _stream(stream)))


def device_status(stream=None) -> int:
    code = ctypes.c_int32()
    _check(lib().gdn_get_device_status(ctypes.byref(code), _stream(stream)))
    return code.value


def debug_wait_expiry(limit_us: int, stream=None):
    """gdn_debug_wait_expiry: a kernel whose bounded wait always runs out
    after limit_us; the device status word then reads 1 (wait timeout)."""
    _check(lib().gdn_debug_wait_expiry(limit_us, _stream(stream)))


def abi_version() -> int:
    return lib().gdn_abi_version()


def launch_count() -> int:
    return lib().gdn_launch_count()


def launch_count_reset():
    lib().gdn_launch_count_reset()


def kernel_name(kid: int) -> str:
    return lib().gdn_kernel_name(kid).decode()


def profiler_enable(on: bool = True):
    _check(lib().gdn_profiler_enable(1 if on else 0))


def profiler_reset():
    _check(lib().gdn_profiler_reset())


def profiler_read(kid: int):
    """(launches, total device ms) of one kernel id since the last reset."""
    n, ms = ctypes.c_int64(), ctypes.c_double()
    _check(lib().gdn_profiler_read(kid, ctypes.byref(n), ctypes.byref(ms)))
    return n.value, ms.value
