"""Device-side buffers for a GDN problem (torch tensors; plumbing only).

``DeviceProblem`` uploads the io tensors, parameters and starting states of a
``GdnInputs`` problem, allocates the output and the prefill workspace, and
calls the C entry points through the binding.
"""

from __future__ import annotations

import numpy as np
import torch

from . import inputs as gi
from . import make_config, prefill_workspace_size
from . import prefill as _prefill
from . import decode_step as _decode_step


def io_tensor(arr: np.ndarray, device="cuda") -> torch.Tensor:
    """io-dtype numpy array (uint16 bf16 bits or float32) -> torch tensor on device."""
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


def io_numpy(t: torch.Tensor) -> np.ndarray:
    """torch io tensor -> numpy (uint16 bf16 bits or float32)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.uint16).numpy()
    return t.numpy()


def io_float(t: torch.Tensor) -> np.ndarray:
    """torch io tensor -> float64 numpy values."""
    return t.detach().float().cpu().numpy().astype(np.float64)


class DeviceProblem:
    def __init__(self, inp: gi.GdnInputs, chunk_size: int = 64, device="cuda"):
        self.inp = inp
        self.geo = inp.geo
        self.cfg = make_config(inp.geo)
        self.chunk_size = chunk_size
        dev = torch.device(device)
        self.device = dev
        self.qkv = io_tensor(inp.qkv, dev)
        self.z = io_tensor(inp.z, dev)
        self.a = io_tensor(inp.a, dev)
        self.b = io_tensor(inp.b, dev)
        self.params = tuple(torch.from_numpy(np.ascontiguousarray(p, np.float32)).to(dev)
                            for p in (inp.conv_w, inp.A_log, inp.dt_bias, inp.norm_w))
        self.cu_host = np.ascontiguousarray(inp.cu_seqlens, np.int32)
        self.cu_dev = torch.from_numpy(self.cu_host).to(dev)
        self.conv_state = io_tensor(inp.conv_state, dev)
        self.state = torch.from_numpy(np.ascontiguousarray(inp.state, np.float32)).to(dev)
        T = inp.total_tokens
        self.o = torch.empty((T, self.geo.value_dim), dtype=self.qkv.dtype, device=dev)
        ws = prefill_workspace_size(self.cfg, T, inp.num_seqs, chunk_size)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    def reset_states(self):
        self.conv_state.copy_(io_tensor(self.inp.conv_state, self.device))
        self.state.copy_(torch.from_numpy(np.ascontiguousarray(self.inp.state, np.float32)).to(self.device))

    def prefill(self, flags: int = 0, stream=None):
        _prefill(self.cfg, self.params, self.qkv, self.z, self.a, self.b, self.cu_dev, self.cu_host, self.chunk_size,
                 flags, self.conv_state, self.state, self.o, self.workspace, stream=stream)

    def decode(self, qkv, z, a, b, o, stream=None):
        _decode_step(self.cfg, self.params, qkv, z, a, b, self.inp.num_seqs, self.conv_state, self.state, o,
                     stream=stream)
