"""Load host weight arrays into libvc's device layout and build a Backbone.

A user with a checkpoint passes each linear weight as an [N][K] array (fp32 to be quantized by
vc_quantize_weight, or bf16 for the dense format) and the small per-layer vectors as fp32.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import (W_BF16, Backbone, State, VcLayerWeights, VcWeights, pack_bf16_weight, qmat, quantize_weight,
               weight_bytes)

LINEAR_NAMES = ("in_proj", "out_proj", "qkv", "o", "up", "down")
SMALL_NAMES = ("norm", "conv_w", "conv_b", "A_log", "D", "dt_bias", "gnorm")


def _to_dev(a, dtype, device):
    """host array / tensor -> contiguous CUDA tensor (uint16 host arrays are bf16 bit patterns)"""
    if isinstance(a, torch.Tensor):
        return a.to(device=device, dtype=dtype).contiguous()
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a).to(device).view(torch.bfloat16).to(dtype)
    return torch.from_numpy(a.astype(np.float32, copy=False)).to(device).to(dtype)


class DeviceModel:
    def __init__(self, cfg, device="cuda"):
        self.cfg = cfg
        self.device = device
        self.L = len(cfg.pattern)
        self.layers = (VcLayerWeights * self.L)()
        self.keep = []
        self.final_norm = None
        self.heads = {}
        self.bytes = 0

    def _linear(self, w, fmt, N, K):
        """w: host fp32 [N][K] (any format) or host uint16 bf16 bits [N][K] (dense format)."""
        if fmt == W_BF16 and isinstance(w, np.ndarray) and w.dtype == np.uint16:
            wd = torch.from_numpy(w).to(self.device).view(torch.bfloat16)
            buf = pack_bf16_weight(wd)
        else:
            wd = _to_dev(w, torch.float32, self.device)
            buf = quantize_weight(wd, fmt, self.cfg.group_size)
        del wd
        self.keep.append(buf)
        self.bytes += buf.numel()
        return buf

    def set_linear(self, layer: int, name: str, w):
        N, K = w.shape
        buf = self._linear(w, self.cfg.wfmt, N, K)
        setattr(self.layers[layer], name, qmat(buf, self.cfg.wfmt, self.cfg.group_size, N, K))

    def set_small(self, layer: int, name: str, v):
        t = _to_dev(v, torch.float32, self.device)
        self.keep.append(t)
        setattr(self.layers[layer], name, t.data_ptr())

    def set_final_norm(self, v):
        self.final_norm = _to_dev(v, torch.float32, self.device)

    def set_head(self, which: str, w):
        N, K = w.shape
        buf = self._linear(w, self.cfg.head_fmt, N, K)
        self.heads[which] = qmat(buf, self.cfg.head_fmt, self.cfg.group_size, N, K)

    def weights(self) -> VcWeights:
        return VcWeights(self.layers, self.final_norm.data_ptr(), self.heads["text"], self.heads["func"])

    def backbone(self, max_batch: int, kv_capacity: int, n_slots: int | None = None) -> Backbone:
        n_slots = max_batch if n_slots is None else n_slots
        return Backbone(self.cfg, self.weights(), max_batch, kv_capacity, n_slots, self.device, keepalive=self)

    def new_state(self, n_slots: int, kv_capacity: int) -> State:
        return State(self.cfg, n_slots, kv_capacity, self.device)
