"""Random-weight models and pre-filled session state from the seeded generator (``synth``).

Used by the benchmark and the tests to build a backbone of a given shape with synthetic
weights (no checkpoint is involved) and to lay a generated session state out in the state
buffers of vc.h.
"""
from __future__ import annotations

import numpy as np
import torch

import synth

from .model import DeviceModel


def build_model(cfg, seed: int = 0, device="cuda") -> DeviceModel:
    dm = DeviceModel(cfg, device)
    for l in range(cfg.n_layers):
        sp = synth.small_params(cfg, seed, l)
        for name, v in sp.items():
            dm.set_small(l, name, v)
        for kind, N, K in synth.linear_shapes(cfg, l):
            name = {synth.K_IN: "in_proj", synth.K_OUT: "out_proj", synth.K_QKV: "qkv", synth.K_O: "o",
                    synth.K_UP: "up", synth.K_DOWN: "down"}[kind]
            if cfg.wfmt == synth.FMT_BF16:
                w = synth.linear_bf16(cfg, seed, l, kind, N, K)
            else:
                w = synth.linear_f32(cfg, seed, l, kind, N, K)
            dm.set_linear(l, name, w)
            del w
    dm.set_final_norm(synth.final_norm(cfg, seed))
    for which, tid in (("text", synth.TID_HEAD_TEXT), ("func", synth.TID_HEAD_FUNC)):
        w = synth.head_bf16(cfg, seed, tid) if cfg.head_fmt == synth.FMT_BF16 else synth.head_f32(cfg, seed, tid)
        dm.set_head(which, w)
        del w
    torch.cuda.synchronize()
    return dm


def fill_state(state, cfg, seed: int, ctx_lens: np.ndarray, cap: int):
    """Pre-fill slots 0..B-1 of a State with the generator's session state at context ctx_lens[b]:
    SSM N(0,1), the last W-1 pre-conv rows N(0,1) (frame t's row goes to ring slot t mod W),
    cached K/V N(0,1) bf16."""
    B = len(ctx_lens)
    W = cfg.conv_width
    for m in range(cfg.n_mamba):
        state.ssm[m, :B] = torch.from_numpy(synth.ssm_state(cfg, seed, m, B)).to(state.ssm.device)
        hist = synth.conv_history(cfg, seed, m, B)           # [B][W-1][Cx] bf16 bits, oldest first
        ring = np.zeros((B, W, cfg.conv_dim), np.uint16)
        for b in range(B):
            t = int(ctx_lens[b])
            for i in range(W - 1):
                ring[b, (t - (W - 1) + i) % W] = hist[b, i]
        state.conv[m, :B] = torch.from_numpy(ring).to(state.conv.device).view(torch.bfloat16)
    for a in range(cfg.n_attn):
        k, v = synth.kv_history(cfg, seed, a, B, cap)
        state.k[a, :B] = torch.from_numpy(k).to(state.k.device).view(torch.bfloat16)
        state.v[a, :B] = torch.from_numpy(v).to(state.v.device).view(torch.bfloat16)
    state.ctx_len[:B] = torch.from_numpy(np.asarray(ctx_lens, np.int32)).to(state.ctx_len.device)


def ring_to_history(conv_ring: np.ndarray, t: int, W: int) -> np.ndarray:
    """GPU conv ring [W][Cx] of a session that has processed t frames -> last W-1 rows, oldest first."""
    return np.stack([conv_ring[(t - (W - 1) + i) % W] for i in range(W - 1)])
