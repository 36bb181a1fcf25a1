"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle harness.

This package holds no model arithmetic.  It defines
  * the workload shapes (the tiny hybrid stack and the Nemotron-Nano-9B-v2
    shaped backbone described on the NemotronLabs VoiceChat model pages), and
  * counter-based random tensors (SplitMix64 + Box-Muller, see synth.c) keyed
    by (seed, tensor id), so any tensor can be regenerated on its own.

Seeds: weights use ``seed``, frame inputs ``seed + 1``, pre-filled session
state ``seed + 2`` and per-session context lengths ``seed + 3``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _SO, src, "-lm"])
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        u64, p = ctypes.c_uint64, ctypes.c_void_p
        L.synth_uniform_u64.argtypes = [u64, u64, u64, p]
        L.synth_normal_f32.argtypes = [u64, u64, u64, ctypes.c_double, ctypes.c_double, p]
        L.synth_normal_bf16.argtypes = [u64, u64, u64, ctypes.c_double, ctypes.c_double, p]
        L.synth_uniform_f32.argtypes = [u64, u64, u64, ctypes.c_double, ctypes.c_double, p]
        L.synth_uniform_i32.argtypes = [u64, u64, u64, ctypes.c_int32, ctypes.c_int32, p]
        L.synth_f32_to_bf16.argtypes = [u64, p, p]
        for f in (L.synth_uniform_u64, L.synth_normal_f32, L.synth_normal_bf16, L.synth_uniform_f32,
                  L.synth_uniform_i32, L.synth_f32_to_bf16):
            f.restype = None
        _lib = L
    return _lib


def _n(shape):
    return int(np.prod(shape)) if len(shape) else 1


def normal_f32(seed, tid, shape, mean=0.0, std=1.0, out=None):
    shape = tuple(shape)
    a = np.empty(shape, np.float32) if out is None else out
    lib().synth_normal_f32(seed, tid, _n(shape), mean, std, a.ctypes.data)
    return a


def normal_bf16(seed, tid, shape, mean=0.0, std=1.0, out=None):
    """bf16 bit patterns (np.uint16) of N(mean, std) samples rounded to nearest even."""
    shape = tuple(shape)
    a = np.empty(shape, np.uint16) if out is None else out
    lib().synth_normal_bf16(seed, tid, _n(shape), mean, std, a.ctypes.data)
    return a


def uniform_f32(seed, tid, shape, lo, hi, out=None):
    shape = tuple(shape)
    a = np.empty(shape, np.float32) if out is None else out
    lib().synth_uniform_f32(seed, tid, _n(shape), lo, hi, a.ctypes.data)
    return a


def uniform_i32(seed, tid, shape, lo, hi):
    shape = tuple(shape)
    a = np.empty(shape, np.int32)
    lib().synth_uniform_i32(seed, tid, _n(shape), lo, hi, a.ctypes.data)
    return a


def uniform_u64(seed, tid, n):
    a = np.empty((n,), np.uint64)
    lib().synth_uniform_u64(seed, tid, n, a.ctypes.data)
    return a


def f32_to_bf16(a):
    a = np.ascontiguousarray(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().synth_f32_to_bf16(a.size, a.ctypes.data, out.ctypes.data)
    return out


def bf16_to_f32(a):
    return (np.ascontiguousarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------------------------
# workload shapes
# ----------------------------------------------------------------------------------------------

FMT_BF16, FMT_W8, FMT_W4, FMT_W3 = 0, 1, 2, 3
FMT_NAMES = {FMT_BF16: "bf16", FMT_W8: "w8", FMT_W4: "w4", FMT_W3: "w3"}


def nano_pattern() -> str:
    """56 layers: attention at 0-based 7, 18, 29, 40; Mamba-2 at the other even indices and 55;
    MLP elsewhere (27 M + 4 attention + 25 MLP)."""
    s = []
    for i in range(56):
        if i in (7, 18, 29, 40):
            s.append("*")
        elif i % 2 == 0 or i == 55:
            s.append("M")
        else:
            s.append("-")
    return "".join(s)


@dataclasses.dataclass
class Config:
    name: str
    d_model: int
    pattern: str
    ssm_heads: int
    ssm_head_dim: int
    ssm_state: int
    ssm_groups: int
    conv_width: int
    norm_groups: int
    attn_q_heads: int
    attn_kv_heads: int
    attn_head_dim: int
    mlp_hidden: int
    vocab_text: int
    vocab_func: int
    eps: float = 1e-5
    wfmt: int = FMT_BF16
    group_size: int = 64
    head_fmt: int = FMT_BF16
    batch: int = 1
    ctx: int = 0            # frames already cached before the first timed step (per session)
    ctx_range: tuple | None = None  # ragged contexts drawn U{lo..hi} per session
    steps: int = 64
    prefill_T: int = 0
    kv_capacity: int = 0
    random_state: bool = False

    @property
    def n_layers(self):
        return len(self.pattern)

    @property
    def d_inner(self):
        return self.ssm_heads * self.ssm_head_dim

    @property
    def conv_dim(self):
        return self.d_inner + 2 * self.ssm_groups * self.ssm_state

    @property
    def in_proj_rows(self):
        return self.d_inner + self.conv_dim + self.ssm_heads

    @property
    def qkv_rows(self):
        return (self.attn_q_heads + 2 * self.attn_kv_heads) * self.attn_head_dim

    @property
    def n_mamba(self):
        return self.pattern.count("M")

    @property
    def n_attn(self):
        return self.pattern.count("*")

    @property
    def n_mlp(self):
        return self.pattern.count("-")

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)


def tiny_config(**kw) -> Config:
    c = Config(name="tiny", d_model=256, pattern="M-*-", ssm_heads=8, ssm_head_dim=32, ssm_state=16,
               ssm_groups=1, conv_width=4, norm_groups=1, attn_q_heads=4, attn_kv_heads=2,
               attn_head_dim=64, mlp_hidden=1024, vocab_text=1024, vocab_func=1024,
               wfmt=FMT_W8, group_size=64, head_fmt=FMT_W8, batch=1, ctx=0, steps=64,
               kv_capacity=128, random_state=False)
    return c.replace(**kw)


def nano_config(**kw) -> Config:
    c = Config(name="nano_bf16", d_model=4480, pattern=nano_pattern(), ssm_heads=128, ssm_head_dim=80,
               ssm_state=128, ssm_groups=8, conv_width=4, norm_groups=8, attn_q_heads=40,
               attn_kv_heads=8, attn_head_dim=128, mlp_hidden=15680, vocab_text=131072,
               vocab_func=131072, wfmt=FMT_BF16, group_size=64, head_fmt=FMT_BF16, batch=1,
               ctx=2000, steps=1000, kv_capacity=3300, random_state=True)
    return c.replace(**kw)


CONFIGS = {
    "tiny_w8": tiny_config(),
    "nano_bf16": nano_config(),
    "nano_w4": nano_config(name="nano_w4", wfmt=FMT_W4, group_size=64),
    "nano_w3": nano_config(name="nano_w3", wfmt=FMT_W3, group_size=64),
    # W4 backbone with 4-bit vocabulary heads too (the heads are 35% of the W4 step's bytes in bf16)
    "nano_w4_qheads": nano_config(name="nano_w4_qheads", wfmt=FMT_W4, group_size=64, head_fmt=FMT_W4),
    "nano_w8_b16": nano_config(name="nano_w8_b16", wfmt=FMT_W8, group_size=128, batch=16,
                               ctx_range=(500, 6000), steps=500, kv_capacity=7000),
    # the W4 backbone serving 16 sessions of ragged contexts (C2's weights with C3's batch)
    "nano_w4_b16": nano_config(name="nano_w4_b16", wfmt=FMT_W4, group_size=64, batch=16,
                               ctx_range=(500, 6000), steps=500, kv_capacity=7000),
    "nano_prefill": nano_config(name="nano_prefill", ctx=0, prefill_T=4096, steps=0,
                                kv_capacity=4096 + 64, random_state=False),
}

# ----------------------------------------------------------------------------------------------
# tensor ids
# ----------------------------------------------------------------------------------------------
K_NORM, K_IN, K_OUT, K_CONVW, K_CONVB, K_ALOG, K_D, K_DTB, K_GNORM, K_QKV, K_O, K_UP, K_DOWN = range(13)
TID_FINAL_NORM, TID_HEAD_TEXT, TID_HEAD_FUNC = 1, 2, 3
TID_EMB_TEXT, TID_EMB_FUNC = 4, 5


def layer_tid(layer, kind):
    return 1000 + layer * 32 + kind


def linear_shapes(cfg: Config, layer: int):
    """(kind, N, K) of the linear weights of one layer."""
    t = cfg.pattern[layer]
    d = cfg.d_model
    if t == "M":
        return [(K_IN, cfg.in_proj_rows, d), (K_OUT, d, cfg.d_inner)]
    if t == "*":
        return [(K_QKV, cfg.qkv_rows, d), (K_O, d, cfg.attn_q_heads * cfg.attn_head_dim)]
    return [(K_UP, cfg.mlp_hidden, d), (K_DOWN, d, cfg.mlp_hidden)]


def linear_f32(cfg: Config, seed: int, layer: int, kind: int, N: int, K: int):
    return normal_f32(seed, layer_tid(layer, kind), (N, K), 0.0, 0.02)


def linear_bf16(cfg: Config, seed: int, layer: int, kind: int, N: int, K: int):
    return normal_bf16(seed, layer_tid(layer, kind), (N, K), 0.0, 0.02)


def head_f32(cfg: Config, seed: int, which: int):
    V = cfg.vocab_text if which == TID_HEAD_TEXT else cfg.vocab_func
    return normal_f32(seed, which, (V, cfg.d_model), 0.0, 0.02)


def head_bf16(cfg: Config, seed: int, which: int):
    V = cfg.vocab_text if which == TID_HEAD_TEXT else cfg.vocab_func
    return normal_bf16(seed, which, (V, cfg.d_model), 0.0, 0.02)


def small_params(cfg: Config, seed: int, layer: int) -> dict:
    """fp32 per-layer vectors: pre-norm gamma and the Mamba-2 mixer's small parameters."""
    t = cfg.pattern[layer]
    d = cfg.d_model
    p = {"norm": normal_f32(seed, layer_tid(layer, K_NORM), (d,), 1.0, 0.1)}
    if t == "M":
        W, Cx, H, E = cfg.conv_width, cfg.conv_dim, cfg.ssm_heads, cfg.d_inner
        p["conv_w"] = uniform_f32(seed, layer_tid(layer, K_CONVW), (Cx, W), -0.5, 0.5)
        p["conv_b"] = uniform_f32(seed, layer_tid(layer, K_CONVB), (Cx,), -0.5, 0.5)
        p["A_log"] = uniform_f32(seed, layer_tid(layer, K_ALOG), (H,), 0.0, 1.5)
        p["D"] = uniform_f32(seed, layer_tid(layer, K_D), (H,), 0.5, 1.5)
        p["dt_bias"] = uniform_f32(seed, layer_tid(layer, K_DTB), (H,), -4.0, -2.0)
        p["gnorm"] = normal_f32(seed, layer_tid(layer, K_GNORM), (E,), 1.0, 0.1)
    return p


def final_norm(cfg: Config, seed: int):
    return normal_f32(seed, TID_FINAL_NORM, (cfg.d_model,), 1.0, 0.1)


def frame_inputs(cfg: Config, seed: int, step: int, B: int | None = None):
    """fused per-frame input embeddings x[B][d] (bf16 bits) for decode step ``step``."""
    B = cfg.batch if B is None else B
    return normal_bf16(seed + 1, 100 + step, (B, cfg.d_model))


def token_embeddings(cfg: Config, seed: int):
    """bf16 bits of the text and function token embedding tables, N(0, 0.5): [Vt][d], [Vf][d]."""
    return (normal_bf16(seed, TID_EMB_TEXT, (cfg.vocab_text, cfg.d_model), 0.0, 0.5),
            normal_bf16(seed, TID_EMB_FUNC, (cfg.vocab_func, cfg.d_model), 0.0, 0.5))


def prefill_inputs(cfg: Config, seed: int, T: int):
    return normal_bf16(seed + 1, 0, (T, cfg.d_model))


def context_lengths(cfg: Config, seed: int, B: int | None = None):
    B = cfg.batch if B is None else B
    if cfg.ctx_range is None:
        return np.full((B,), cfg.ctx, np.int32)
    lo, hi = cfg.ctx_range
    return uniform_i32(seed + 3, 0, (B,), lo, hi)


# pre-filled session state (logical layouts):
#   ssm[m]  : [B][H][P][N] fp32
#   conv[m] : [B][W-1][Cx] bf16, the last W-1 pre-conv xBC rows, oldest first
#   k[a], v[a] : [B][Hk][ctx][Dh] bf16, cached frames 0..ctx-1
def ssm_state(cfg: Config, seed: int, m: int, B: int):
    return normal_f32(seed + 2, 100 + m, (B, cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state))


def conv_history(cfg: Config, seed: int, m: int, B: int):
    return normal_bf16(seed + 2, 200 + m, (B, cfg.conv_width - 1, cfg.conv_dim))


def kv_history(cfg: Config, seed: int, a: int, B: int, cap: int):
    k = normal_bf16(seed + 2, 300 + a, (B, cfg.attn_kv_heads, cap, cfg.attn_head_dim))
    v = normal_bf16(seed + 2, 400 + a, (B, cfg.attn_kv_heads, cap, cfg.attn_head_dim))
    return k, v
