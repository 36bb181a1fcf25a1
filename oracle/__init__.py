"""ctypes harness around the plain-C oracle (liboracle.so).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
benchmark's CPU-baseline / reference leg.  Nothing in the CUDA library imports
this package, and this package imports nothing from the CUDA library.

Weights are generated here from the seeded ``synth`` package: bf16 matrices are
taken as generated; quantized matrices are produced by the oracle's own RTN
quantizer (``or_quantize``) from the generated fp32 weights.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

import synth

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

EXACT, MIRROR = 0, 1
BF16, W8, W4, W3 = 0, 1, 2, 3
BITS = {W8: 8, W4: 4, W3: 3}


def build(force: bool = False) -> str:
    src = [os.path.join(_HERE, "oracle.c"), os.path.join(_HERE, "oracle.h")]
    if force or not os.path.exists(_SO) or any(os.path.getmtime(_SO) < os.path.getmtime(s) for s in src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _SO, src[0], "-lm"])
    return _SO


class OrMat(C.Structure):
    _fields_ = [("fmt", C.c_int), ("group", C.c_int), ("N", C.c_int), ("K", C.c_int), ("q", C.c_void_p),
                ("scales", C.c_void_p), ("zeros", C.c_void_p)]


class OrConfig(C.Structure):
    _fields_ = [("d_model", C.c_int), ("pattern", C.c_char_p), ("ssm_heads", C.c_int), ("ssm_head_dim", C.c_int),
                ("ssm_state", C.c_int), ("ssm_groups", C.c_int), ("conv_width", C.c_int), ("norm_groups", C.c_int),
                ("attn_q_heads", C.c_int), ("attn_kv_heads", C.c_int), ("attn_head_dim", C.c_int),
                ("mlp_hidden", C.c_int), ("vocab_text", C.c_int), ("vocab_func", C.c_int), ("eps", C.c_double)]


class OrLayer(C.Structure):
    _fields_ = [("norm", C.c_void_p), ("in_proj", OrMat), ("out_proj", OrMat), ("conv_w", C.c_void_p),
                ("conv_b", C.c_void_p), ("A_log", C.c_void_p), ("D", C.c_void_p), ("dt_bias", C.c_void_p),
                ("gnorm", C.c_void_p), ("qkv", OrMat), ("o", OrMat), ("up", OrMat), ("down", OrMat)]


class OrWeights(C.Structure):
    _fields_ = [("layers", C.POINTER(OrLayer)), ("final_norm", C.c_void_p), ("head_text", OrMat),
                ("head_func", OrMat)]


class OrState(C.Structure):
    _fields_ = [("n_slots", C.c_int), ("kv_capacity", C.c_int), ("ssm", C.c_void_p), ("conv", C.c_void_p),
                ("k", C.c_void_p), ("v", C.c_void_p), ("ctx_len", C.c_void_p)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(_SO)
        p = C.c_void_p
        L.or_quantize.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, p, p, p, p]
        L.or_quantize.restype = None
        L.or_codes.argtypes = [C.POINTER(OrMat), p, p, p]
        L.or_codes.restype = None
        L.or_dequant.argtypes = [C.POINTER(OrMat), p]
        L.or_dequant.restype = None
        L.or_matvec.argtypes = [C.POINTER(OrMat), p, p]
        L.or_matvec.restype = None
        L.or_step.argtypes = [C.POINTER(OrConfig), C.POINTER(OrWeights), C.POINTER(OrState), C.c_int, p, p, C.c_int,
                              p, p, p, p]
        L.or_step.restype = C.c_int
        L.or_layer_step.argtypes = [C.POINTER(OrConfig), C.POINTER(OrWeights), C.POINTER(OrState), C.c_int, C.c_int,
                                    p, p, C.c_int, p]
        L.or_layer_step.restype = C.c_int
        L.or_prefill_layer.argtypes = [C.POINTER(OrConfig), C.POINTER(OrWeights), C.POINTER(OrState), C.c_int, C.c_int,
                                       C.c_int, p, C.c_int, C.c_int, p]
        L.or_prefill_layer.restype = C.c_int
        L.or_heads.argtypes = [C.POINTER(OrConfig), C.POINTER(OrWeights), C.c_int, p, C.c_int, p, p, p]
        L.or_heads.restype = None
        L.or_prefill.argtypes = [C.POINTER(OrConfig), C.POINTER(OrWeights), C.POINTER(OrState), C.c_int, C.c_int, p,
                                 C.c_int, C.c_int, p]
        L.or_prefill.restype = C.c_int
        L.or_mamba_mixer.argtypes = [C.POINTER(OrConfig), C.POINTER(OrLayer), C.c_int, p, p, p, C.c_int, p, p]
        L.or_mamba_mixer.restype = None
        L.or_fuse_inputs.argtypes = [C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_int,
                                     C.c_void_p, C.c_void_p, C.c_void_p]
        L.or_fuse_inputs.restype = None
        L.or_round_bf16.argtypes = [C.c_double]
        L.or_round_bf16.restype = C.c_double
        L.or_round_fp16.argtypes = [C.c_double]
        L.or_round_fp16.restype = C.c_double
        L.or_threads.argtypes = []
        L.or_threads.restype = C.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


# ------------------------------------------------------------------------------------------------
# quantized matrices
# ------------------------------------------------------------------------------------------------

class Mat:
    """A weight matrix in the oracle's canonical storage, with its numpy buffers kept alive."""

    def __init__(self, fmt, group, N, K, q, scales=None, zeros=None):
        self.fmt, self.group, self.N, self.K = fmt, group, N, K
        self.q, self.scales, self.zeros = q, scales, zeros

    def c(self) -> OrMat:
        return OrMat(self.fmt, self.group, self.N, self.K, _ptr(self.q), _ptr(self.scales), _ptr(self.zeros))

    def dequant(self) -> np.ndarray:
        out = np.empty((self.N, self.K), np.float64)
        m = self.c()
        lib().or_dequant(C.byref(m), out.ctypes.data)
        return out

    def codes(self):
        ng = (self.K + self.group - 1) // self.group
        codes = np.empty((self.N, self.K), np.int32)
        zeros = np.empty((self.N, ng), np.int32)
        scales = np.empty((self.N, ng), np.float64)
        m = self.c()
        lib().or_codes(C.byref(m), codes.ctypes.data, zeros.ctypes.data, scales.ctypes.data)
        return codes, zeros, scales

    def matvec(self, u: np.ndarray) -> np.ndarray:
        u = np.ascontiguousarray(u, np.float64)
        y = np.empty((self.N,), np.float64)
        m = self.c()
        lib().or_matvec(C.byref(m), u.ctypes.data, y.ctypes.data)
        return y


def quantize(fmt: int, group: int, w: np.ndarray) -> Mat:
    w = np.ascontiguousarray(w, np.float32)
    N, K = w.shape
    b = BITS[fmt]
    ng = (K + group - 1) // group
    q = np.zeros((N, (K * b + 31) // 32), np.uint32)
    scales = np.zeros((N, ng), np.uint16)
    zeros = np.zeros((N, (ng * b + 31) // 32), np.uint32) if fmt != W8 else None
    lib().or_quantize(fmt, group, N, K, w.ctypes.data, q.ctypes.data, scales.ctypes.data, _ptr(zeros))
    return Mat(fmt, group, N, K, q, scales, zeros)


def bf16_mat(wbits: np.ndarray) -> Mat:
    wbits = np.ascontiguousarray(wbits, np.uint16)
    return Mat(BF16, 64, wbits.shape[0], wbits.shape[1], wbits)


def fuse_inputs(speech_bits, emb_text_bits, emb_func_bits, tok_text, tok_func):
    """bf16 bits of speech + emb_text[tok_text] + emb_func[tok_func] per row (exact sum, one RNE
    rounding; tokens outside the vocabulary add nothing)"""
    sp = np.ascontiguousarray(speech_bits, np.uint16)
    et = np.ascontiguousarray(emb_text_bits, np.uint16)
    ef = np.ascontiguousarray(emb_func_bits, np.uint16)
    tt = np.ascontiguousarray(tok_text, np.int32)
    tf = np.ascontiguousarray(tok_func, np.int32)
    B, d = sp.shape
    out = np.empty_like(sp)
    lib().or_fuse_inputs(B, d, sp.ctypes.data, et.ctypes.data, et.shape[0], ef.ctypes.data, ef.shape[0],
                         tt.ctypes.data, tf.ctypes.data, out.ctypes.data)
    return out


def round_bf16(v: float) -> float:
    return lib().or_round_bf16(float(v))


def round_fp16(v: float) -> float:
    return lib().or_round_fp16(float(v))


def threads() -> int:
    """threads the oracle's parallel loops run on"""
    return int(lib().or_threads())


# ------------------------------------------------------------------------------------------------
# model
# ------------------------------------------------------------------------------------------------

def make_config(cfg: synth.Config) -> OrConfig:
    oc = OrConfig()
    oc.d_model = cfg.d_model
    oc._pattern = cfg.pattern.encode()
    oc.pattern = oc._pattern
    for f in ("ssm_heads", "ssm_head_dim", "ssm_state", "ssm_groups", "conv_width", "norm_groups", "attn_q_heads",
              "attn_kv_heads", "attn_head_dim", "mlp_hidden", "vocab_text", "vocab_func"):
        setattr(oc, f, getattr(cfg, f))
    oc.eps = cfg.eps
    return oc


def _mat_from_synth(cfg, seed, layer, kind, N, K, fmt):
    if fmt == BF16:
        return bf16_mat(synth.linear_bf16(cfg, seed, layer, kind, N, K))
    return quantize(fmt, cfg.group_size, synth.linear_f32(cfg, seed, layer, kind, N, K))


class Model:
    """Oracle weights for a synth.Config (numpy buffers + ctypes views)."""

    def __init__(self, cfg: synth.Config, seed: int = 0):
        self.cfg = cfg
        self.seed = seed
        self.ocfg = make_config(cfg)
        n = cfg.n_layers
        self.layers = (OrLayer * n)()
        self.keep = []
        self.mats = {}
        self.small = {}
        for l in range(n):
            L = self.layers[l]
            sp = synth.small_params(cfg, seed, l)
            self.small[l] = sp
            self.keep.append(sp)
            L.norm = _ptr(sp["norm"])
            if cfg.pattern[l] == "M":
                L.conv_w, L.conv_b = _ptr(sp["conv_w"]), _ptr(sp["conv_b"])
                L.A_log, L.D, L.dt_bias, L.gnorm = _ptr(sp["A_log"]), _ptr(sp["D"]), _ptr(sp["dt_bias"]), _ptr(sp["gnorm"])
            for kind, N, K in synth.linear_shapes(cfg, l):
                m = _mat_from_synth(cfg, seed, l, kind, N, K, cfg.wfmt)
                self.mats[(l, kind)] = m
                name = {synth.K_IN: "in_proj", synth.K_OUT: "out_proj", synth.K_QKV: "qkv", synth.K_O: "o",
                        synth.K_UP: "up", synth.K_DOWN: "down"}[kind]
                setattr(L, name, m.c())
        self.final_norm = synth.final_norm(cfg, seed)
        heads = []
        for which in (synth.TID_HEAD_TEXT, synth.TID_HEAD_FUNC):
            if cfg.head_fmt == BF16:
                heads.append(bf16_mat(synth.head_bf16(cfg, seed, which)))
            else:
                heads.append(quantize(cfg.head_fmt, cfg.group_size, synth.head_f32(cfg, seed, which)))
        self.head_text, self.head_func = heads
        self.weights = OrWeights(self.layers, _ptr(self.final_norm), self.head_text.c(), self.head_func.c())

    # -------------------------------------------------------------------------------------------
    def new_state(self, n_slots: int, cap: int) -> "State":
        return State(self.cfg, n_slots, cap)

    def step(self, st: "State", x_bits: np.ndarray, mode: int = MIRROR, slots=None, taps: bool = False):
        x_bits = np.ascontiguousarray(x_bits, np.uint16)
        B = x_bits.shape[0]
        cfg = self.cfg
        tt = np.empty((B,), np.int32)
        tf = np.empty((B,), np.int32)
        hidden = np.zeros((cfg.n_layers + 1, B, cfg.d_model), np.float64) if taps else None
        V = max(cfg.vocab_text, cfg.vocab_func)
        logits = np.zeros((2, B, V), np.float64) if taps else None
        sl = None if slots is None else np.ascontiguousarray(slots, np.int32)
        rc = lib().or_step(C.byref(self.ocfg), C.byref(self.weights), C.byref(st.c), B, x_bits.ctypes.data, _ptr(sl),
                           mode, tt.ctypes.data, tf.ctypes.data, _ptr(hidden), _ptr(logits))
        return dict(rc=rc, tok_text=tt, tok_func=tf, hidden=hidden, logits=logits)

    def layer_step(self, st: "State", layer: int, r_in: np.ndarray, mode: int = MIRROR, slots=None):
        """One layer teacher-forced from the residual stream r_in [B][d] entering it; updates that
        layer's state in st (ctx_len is not advanced) and returns (rc, r_out [B][d])."""
        r_in = np.ascontiguousarray(r_in, np.float64)
        B = r_in.shape[0]
        r_out = np.empty_like(r_in)
        sl = None if slots is None else np.ascontiguousarray(slots, np.int32)
        rc = lib().or_layer_step(C.byref(self.ocfg), C.byref(self.weights), C.byref(st.c), layer, B,
                                 r_in.ctypes.data, _ptr(sl), mode, r_out.ctypes.data)
        return rc, r_out

    def heads(self, r: np.ndarray, mode: int = MIRROR):
        """Final norm, both heads and the greedy tokens from the residual r [B][d] leaving the last layer."""
        r = np.ascontiguousarray(r, np.float64)
        B = r.shape[0]
        tt = np.empty((B,), np.int32)
        tf = np.empty((B,), np.int32)
        V = max(self.cfg.vocab_text, self.cfg.vocab_func)
        logits = np.zeros((2, B, V), np.float64)
        lib().or_heads(C.byref(self.ocfg), C.byref(self.weights), B, r.ctypes.data, mode, tt.ctypes.data,
                       tf.ctypes.data, logits.ctypes.data)
        return dict(tok_text=tt, tok_func=tf, logits=logits)

    def prefill(self, st: "State", slot: int, x_bits: np.ndarray, mode: int = MIRROR, ssd_chunk: int = 0,
                taps: bool = False):
        x_bits = np.ascontiguousarray(x_bits, np.uint16)
        T = x_bits.shape[0]
        hidden = np.zeros((self.cfg.n_layers + 1, T, self.cfg.d_model), np.float64) if taps else None
        rc = lib().or_prefill(C.byref(self.ocfg), C.byref(self.weights), C.byref(st.c), slot, T, x_bits.ctypes.data,
                              mode, ssd_chunk, _ptr(hidden))
        return dict(rc=rc, hidden=hidden)

    def prefill_layer(self, st: "State", slot: int, layer: int, r_in: np.ndarray, mode: int = MIRROR,
                      ssd_chunk: int = 0):
        """One prefill layer teacher-forced from the residual r_in [T][d] of the frames entering it;
        updates that layer's state of the slot (ctx_len not advanced); returns (rc, r_out [T][d])."""
        r_in = np.ascontiguousarray(r_in, np.float64)
        T = r_in.shape[0]
        r_out = np.empty_like(r_in)
        rc = lib().or_prefill_layer(C.byref(self.ocfg), C.byref(self.weights), C.byref(st.c), slot, layer, T,
                                    r_in.ctypes.data, mode, ssd_chunk, r_out.ctypes.data)
        return rc, r_out

    def mamba_mixer(self, layer: int, zxbcdt: np.ndarray, ssm: np.ndarray, conv: np.ndarray, ssd_chunk: int = 0):
        """Isolated Mamba-2 mixer over T frames; ssm [H][P][N] and conv [W-1][Cx] are updated in place."""
        zxbcdt = np.ascontiguousarray(zxbcdt, np.float64)
        T = zxbcdt.shape[0]
        E = self.cfg.d_inner
        y = np.empty((T, E), np.float64)
        v = np.empty((T, E), np.float64)
        lib().or_mamba_mixer(C.byref(self.ocfg), C.byref(self.layers[layer]), T, zxbcdt.ctypes.data, ssm.ctypes.data,
                             conv.ctypes.data, ssd_chunk, y.ctypes.data, v.ctypes.data)
        return y, v


class State:
    """Oracle session state (double), logical layouts:
    ssm [nm][slots][H][P][N], conv [nm][slots][W-1][Cx], k/v [na][slots][Hk][cap][Dh], ctx_len [slots]."""

    def __init__(self, cfg: synth.Config, n_slots: int, cap: int):
        self.cfg = cfg
        self.n_slots, self.cap = n_slots, cap
        nm, na = max(cfg.n_mamba, 1), max(cfg.n_attn, 1)
        self.ssm = np.zeros((nm, n_slots, cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state), np.float64)
        self.conv = np.zeros((nm, n_slots, cfg.conv_width - 1, cfg.conv_dim), np.float64)
        self.k = np.zeros((na, n_slots, cfg.attn_kv_heads, cap, cfg.attn_head_dim), np.float64)
        self.v = np.zeros_like(self.k)
        self.ctx_len = np.zeros((n_slots,), np.int32)
        self.c = OrState(n_slots, cap, _ptr(self.ssm), _ptr(self.conv), _ptr(self.k), _ptr(self.v), _ptr(self.ctx_len))

    def clone(self) -> "State":
        o = State.__new__(State)
        o.cfg, o.n_slots, o.cap = self.cfg, self.n_slots, self.cap
        o.ssm, o.conv, o.k, o.v = self.ssm.copy(), self.conv.copy(), self.k.copy(), self.v.copy()
        o.ctx_len = self.ctx_len.copy()
        o.c = OrState(o.n_slots, o.cap, _ptr(o.ssm), _ptr(o.conv), _ptr(o.k), _ptr(o.v), _ptr(o.ctx_len))
        return o

    def fill_random(self, seed: int, ctx_lens: np.ndarray):
        """Pre-fill every slot from the seeded generator (the same tensors the GPU harness uploads)."""
        cfg = self.cfg
        B = self.n_slots
        for m in range(cfg.n_mamba):
            self.ssm[m] = synth.ssm_state(cfg, seed, m, B)
            self.conv[m] = synth.bf16_to_f32(synth.conv_history(cfg, seed, m, B))
        for a in range(cfg.n_attn):
            k, v = synth.kv_history(cfg, seed, a, B, self.cap)
            self.k[a] = synth.bf16_to_f32(k)
            self.v[a] = synth.bf16_to_f32(v)
        self.ctx_len[:] = ctx_lens
