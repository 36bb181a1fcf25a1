"""Python binding of libvc (include/vc.h): argument marshalling only.

Every computation runs in the CUDA kernels of libvc.so; PyTorch provides device memory and
streams.  Importing this package fails loudly if libvc.so has not been built
(``python attention_frame_decode_b200/build.py``).
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvc.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libvc.so not found at {LIB_PATH}; build it with `python attention_frame_decode_b200/build.py`")

_lib = C.CDLL(LIB_PATH)

VC_OK, VC_ERR_INVALID_ARG, VC_ERR_UNSUPPORTED, VC_ERR_CUDA, VC_ERR_CAPACITY, VC_ERR_STATE = range(6)
VC_DEV_CAPACITY, VC_DEV_NONFINITE, VC_DEV_TIMEOUT = 1, 2, 4
W_BF16, W_INT8_SYM, W_INT4_ASYM, W_INT3_ASYM = 0, 1, 2, 3
OPT_GRAPH, OPT_PDL, OPT_FRAME, OPT_GEMV_SHAPE = 1, 2, 3, 4


class VcConfig(C.Structure):
    _fields_ = [("d_model", C.c_int), ("pattern", C.c_char_p), ("ssm_heads", C.c_int), ("ssm_head_dim", C.c_int),
                ("ssm_state", C.c_int), ("ssm_groups", C.c_int), ("conv_width", C.c_int), ("norm_groups", C.c_int),
                ("attn_q_heads", C.c_int), ("attn_kv_heads", C.c_int), ("attn_head_dim", C.c_int),
                ("mlp_hidden", C.c_int), ("vocab_text", C.c_int), ("vocab_func", C.c_int), ("eps", C.c_float),
                ("wfmt", C.c_int), ("group_size", C.c_int), ("head_fmt", C.c_int), ("max_batch", C.c_int),
                ("kv_capacity", C.c_int), ("n_slots", C.c_int)]


class VcQmat(C.Structure):
    _fields_ = [("data", C.c_void_p), ("fmt", C.c_int), ("group", C.c_int), ("N", C.c_int), ("K", C.c_int)]


class VcLayerWeights(C.Structure):
    _fields_ = [("norm", C.c_void_p), ("in_proj", VcQmat), ("out_proj", VcQmat), ("conv_w", C.c_void_p),
                ("conv_b", C.c_void_p), ("A_log", C.c_void_p), ("D", C.c_void_p), ("dt_bias", C.c_void_p),
                ("gnorm", C.c_void_p), ("qkv", VcQmat), ("o", VcQmat), ("up", VcQmat), ("down", VcQmat)]


class VcWeights(C.Structure):
    _fields_ = [("layers", C.POINTER(VcLayerWeights)), ("final_norm", C.c_void_p), ("head_text", VcQmat),
                ("head_func", VcQmat)]


class VcTokenEmbeddings(C.Structure):
    _fields_ = [("emb_text", C.c_void_p), ("emb_func", C.c_void_p)]


class VcState(C.Structure):
    _fields_ = [("ssm", C.c_void_p), ("conv", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p),
                ("ctx_len", C.c_void_p), ("status", C.c_void_p)]


_p = C.c_void_p
_i = C.c_int
_lib.vc_weight_bytes.argtypes = [_i, _i, _i, _i]
_lib.vc_weight_bytes.restype = C.c_size_t
_lib.vc_quantize_weight.argtypes = [_i, _i, _i, _i, _p, _p, _p]
_lib.vc_pack_bf16_weight.argtypes = [_i, _i, _p, _p, _p]
_lib.vc_pack_weight.argtypes = [_i, _i, _i, _i, _p, _p, _p, _p, _p]
_lib.vc_debug_dequant.argtypes = [C.POINTER(VcQmat), _p, _p]
_lib.vc_workspace_bytes.argtypes = [C.POINTER(VcConfig)]
_lib.vc_workspace_bytes.restype = C.c_size_t
_lib.vc_backbone_create.argtypes = [C.POINTER(VcConfig), C.POINTER(VcWeights), _p, C.c_size_t, _p, C.POINTER(_p)]
_lib.vc_set_option.argtypes = [_p, _i, _i]
_lib.vc_uses_frame_kernel.argtypes = [_p, _i]
_lib.vc_uses_frame_kernel.restype = _i
_lib.vc_step.argtypes = [_p, _p, _i, _p, C.POINTER(VcState), _p, _p, _p]
_lib.vc_step_fused.argtypes = [_p, _p, C.POINTER(VcTokenEmbeddings), _i, _p, C.POINTER(VcState), _p, _p, _p]
_lib.vc_step_host.argtypes = [_p, _p, _i, _p, C.POINTER(VcState), _p, _p, _p]
_lib.vc_prefill.argtypes = [_p, _p, _i, _i, C.POINTER(VcState), _p]
_lib.vc_debug_set_taps.argtypes = [_p, _p, _p]
_lib.vc_debug_set_prefill_taps.argtypes = [_p, _p, _p]
_lib.vc_debug_set_zx_taps.argtypes = [_p, _p]
_lib.vc_debug_mamba_step.argtypes = [C.POINTER(VcConfig), C.POINTER(VcLayerWeights), _p, _i, _p, _p, _p, _p, _p, _p,
                                      _p, _p]
_lib.vc_gemv_scratch_bytes.argtypes = []
_lib.vc_gemv_scratch_bytes.restype = C.c_size_t
_lib.vc_debug_gemv.argtypes = [C.POINTER(VcQmat), _p, _i, _i, _p, _p, _p]
_lib.vc_gemv_noalloc_scratch_bytes.argtypes = []
_lib.vc_gemv_noalloc_scratch_bytes.restype = C.c_size_t
_lib.vc_debug_gemv_noalloc.argtypes = [C.POINTER(VcQmat), _p, _i, _i, _p, _p]
_lib.vc_gemv_noalloc_status.argtypes = [C.POINTER(C.c_int32), _p]
_lib.vc_gemv_noalloc_reset.argtypes = [_p]
_lib.vc_debug_gemm.argtypes = [_p, _i, _i, _p, _i, _i, _i, _i, _p, _i, _p, _p]
_lib.vc_debug_mamba_prefill_scratch_bytes.argtypes = [C.POINTER(VcConfig), _i]
_lib.vc_debug_mamba_prefill_scratch_bytes.restype = C.c_size_t
_lib.vc_debug_mamba_prefill.argtypes = [C.POINTER(VcConfig), C.POINTER(VcLayerWeights), _p, _i, _p, _p, _p, _p, _p,
                                        _p]
_lib.vc_destroy.argtypes = [_p]
_lib.vc_destroy.restype = None
_lib.vc_status_string.argtypes = [_i]
_lib.vc_status_string.restype = C.c_char_p
_lib.vc_last_cuda_error.argtypes = []
_lib.vc_last_cuda_error.restype = C.c_char_p
for _f in ("vc_quantize_weight", "vc_pack_bf16_weight", "vc_pack_weight", "vc_debug_dequant", "vc_backbone_create",
           "vc_set_option", "vc_step", "vc_step_fused", "vc_step_host", "vc_prefill", "vc_debug_set_taps",
           "vc_debug_set_prefill_taps", "vc_debug_set_zx_taps", "vc_debug_mamba_step",
           "vc_debug_gemv", "vc_debug_gemm", "vc_debug_mamba_prefill", "vc_debug_gemv_noalloc",
           "vc_gemv_noalloc_status", "vc_gemv_noalloc_reset"):
    getattr(_lib, _f).restype = _i

EXPORTS = ("vc_weight_bytes", "vc_quantize_weight", "vc_pack_bf16_weight", "vc_pack_weight", "vc_debug_dequant",
           "vc_workspace_bytes", "vc_backbone_create", "vc_set_option", "vc_uses_frame_kernel", "vc_step", "vc_step_fused", "vc_step_host",
           "vc_prefill",
           "vc_debug_set_taps", "vc_debug_set_prefill_taps", "vc_debug_set_zx_taps", "vc_debug_mamba_step",
           "vc_gemv_scratch_bytes",
           "vc_debug_gemv", "vc_debug_gemm", "vc_gemv_noalloc_scratch_bytes", "vc_debug_gemv_noalloc",
           "vc_gemv_noalloc_status", "vc_gemv_noalloc_reset",
           "vc_debug_mamba_prefill_scratch_bytes", "vc_debug_mamba_prefill", "vc_destroy",
           "vc_status_string", "vc_last_cuda_error")


class VcError(RuntimeError):
    def __init__(self, code, where):
        msg = _lib.vc_status_string(code).decode()
        if code == VC_ERR_CUDA:
            msg += ": " + _lib.vc_last_cuda_error().decode()
        super().__init__(f"{where}: {msg}")
        self.code = code


def _check(code, where):
    if code != VC_OK:
        raise VcError(code, where)


def lib():
    return _lib


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


# ------------------------------------------------------------------------------------------------
# weight preparation
# ------------------------------------------------------------------------------------------------

def weight_bytes(fmt: int, group: int, N: int, K: int) -> int:
    return int(_lib.vc_weight_bytes(fmt, group, N, K))


def qmat(buf, fmt, group, N, K) -> VcQmat:
    return VcQmat(buf.data_ptr(), fmt, group, N, K)


def quantize_weight(w, fmt: int, group: int, out=None, stream=None):
    """w: fp32 CUDA tensor [N][K] -> uint8 CUDA tensor in the device layout."""
    import torch
    N, K = w.shape
    assert w.dtype == torch.float32 and w.is_cuda and w.is_contiguous()
    if out is None:
        out = torch.empty(weight_bytes(fmt, group, N, K), dtype=torch.uint8, device=w.device)
    _check(_lib.vc_quantize_weight(fmt, group, N, K, _ptr(w), _ptr(out), _stream(stream)), "vc_quantize_weight")
    return out


def pack_bf16_weight(w, out=None, stream=None):
    """w: bf16 CUDA tensor [N][K] -> device layout."""
    import torch
    N, K = w.shape
    assert w.dtype == torch.bfloat16 and w.is_cuda and w.is_contiguous()
    if out is None:
        out = torch.empty(weight_bytes(W_BF16, 64, N, K), dtype=torch.uint8, device=w.device)
    _check(_lib.vc_pack_bf16_weight(N, K, _ptr(w), _ptr(out), _stream(stream)), "vc_pack_bf16_weight")
    return out


def pack_weight(fmt, group, N, K, q, scales, zeros=None, out=None, stream=None):
    """GPTQ-style packed codes (CUDA int32 tensors) -> device layout."""
    import torch
    if out is None:
        out = torch.empty(weight_bytes(fmt, group, N, K), dtype=torch.uint8, device=q.device)
    _check(_lib.vc_pack_weight(fmt, group, N, K, _ptr(q), _ptr(scales), _ptr(zeros), _ptr(out), _stream(stream)),
           "vc_pack_weight")
    return out


def debug_dequant(buf, fmt, group, N, K, stream=None):
    import torch
    out = torch.empty((N, K), dtype=torch.float32, device=buf.device)
    m = qmat(buf, fmt, group, N, K)
    _check(_lib.vc_debug_dequant(C.byref(m), _ptr(out), _stream(stream)), "vc_debug_dequant")
    return out


# ------------------------------------------------------------------------------------------------
# backbone
# ------------------------------------------------------------------------------------------------

def make_config(cfg, max_batch: int, kv_capacity: int, n_slots: int) -> VcConfig:
    """cfg: any object with the vc_config field names (e.g. synth.Config)."""
    c = VcConfig()
    c._pattern = cfg.pattern.encode()
    c.pattern = c._pattern
    for f in ("d_model", "ssm_heads", "ssm_head_dim", "ssm_state", "ssm_groups", "conv_width", "norm_groups",
              "attn_q_heads", "attn_kv_heads", "attn_head_dim", "mlp_hidden", "vocab_text", "vocab_func",
              "wfmt", "group_size", "head_fmt"):
        setattr(c, f, int(getattr(cfg, f)))
    c.eps = float(cfg.eps)
    c.max_batch, c.kv_capacity, c.n_slots = max_batch, kv_capacity, n_slots
    return c


def workspace_bytes(c: VcConfig) -> int:
    return int(_lib.vc_workspace_bytes(C.byref(c)))


def gemv_scratch(device="cuda"):
    import torch
    return torch.zeros(int(_lib.vc_gemv_scratch_bytes()), dtype=torch.uint8, device=device)


def debug_gemv(wbuf, fmt, group, N, K, act, scratch, out=None, stream=None):
    """y[B][N] = W act^T with the step's GEMV kernel; act: 16-bit CUDA tensor [B][act_ld]"""
    import torch
    B, act_ld = act.shape
    if out is None:
        out = torch.empty((B, N), dtype=torch.float32, device=act.device)
    m = qmat(wbuf, fmt, group, N, K)
    _check(_lib.vc_debug_gemv(C.byref(m), _ptr(act), act_ld, B, _ptr(out), _ptr(scratch), _stream(stream)),
           "vc_debug_gemv")
    return out


def gemv_noalloc_status(stream=None) -> int:
    """VC_DEV_* bits the no-allocation GEMV's launches left in its static status word"""
    v = C.c_int32(0)
    _check(_lib.vc_gemv_noalloc_status(C.byref(v), _stream(stream)), "vc_gemv_noalloc_status")
    return int(v.value)


def gemv_noalloc_reset(stream=None):
    """zero the no-allocation GEMV's static counters and status word"""
    _check(_lib.vc_gemv_noalloc_reset(_stream(stream)), "vc_gemv_noalloc_reset")


def debug_gemv_noalloc(wbuf, fmt, group, N, K, act, out=None, stream=None):
    """as debug_gemv, with the library's static scratch (no scratch argument, nothing allocated
    by the library)"""
    import torch
    B, act_ld = act.shape
    if out is None:
        out = torch.empty((B, N), dtype=torch.float32, device=act.device)
    m = qmat(wbuf, fmt, group, N, K)
    _check(_lib.vc_debug_gemv_noalloc(C.byref(m), _ptr(act), act_ld, B, _ptr(out), _stream(stream)),
           "vc_debug_gemv_noalloc")
    return out


def debug_gemm(A, W, status, out=None, stream=None):
    """out[M][N] = A W^T (fp32) with the prefill's tensor-core GEMM; A [M][K] and W [N][K] are bf16 or
    fp16 CUDA tensors (same dtype; row strides multiples of 8 elements)."""
    import torch
    M, K = A.shape
    N = W.shape[0]
    assert W.shape[1] == K and A.dtype == W.dtype and A.dtype in (torch.bfloat16, torch.float16)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    _check(_lib.vc_debug_gemm(_ptr(A), A.stride(0), M, _ptr(W), W.stride(0), N, K, int(A.dtype == torch.float16),
                              _ptr(out), out.stride(0), _ptr(status), _stream(stream)), "vc_debug_gemm")
    return out


def debug_mamba_prefill(cfg_c: VcConfig, layer: VcLayerWeights, zx, ssm, conv, y, act, stream=None):
    """the prefill's Mamba-2 mixer over T = zx.shape[0] frames from an empty state"""
    import torch
    T = zx.shape[0]
    nbytes = _lib.vc_debug_mamba_prefill_scratch_bytes(C.byref(cfg_c), T)
    if nbytes == 0:
        raise VcError(VC_ERR_INVALID_ARG, "vc_debug_mamba_prefill_scratch_bytes")
    scratch = torch.empty((nbytes,), dtype=torch.uint8, device=zx.device)
    _check(_lib.vc_debug_mamba_prefill(C.byref(cfg_c), C.byref(layer), _ptr(zx), T, _ptr(ssm), _ptr(conv), _ptr(y),
                                       _ptr(act), _ptr(scratch), _stream(stream)), "vc_debug_mamba_prefill")


def debug_mamba_step(cfg_c: VcConfig, layer: VcLayerWeights, zx, slots, ssm, conv, ctx_len, act, parts, status,
                     stream=None):
    B = zx.shape[0]
    _check(_lib.vc_debug_mamba_step(C.byref(cfg_c), C.byref(layer), _ptr(zx), B, _ptr(slots), _ptr(ssm), _ptr(conv),
                                    _ptr(ctx_len), _ptr(act), _ptr(parts), _ptr(status), _stream(stream)),
           "vc_debug_mamba_step")


class State:
    """Session state tensors (see vc_state in vc.h)."""

    def __init__(self, cfg, n_slots: int, kv_capacity: int, device="cuda"):
        import torch
        nm, na = max(cfg.pattern.count("M"), 1), max(cfg.pattern.count("*"), 1)
        H, P, N = cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state
        Cx = H * P + 2 * cfg.ssm_groups * N
        self.ssm = torch.zeros((nm, n_slots, H, P, N), dtype=torch.float32, device=device)
        self.conv = torch.zeros((nm, n_slots, cfg.conv_width, Cx), dtype=torch.bfloat16, device=device)
        self.k = torch.zeros((na, n_slots, cfg.attn_kv_heads, kv_capacity, cfg.attn_head_dim), dtype=torch.bfloat16,
                             device=device)
        self.v = torch.zeros_like(self.k)
        self.ctx_len = torch.zeros((n_slots,), dtype=torch.int32, device=device)
        self.status = torch.zeros((1,), dtype=torch.int32, device=device)
        self.c = VcState(self.ssm.data_ptr(), self.conv.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                         self.ctx_len.data_ptr(), self.status.data_ptr())


class Backbone:
    """Handle over vc_backbone_create / vc_step / vc_prefill / vc_destroy."""

    def __init__(self, cfg, weights: VcWeights, max_batch: int, kv_capacity: int, n_slots: int, device="cuda",
                 keepalive=None, stream=None):
        import torch
        self.cfg = cfg
        self.c = make_config(cfg, max_batch, kv_capacity, n_slots)
        nbytes = workspace_bytes(self.c)
        if nbytes == 0:
            raise VcError(VC_ERR_INVALID_ARG, "vc_workspace_bytes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.weights = weights
        self.keepalive = keepalive
        h = C.c_void_p()
        _check(_lib.vc_backbone_create(C.byref(self.c), C.byref(weights), _ptr(self.workspace), nbytes,
                                       _stream(stream), C.byref(h)), "vc_backbone_create")
        self.h = h
        self.max_batch, self.kv_capacity, self.n_slots = max_batch, kv_capacity, n_slots

    def set_option(self, option: int, value: int):
        _check(_lib.vc_set_option(self.h, option, value), "vc_set_option")

    def uses_frame_kernel(self, B: int) -> bool:
        """whether a step of B rows runs as one launch of the frame kernel"""
        return bool(_lib.vc_uses_frame_kernel(self.h, B))

    def set_taps(self, hidden=None, logits=None):
        self._taps = (hidden, logits)
        _check(_lib.vc_debug_set_taps(self.h, _ptr(hidden), _ptr(logits)), "vc_debug_set_taps")

    def set_zx_taps(self, zx=None):
        """fp32 [n_mamba][B][E+Cx+H]: each Mamba-2 layer's in_proj output before its bf16 rounding"""
        self._ztaps = zx
        _check(_lib.vc_debug_set_zx_taps(self.h, _ptr(zx)), "vc_debug_set_zx_taps")

    def set_prefill_taps(self, hidden=None, zx=None):
        """hidden fp32 [n_layers+1][T][d]; zx bf16 [n_mamba][T][E+Cx+H] (each Mamba-2 layer's in_proj output)"""
        self._ptaps = (hidden, zx)
        _check(_lib.vc_debug_set_prefill_taps(self.h, _ptr(hidden), _ptr(zx)), "vc_debug_set_prefill_taps")

    def step(self, x, state: State, tok_text, tok_func, slots=None, stream=None):
        B = x.shape[0]
        _check(_lib.vc_step(self.h, _ptr(x), B, _ptr(slots), C.byref(state.c), _ptr(tok_text), _ptr(tok_func),
                            _stream(stream)), "vc_step")

    def step_fused(self, speech, emb_text, emb_func, state: State, tok_text, tok_func, slots=None, stream=None):
        """one frame with its input fused on the device: speech + emb_text[tok_text] + emb_func[tok_func]
        (the previous frame's tokens, read from and then overwritten in tok_text / tok_func)"""
        B = speech.shape[0]
        emb = VcTokenEmbeddings(_ptr(emb_text), _ptr(emb_func))
        self._emb = (emb_text, emb_func)
        _check(_lib.vc_step_fused(self.h, _ptr(speech), C.byref(emb), B, _ptr(slots), C.byref(state.c),
                                  _ptr(tok_text), _ptr(tok_func), _stream(stream)), "vc_step_fused")

    def step_host(self, x_host, state: State, tok_text_host, tok_func_host, slots=None, stream=None):
        B = x_host.shape[0]
        _check(_lib.vc_step_host(self.h, _ptr(x_host), B, _ptr(slots), C.byref(state.c), _ptr(tok_text_host),
                                 _ptr(tok_func_host), _stream(stream)), "vc_step_host")

    def prefill(self, x, slot: int, state: State, stream=None):
        T = x.shape[0]
        _check(_lib.vc_prefill(self.h, _ptr(x), T, slot, C.byref(state.c), _stream(stream)), "vc_prefill")

    def close(self):
        if getattr(self, "h", None):
            _lib.vc_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
