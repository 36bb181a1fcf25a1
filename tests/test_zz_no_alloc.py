"""The no-allocation GEMV entry (vc_debug_gemv_noalloc: static device scratch, no scratch
argument) against the existing entry vc_debug_gemv on the same weights and activations, and
against the CPU oracle's product on the same quantized weights (independent of the kernel).

Tolerance: the kernels accumulate in fp32 on different grids, so the stream-K split and the
summation order differ, and the oracle sums in double: max |noalloc - other| <= 1e-4 * RMS(other).
Two no-alloc calls in a row give identical results (the fixup sums partials in a fixed worker
order, and the first call leaves the static counters at zero for the second), and leave the
static status word clear.  This file is collected last, so it also runs after every other test
has used the library in the same process.
"""
import numpy as np
import pytest

import oracle
import synth

TOL = 1e-4

pytestmark = pytest.mark.gpu


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b * b)), 1e-30))


def _weight(fmt, group, N, K, seed):
    import torch
    import attention_frame_decode_b200 as vc
    w = torch.from_numpy(synth.normal_f32(seed, 1, (N, K), 0.0, 0.02)).cuda()
    if fmt == vc.W_BF16:
        return vc.pack_bf16_weight(w.to(torch.bfloat16).contiguous())
    return vc.quantize_weight(w, fmt, group)


def _oracle_product(fmt, group, N, K, seed, act, B):
    """the oracle's y = W u for each activation row, on the weights _weight quantized (the same
    RTN decisions, pinned bit-exact against the device quantizer elsewhere)"""
    w = synth.normal_f32(seed, 1, (N, K), 0.0, 0.02)
    if fmt == oracle.BF16:
        m = oracle.bf16_mat(synth.f32_to_bf16(w))
    else:
        m = oracle.quantize(fmt, group, w)
    u = act[:, :K].float().cpu().numpy().astype(np.float64)
    return np.stack([m.matvec(u[b]) for b in range(B)])


def _act(B, K, fp16, seed):
    import torch
    ld = (K + 127) // 128 * 128
    a = torch.zeros((B, ld), dtype=torch.float16 if fp16 else torch.bfloat16, device="cuda")
    a[:, :K] = torch.from_numpy(synth.bf16_to_f32(synth.normal_bf16(seed, 2, (B, K)))).cuda().to(a.dtype)
    return a


@pytest.mark.parametrize("fmt,group,N,K,B", [(0, 64, 4480, 10240, 1), (2, 64, 4480, 10240, 3),
                                             (1, 128, 15680, 4480, 16), (3, 64, 7168, 4480, 2),
                                             (0, 64, 131072, 4480, 1)])
def test_noalloc_matches_scratch_entry_twice(cuda, fmt, group, N, K, B):
    import torch
    import attention_frame_decode_b200 as vc
    wbuf = _weight(fmt, group, N, K, 21)
    act = _act(B, K, fmt != vc.W_BF16, 22)
    scratch = vc.gemv_scratch()
    ref = vc.debug_gemv(wbuf, fmt, group, N, K, act, scratch)
    first = vc.debug_gemv_noalloc(wbuf, fmt, group, N, K, act)
    second = vc.debug_gemv_noalloc(wbuf, fmt, group, N, K, act)
    torch.cuda.synchronize()
    r = ref.cpu().numpy()
    assert rel(first.cpu().numpy(), r) <= TOL
    assert rel(second.cpu().numpy(), r) <= TOL
    assert torch.equal(first, second)
    assert vc.gemv_noalloc_status() == 0
    o = _oracle_product(fmt, group, N, K, 21, act, B)
    assert rel(first.cpu().numpy(), o) <= TOL


def test_noalloc_rejects_beyond_its_limits(cuda):
    import torch
    import attention_frame_decode_b200 as vc
    assert vc.lib().vc_gemv_noalloc_scratch_bytes() == (4 << 20) + 65536 * 4 + 256
    wbuf = _weight(0, 64, 64, 128, 23)
    act = _act(1, 128, False, 24)
    # more row units than the static counters hold: refused on the host, nothing launched
    m = vc.qmat(wbuf, 0, 64, 65536 * 32 + 1, 128)
    out = torch.empty((1, 64), dtype=torch.float32, device="cuda")
    rc = vc.lib().vc_debug_gemv_noalloc(m, act.data_ptr(), act.shape[1], 1, out.data_ptr(), None)
    assert rc == vc.VC_ERR_CAPACITY
    rc = vc.lib().vc_debug_gemv_noalloc(vc.qmat(wbuf, 0, 64, 64, 128), act.data_ptr(), act.shape[1], 17,
                                        out.data_ptr(), None)
    assert rc == vc.VC_ERR_INVALID_ARG


def test_noalloc_reset_clears_the_status_and_keeps_results(cuda):
    """the reset entry (a device memset of the counters and status word) leaves the entry working"""
    import torch
    import attention_frame_decode_b200 as vc
    wbuf = _weight(2, 64, 448, 640, 25)
    act = _act(2, 640, True, 26)
    before = vc.debug_gemv_noalloc(wbuf, 2, 64, 448, 640, act)
    vc.gemv_noalloc_reset()
    after = vc.debug_gemv_noalloc(wbuf, 2, 64, 448, 640, act)
    torch.cuda.synchronize()
    assert vc.gemv_noalloc_status() == 0
    assert torch.equal(before, after)
