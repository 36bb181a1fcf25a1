"""GPU parity of the prefill path (the opening context of a session consumed in one call) against
fp64 references and the CPU oracle, on the same seeded inputs.

Tolerances:
  * tensor-core GEMM, fp32 accumulation of 16-bit products: max |gpu - fp64| <= 1e-4 * RMS(fp64);
  * Mamba-2 mixer over the frames on identical bf16 inputs: final SSM state (fp32 chunk states
    and scan) within 1e-4 * RMS of the oracle's sequential recurrence; y (intra-chunk products
    on fp16, entering-state products on bf16 tensor-core operands) within one bf16 ulp of each
    element plus 2e-2 * RMS; conv ring
    bit-exact; gated-norm output within one bf16 ulp of the value exact arithmetic gives from
    the kernel's own y;
  * whole stacks: state after the prefill (SSM per head, conv rows, KV rows) and the hidden
    states / logits of the decode steps that follow within max(2e-2, 2 x floor) * RMS, floor the
    oracle's own response to 1-ulp flips in ~1% of the prefill inputs (for the bf16-stored conv
    rows and K/V, beyond one bf16 ulp of each value); greedy tokens identical where the oracle's
    top-2 logit margin exceeds 1e-3 and twice that perturbation's logit change.
"""
import numpy as np
import pytest

import oracle
import synth

GEMM_TOL = 1e-4
SSM_TOL = 1e-4
HID_TOL = 2e-2
MARGIN = 1e-3

pytestmark = pytest.mark.gpu


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b * b)), 1e-30))


def rel_heads(a, b):
    """max over SSM heads of max |a - b| / RMS(b) within the head ([H][P][N] arrays).  The state
    is heavy-tailed across heads (slowly decaying heads hold values ~50x the overall RMS), so the
    unit of scale is the head, each an independent recurrence."""
    a = np.asarray(a, np.float64).reshape(a.shape[0], -1)
    b = np.asarray(b, np.float64).reshape(b.shape[0], -1)
    rms = np.maximum(np.sqrt(np.mean(b * b, axis=1)), 1e-30)
    return float(np.max(np.max(np.abs(a - b), axis=1) / rms))


def rel_stored(a, b, ulp=2.0 ** -7):
    """as rel, for values both sides store in bf16: a rounding decision that went the other way
    (one bf16 ulp, at most 2^-7 of the value) is not counted"""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    excess = np.maximum(np.abs(a - b) - ulp * np.abs(b), 0.0)
    return float(np.max(excess) / max(np.sqrt(np.mean(b * b)), 1e-30))


# ------------------------------------------------------------------------------------------------
# the tcgen05 GEMM
# ------------------------------------------------------------------------------------------------

def _operands(M, N, K, dtype, lda=None, seed=11):
    import torch
    lda = K if lda is None else lda
    a = synth.bf16_to_f32(synth.normal_bf16(seed, 1, (M, lda)))
    w = synth.bf16_to_f32(synth.normal_bf16(seed, 2, (N, K), 0.0, 0.05))
    At = torch.from_numpy(a).cuda().to(dtype)
    Wt = torch.from_numpy(w).cuda().to(dtype)
    return At, Wt


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (129, 257, 72), (300, 520, 448), (512, 1024, 200),
                                   (128, 4480, 1024)])
@pytest.mark.parametrize("half", [False, True])
def test_gemm_matches_fp64(cuda, M, N, K, half):
    import torch
    import attention_frame_decode_b200 as vc
    dt = torch.float16 if half else torch.bfloat16
    A, W = _operands(M, N, K, dt)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    out = vc.debug_gemm(A, W, status)
    ref = A.double() @ W.double().T
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert rel(out.cpu().numpy(), ref.cpu().numpy()) < GEMM_TOL


def test_gemm_row_stride_and_two_calls(cuda):
    """A with a row stride larger than K (a column slice), called twice into the same output"""
    import torch
    import attention_frame_decode_b200 as vc
    A_wide, W = _operands(200, 384, 136, torch.bfloat16, lda=192)
    A = A_wide[:, :136]
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    out = torch.full((200, 384), float("nan"), dtype=torch.float32, device="cuda")
    vc.debug_gemm(A, W, status, out=out)
    first = out.clone()
    vc.debug_gemm(A, W, status, out=out)
    ref = A.double() @ W.double().T
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert rel(out.cpu().numpy(), ref.cpu().numpy()) < GEMM_TOL
    assert torch.equal(first, out)


@pytest.mark.parametrize("N,K", [(22656, 4480), (4480, 15680)])
def test_gemm_projection_shapes_sampled(cuda, N, K):
    """Nano projection shapes over 4096 frames; 64 sampled rows against fp64"""
    import torch
    import attention_frame_decode_b200 as vc
    M = 4096
    A, W = _operands(M, N, K, torch.bfloat16, seed=12)
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    out = vc.debug_gemm(A, W, status)
    rows = torch.arange(0, M, M // 64, device="cuda")
    ref = A[rows].double() @ W.double().T
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert rel(out[rows].cpu().numpy(), ref.cpu().numpy()) < GEMM_TOL


# ------------------------------------------------------------------------------------------------
# kernel level: the Mamba-2 mixer over the frames (chunked SSD) vs the oracle's recurrence
# ------------------------------------------------------------------------------------------------

def nano_layer_cfg(pattern, wfmt=synth.FMT_BF16, group=64, **kw):
    return synth.nano_config(name="nano_layer_" + pattern, pattern=pattern, vocab_text=2048, vocab_func=2048,
                             wfmt=wfmt, group_size=group, head_fmt=synth.FMT_BF16, **kw)


@pytest.mark.parametrize("T,tiny", [(1, False), (300, False), (777, False), (600, True)])
def test_mamba_prefill_mixer(cuda, T, tiny):
    import torch
    import attention_frame_decode_b200 as vc
    from attention_frame_decode_b200.model import DeviceModel
    from attention_frame_decode_b200.synthetic import ring_to_history
    cfg = synth.tiny_config(pattern="M") if tiny else nano_layer_cfg("M")
    small = synth.small_params(cfg, 5, 0)
    dm = DeviceModel(cfg)
    for k, v in small.items():
        dm.set_small(0, k, v)
    c = vc.make_config(cfg, 1, max(T, 64), 1)
    R = cfg.in_proj_rows
    E, Cx, W = cfg.d_inner, cfg.conv_dim, cfg.conv_width
    zx_bits = synth.normal_bf16(5, 600, (T, R), 0.0, 1.0)
    zx = torch.from_numpy(zx_bits).cuda().view(torch.bfloat16)
    ssm = torch.full((cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state), float("nan"), device="cuda")
    conv = torch.full((W, Cx), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    act = torch.zeros((T, E), dtype=torch.bfloat16, device="cuda")
    vc.debug_mamba_prefill(c, dm.layers[0], zx, ssm, conv, y, act)
    torch.cuda.synchronize()
    om = oracle.Model(cfg.replace(vocab_text=16, vocab_func=16), 5)
    S = np.zeros((cfg.ssm_heads, cfg.ssm_head_dim, cfg.ssm_state), np.float64)
    hist = np.zeros((W - 1, Cx), np.float64)
    yo, vo = om.mamba_mixer(0, synth.bf16_to_f32(zx_bits).astype(np.float64), S, hist, 0)
    assert rel(ssm.cpu().numpy(), S) < SSM_TOL
    # y: the intra-chunk products run on fp16 tensor-core operands, the entering-state product on
    # bf16 ones.  y feeds a bf16 storage point (the gated-norm output), so each element may be off
    # by one bf16 ulp of itself (2^-8) on top of the 2e-2 * RMS bound; y is heavy-tailed (max/RMS
    # ~ 27 here), and bf16 operands would exceed this bound where fp16 ones stay well inside it.
    assert rel_stored(y.cpu().numpy(), yo, ulp=2.0 ** -8) < HID_TOL
    ring = conv.view(torch.int16).cpu().numpy().view(np.uint16)
    got_hist = ring_to_history(ring, T, W)
    want_hist = np.zeros((W - 1, Cx), np.uint16)
    for i in range(W - 1):
        t = T - (W - 1) + i
        if t >= 0:
            want_hist[i] = zx_bits[t, E:E + Cx]
    assert np.array_equal(got_hist, want_hist)
    assert np.all(ring[T % W] == 0)
    # gated RMSNorm output from the kernel's own y: one bf16 rounding of the exact value (within
    # one bf16 ulp of it, 2^-8 relative, plus the fp32 arithmetic before the rounding)
    gs = E // cfg.norm_groups
    z = synth.bf16_to_f32(zx_bits[:, :E]).astype(np.float64)
    v = (y.cpu().numpy().astype(np.float64) * (z / (1.0 + np.exp(-z)))).reshape(T, cfg.norm_groups, gs)
    inv = 1.0 / np.sqrt((v * v).mean(axis=2, keepdims=True) + cfg.eps)
    ref = (v * inv).reshape(T, E) * small["gnorm"].astype(np.float64)
    got = act.float().cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * rms)


# ------------------------------------------------------------------------------------------------
# whole stacks: prefill, then decode steps, against the oracle
# ------------------------------------------------------------------------------------------------

def perturbed(x):
    x = x.copy()
    x[:, ::97] ^= 1      # last mantissa bit of ~1% of the inputs
    return x


class PrefillRun:
    """A GPU backbone and the oracle on the same synthetic model; the oracle also runs on inputs
    with 1-ulp flips in ~1% of the values, and each bound is max(2e-2, 2 x that floor): the
    in_proj outputs are bf16 storage points, and a rounding decision that goes the other way on
    a dt or B value moves the SSM state of a whole head, so two correct implementations that
    accumulate in different orders differ by about the oracle's own response to such flips."""

    def __init__(self, cfg, seed, T, cap):
        import torch
        from attention_frame_decode_b200.synthetic import build_model
        self.cfg, self.seed, self.T, self.cap = cfg, seed, T, cap
        self.dm = build_model(cfg, seed)
        self.bb = self.dm.backbone(1, cap, 1)
        self.st = self.dm.new_state(1, cap)
        self.om = oracle.Model(cfg, seed)
        self.ost = self.om.new_state(1, cap)
        self.ostp = self.om.new_state(1, cap)
        V = max(cfg.vocab_text, cfg.vocab_func)
        self.hid = torch.zeros((cfg.n_layers + 1, 1, cfg.d_model), dtype=torch.float32, device="cuda")
        self.lg = torch.zeros((2, 1, V), dtype=torch.float32, device="cuda")
        self.bb.set_taps(self.hid, self.lg)
        self.tt = torch.zeros((1,), dtype=torch.int32, device="cuda")
        self.tf = torch.zeros((1,), dtype=torch.int32, device="cuda")

    def prefill(self):
        """prefill on both sides; the residual stream of every frame after every layer within
        max(2e-2, 2 x floor) of the oracle's"""
        import torch
        cfg, T = self.cfg, self.T
        x = synth.prefill_inputs(cfg, self.seed, T)
        tap = torch.zeros((cfg.n_layers + 1, T, cfg.d_model), dtype=torch.float32, device="cuda")
        self.bb.set_prefill_taps(tap)
        self.bb.prefill(torch.from_numpy(x).cuda().view(torch.bfloat16), 0, self.st)
        torch.cuda.synchronize()
        self.bb.set_prefill_taps(None)
        ro = self.om.prefill(self.ost, 0, x, oracle.MIRROR, ssd_chunk=256, taps=True)
        rp = self.om.prefill(self.ostp, 0, perturbed(x), oracle.MIRROR, ssd_chunk=256, taps=True)
        assert ro["rc"] == 0 and rp["rc"] == 0
        hid = tap.cpu().numpy()
        self.hidden_errs = []
        for l in range(cfg.n_layers + 1):
            err, floor = rel(hid[l], ro["hidden"][l]), rel(rp["hidden"][l], ro["hidden"][l])
            self.hidden_errs.append((err, floor))
            assert err <= max(HID_TOL, 2.0 * floor), (l, err, floor)

    def check_state(self):
        from attention_frame_decode_b200.synthetic import ring_to_history
        cfg, T = self.cfg, self.T
        assert int(self.st.ctx_len.cpu().numpy()[0]) == T
        assert int(self.ost.ctx_len[0]) == T
        assert int(self.st.status.cpu()[0]) == 0
        res = {}
        for m in range(cfg.n_mamba):
            res[f"ssm{m}"] = (rel_heads(self.st.ssm[m, 0].cpu().numpy(), self.ost.ssm[m, 0]),
                              rel_heads(self.ostp.ssm[m, 0], self.ost.ssm[m, 0]))
            ring = self.st.conv[m, 0].float().cpu().numpy()
            res[f"conv{m}"] = (rel_stored(ring_to_history(ring, T, cfg.conv_width), self.ost.conv[m, 0]),
                               rel_stored(self.ostp.conv[m, 0], self.ost.conv[m, 0]))
        for a in range(cfg.n_attn):
            for nm, g, o, op in (("k", self.st.k, self.ost.k, self.ostp.k), ("v", self.st.v, self.ost.v, self.ostp.v)):
                res[f"{nm}{a}"] = (rel_stored(g[a, 0, :, :T].float().cpu().numpy(), o[a, 0, :, :T]),
                                   rel_stored(op[a, 0, :, :T], o[a, 0, :, :T]))
        bad = {k: v for k, v in res.items() if v[0] > max(HID_TOL, 2.0 * v[1])}
        assert not bad, res
        return res

    def steps(self, n):
        import torch
        compared = 0
        for i in range(n):
            x = synth.frame_inputs(self.cfg, self.seed, i, 1)
            self.bb.step(torch.from_numpy(x).cuda().view(torch.bfloat16), self.st, self.tt, self.tf)
            torch.cuda.synchronize()
            ro = self.om.step(self.ost, x, oracle.MIRROR, taps=True)
            rp = self.om.step(self.ostp, x, oracle.MIRROR, taps=True)
            hid = self.hid.cpu().numpy()
            for l in range(self.cfg.n_layers + 1):
                err, floor = rel(hid[l], ro["hidden"][l]), rel(rp["hidden"][l], ro["hidden"][l])
                assert err <= max(HID_TOL, 2.0 * floor), (i, l, err, floor)
            lg = self.lg.cpu().numpy()
            for hsel, (tg, to, V) in enumerate(((self.tt, ro["tok_text"], self.cfg.vocab_text),
                                                (self.tf, ro["tok_func"], self.cfg.vocab_func))):
                lo = ro["logits"][hsel, 0, :V]
                lp = rp["logits"][hsel, 0, :V]
                assert rel(lg[hsel, 0, :V], lo) <= max(HID_TOL, 2.0 * rel(lp, lo))
                noise = float(np.max(np.abs(lp - lo)))
                top2 = np.sort(lo)[-2:]
                if top2[1] - top2[0] > max(MARGIN, 2.0 * noise):
                    compared += 1
                    assert int(tg.cpu().numpy()[0]) == int(to[0])
        return compared


@pytest.mark.parametrize("wfmt", [synth.FMT_W8, synth.FMT_BF16])
@pytest.mark.parametrize("T", [1, 600])
def test_tiny_stack_prefill_then_decode(cuda, wfmt, T):
    cfg = synth.tiny_config(wfmt=wfmt, head_fmt=wfmt)
    run = PrefillRun(cfg, 7, T, T + 64)
    run.prefill()
    run.check_state()
    assert run.steps(8) > 0


@pytest.mark.parametrize("pattern,wfmt", [("M", synth.FMT_BF16), ("*", synth.FMT_BF16), ("-M", synth.FMT_BF16),
                                          ("M", synth.FMT_W4)])
def test_nano_layers_prefill(cuda, pattern, wfmt):
    cfg = nano_layer_cfg(pattern, wfmt=wfmt)
    run = PrefillRun(cfg, 9, 300, 364)
    run.prefill()
    run.check_state()
    run.steps(2)


def test_prefill_rejects_bad_arguments(cuda):
    import torch
    import attention_frame_decode_b200 as vc
    from attention_frame_decode_b200.synthetic import build_model
    cfg = synth.tiny_config()
    dm = build_model(cfg, 1)
    bb = dm.backbone(1, 64, 1)
    st = dm.new_state(1, 64)
    x = torch.zeros((65, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vc.VcError) as e:
        bb.prefill(x, 0, st)
    assert e.value.code == vc.VC_ERR_CAPACITY
    with pytest.raises(vc.VcError) as e:
        bb.prefill(x[:8], 1, st)
    assert e.value.code == vc.VC_ERR_INVALID_ARG
    # empty inputs: no frames to prefill, no sessions to step; and more sessions than max_batch
    with pytest.raises(vc.VcError) as e:
        bb.prefill(x[:0], 0, st)
    assert e.value.code == vc.VC_ERR_INVALID_ARG
    tt = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tf = torch.zeros((1,), dtype=torch.int32, device="cuda")
    with pytest.raises(vc.VcError) as e:
        bb.step(x[:0], st, tt, tf)
    assert e.value.code == vc.VC_ERR_INVALID_ARG
    with pytest.raises(vc.VcError) as e:
        bb.step(x[:2], st, tt, tf)
    assert e.value.code == vc.VC_ERR_INVALID_ARG
    # every rejection came before any launch: the session is untouched
    torch.cuda.synchronize()
    assert int(st.ctx_len[0]) == 0 and int(st.status[0]) == 0


def test_prefill_on_a_second_stream_while_another_session_steps(cuda):
    """A new session's opening context is prefilled into slot 1 on one stream while the session in
    slot 0 steps frame by frame on another; both end as the oracle's do."""
    import torch
    from attention_frame_decode_b200.synthetic import build_model, ring_to_history
    cfg = synth.tiny_config()
    seed, T, cap = 4, 300, 400
    dm = build_model(cfg, seed)
    bb = dm.backbone(1, cap, 2)
    st = dm.new_state(2, cap)
    om = oracle.Model(cfg, seed)
    ost = om.new_state(2, cap)
    xp = synth.prefill_inputs(cfg, seed, T)
    xpd = torch.from_numpy(xp).cuda().view(torch.bfloat16)
    xs = [synth.frame_inputs(cfg, seed, t, 1) for t in range(8)]
    xsd = [torch.from_numpy(x).cuda().view(torch.bfloat16) for x in xs]
    tt = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tf = torch.zeros_like(tt)
    slot0 = torch.zeros((1,), dtype=torch.int32, device="cuda")
    s_pf, s_dec = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s_pf):
        bb.prefill(xpd, 1, st, stream=s_pf)
    toks = []
    with torch.cuda.stream(s_dec):
        for x in xsd:
            bb.step(x, st, tt, tf, slots=slot0, stream=s_dec)
            toks.append((tt.clone(), tf.clone()))
    torch.cuda.synchronize()
    assert om.prefill(ost, 1, xp, oracle.MIRROR, ssd_chunk=256)["rc"] == 0
    for i, x in enumerate(xs):
        ro = om.step(ost, x, oracle.MIRROR, slots=[0], taps=True)
        for hsel, key, V in ((0, "tok_text", cfg.vocab_text), (1, "tok_func", cfg.vocab_func)):
            top2 = np.sort(ro["logits"][hsel, 0, :V])[-2:]
            if top2[1] - top2[0] > MARGIN:
                assert int(toks[i][hsel].cpu()[0]) == int(ro[key][0]), (i, key)
    assert st.ctx_len.cpu().numpy().tolist() == [8, T]
    assert int(st.status.cpu()[0]) == 0
    for m in range(cfg.n_mamba):
        for slot, t in ((0, 8), (1, T)):
            assert rel_heads(st.ssm[m, slot].cpu().numpy(), ost.ssm[m, slot]) < HID_TOL
            ring = st.conv[m, slot].float().cpu().numpy()
            assert rel_stored(ring_to_history(ring, t, cfg.conv_width), ost.conv[m, slot]) < HID_TOL
    for a in range(cfg.n_attn):
        for slot, t in ((0, 8), (1, T)):
            assert rel_stored(st.k[a, slot, :, :t].float().cpu().numpy(), ost.k[a, slot, :, :t]) < HID_TOL
            assert rel_stored(st.v[a, slot, :, :t].float().cpu().numpy(), ost.v[a, slot, :, :t]) < HID_TOL
