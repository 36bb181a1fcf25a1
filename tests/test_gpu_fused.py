"""The fused-input step (vc_step_fused): each frame's input is formed on the device from this
frame's speech embedding and the tokens the previous frame emitted, so a session runs frame after
frame without its tokens leaving the device.  Checked against the oracle running the same loop
with its own tokens (oracle.fuse_inputs + the oracle step):
  * the fused input (the residual stream entering layer 0) within one bf16 ulp of the oracle's;
  * hidden states and logits within 2e-2 x RMS per layer;
  * tokens equal wherever the oracle's top-2 margin exceeds 1e-3; a frame whose token is not
    decidable ends the comparison if the two sides took different tokens (the sessions' inputs
    then legitimately differ)."""
import numpy as np
import pytest

import oracle
import synth
from tests.test_gpu_decode import HID_TOL, MARGIN, Run, rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("graph", [1, 0])
def test_tiny_session_with_fused_inputs(cuda, graph):
    import torch
    import attention_frame_decode_b200 as vc
    cfg = synth.tiny_config()
    seed = 2
    run = Run(cfg, seed, 1, cfg.kv_capacity)
    run.bb.set_option(vc.OPT_GRAPH, graph)
    run.bb.set_taps(run.hid, run.lg)
    et, ef = synth.token_embeddings(cfg, seed)
    etd = torch.from_numpy(et).cuda().view(torch.bfloat16)
    efd = torch.from_numpy(ef).cuda().view(torch.bfloat16)
    run.tt.fill_(-1)
    run.tf.fill_(-1)
    ott, otf = np.array([-1], np.int32), np.array([-1], np.int32)
    compared = 0
    for t in range(24):
        sp = synth.frame_inputs(cfg, seed, t, 1)
        run.bb.step_fused(torch.from_numpy(sp).cuda().view(torch.bfloat16), etd, efd, run.st, run.tt, run.tf)
        torch.cuda.synchronize()
        x = oracle.fuse_inputs(sp, et, ef, ott, otf)
        ro = run.om.step(run.ost, x, oracle.MIRROR, taps=True)
        hid = run.hid.cpu().numpy()
        xo = synth.bf16_to_f32(x)[0].astype(np.float64)
        assert np.all(np.abs(hid[0, 0] - xo) <= 2.0 ** -8 * np.abs(xo)), t
        for layer in range(cfg.n_layers + 1):
            assert rel(hid[layer], ro["hidden"][layer]) < HID_TOL, (t, layer)
        lg = run.lg.cpu().numpy()
        gt, gf = int(run.tt.cpu()[0]), int(run.tf.cpu()[0])
        diverged = False
        for hsel, (g, o, V) in enumerate(((gt, int(ro["tok_text"][0]), cfg.vocab_text),
                                          (gf, int(ro["tok_func"][0]), cfg.vocab_func))):
            lo = ro["logits"][hsel, 0, :V]
            assert rel(lg[hsel, 0, :V], lo) < HID_TOL
            top2 = np.sort(lo)[-2:]
            if top2[1] - top2[0] > MARGIN:
                compared += 1
                assert g == o, (t, hsel, g, o)
            elif g != o:
                diverged = True
        if diverged:
            break
        ott, otf = ro["tok_text"].astype(np.int32), ro["tok_func"].astype(np.int32)
    assert compared >= 8
    assert int(run.st.status.cpu()[0]) == 0


def test_fused_step_rejects_missing_tables(cuda):
    import torch
    import attention_frame_decode_b200 as vc
    cfg = synth.tiny_config()
    run = Run(cfg, 3, 1, cfg.kv_capacity, taps=False)
    sp = torch.zeros((1, cfg.d_model), dtype=torch.bfloat16, device="cuda")
    emb = vc.VcTokenEmbeddings(None, None)
    rc = vc.lib().vc_step_fused(run.bb.h, sp.data_ptr(), emb, 1, None, run.st.c, run.tt.data_ptr(),
                                run.tf.data_ptr(), None)
    assert rc == vc.VC_ERR_INVALID_ARG
