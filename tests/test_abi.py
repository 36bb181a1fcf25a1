"""The C-ABI library loads on a machine without a GPU and exports every function vc.h declares;
host-side argument validation (no device work) rejects bad shapes before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "vc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vc_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for f in ("vc_backbone_create", "vc_prefill", "vc_step", "vc_destroy"):
        assert f in names


def test_library_exports_every_declared_symbol():
    import attention_frame_decode_b200 as vc
    lib = vc.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(vc.EXPORTS) <= set(declared_functions())


def test_weight_bytes_and_workspace_host_only():
    import attention_frame_decode_b200 as vc
    import synth
    assert vc.weight_bytes(vc.W_INT4_ASYM, 64, 22656, 4480) > 0
    # W4 g64 rows of 16: 16*64 weights -> 512 B of codes + 40 B of metadata per 16-row slab and group
    assert vc.weight_bytes(vc.W_INT4_ASYM, 64, 64, 64) == 4 * 512 + 4 * 40
    assert vc.weight_bytes(vc.W_BF16, 64, 32, 64) == 32 * 64 * 2
    assert vc.weight_bytes(7, 64, 16, 64) == 0
    assert vc.weight_bytes(vc.W_INT8_SYM, 32, 16, 64) == 0      # unsupported group size
    cfg = synth.nano_config()
    c = vc.make_config(cfg, 1, 3000, 1)
    assert vc.workspace_bytes(c) > 0
    bad = synth.nano_config(d_model=4470)
    assert vc.workspace_bytes(vc.make_config(bad, 1, 3000, 1)) == 0
    c17 = vc.make_config(cfg, 17, 3000, 17)
    assert vc.workspace_bytes(c17) == 0


def test_create_rejects_bad_arguments_without_a_gpu():
    import attention_frame_decode_b200 as vc
    import synth
    cfg = synth.tiny_config()
    c = vc.make_config(cfg, 1, 128, 1)
    h = ctypes.c_void_p()
    w = vc.VcWeights()
    # NULL weights / workspace: rejected on the host, before any CUDA call
    rc = vc.lib().vc_backbone_create(ctypes.byref(c), None, None, 0, None, ctypes.byref(h))
    assert rc == vc.VC_ERR_INVALID_ARG
    rc = vc.lib().vc_backbone_create(ctypes.byref(c), ctypes.byref(w), None, 0, None, ctypes.byref(h))
    assert rc == vc.VC_ERR_INVALID_ARG
    assert vc.lib().vc_step(None, None, 1, None, None, None, None, None) == vc.VC_ERR_INVALID_ARG
    assert vc.lib().vc_prefill(None, None, 4, 0, None, None) == vc.VC_ERR_INVALID_ARG
    assert vc.lib().vc_status_string(vc.VC_ERR_CAPACITY) == b"capacity exceeded"
