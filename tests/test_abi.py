"""The C-ABI library loads on a machine without a GPU and exports every function vc.h declares;
host-side argument validation (no device work) rejects bad shapes before any launch; vc.h
compiles as plain C99, the binding's ctypes structures have the sizes and member offsets the C
compiler gives the header's structs, every bound call's argument and return types agree with its
prototype, a plain C program links the library and calls it, and the package refuses to import
without the library."""
import ctypes
import os
import re
import shutil
import subprocess
import sys

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


def test_option_numbers_match_the_header():
    """every VC_OPT_* the header defines has the same number in the binding, and vc_set_option
    refuses a NULL handle on the host"""
    import attention_frame_decode_b200 as vc
    src = open(os.path.join(ROOT, "include", "vc.h")).read()
    opts = dict(re.findall(r"#define VC_(OPT_[A-Z_]+) (\d+)", src))
    assert set(opts) == {"OPT_GRAPH", "OPT_PDL", "OPT_FRAME", "OPT_GEMV_SHAPE"}
    for name, num in opts.items():
        assert getattr(vc, name) == int(num), name
    assert vc.lib().vc_set_option(None, vc.OPT_GEMV_SHAPE, 1) == vc.VC_ERR_INVALID_ARG


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


def test_create_refuses_shapes_the_decode_kernels_do_not_cover():
    """valid configurations outside what the mixer kernels handle are refused with
    VC_ERR_UNSUPPORTED at create time, before any CUDA call (here: no GPU at all)"""
    import attention_frame_decode_b200 as vc
    import synth
    h = ctypes.c_void_p()

    def create(cfg):
        c = vc.make_config(cfg, 1, 128, 1)
        return vc.lib().vc_backbone_create(ctypes.byref(c), None, None, 0, None, ctypes.byref(h))

    assert create(synth.tiny_config()) == vc.VC_ERR_INVALID_ARG             # supported; NULL weights
    assert create(synth.tiny_config(attn_head_dim=48)) == vc.VC_ERR_UNSUPPORTED   # 256 % 48 != 0
    assert create(synth.tiny_config(attn_head_dim=32)) == vc.VC_ERR_INVALID_ARG
    big_state = synth.tiny_config(pattern="M-", ssm_heads=64, ssm_head_dim=2, ssm_state=256)
    assert create(big_state) == vc.VC_ERR_UNSUPPORTED                        # P/2 + 2N = 513
    assert create(big_state.replace(ssm_state=252)) == vc.VC_ERR_INVALID_ARG  # 505: supported
    assert not h.value


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a host C compiler")
def test_header_is_c99_and_binding_structs_match_it(tmp_path):
    import attention_frame_decode_b200 as vc
    exe = str(tmp_path / "abi_layout")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-o", exe,
                    os.path.join(ROOT, "tests", "host", "abi_layout.c")], check=True, capture_output=True,
                   timeout=300)
    out = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60).stdout
    py = {"vc_config": vc.VcConfig, "vc_qmat": vc.VcQmat, "vc_layer_weights": vc.VcLayerWeights,
          "vc_weights": vc.VcWeights, "vc_state": vc.VcState, "vc_token_embeddings": vc.VcTokenEmbeddings}
    seen = set()
    for line in out.splitlines():
        name, value = line.split()
        if "." in name:
            struct, member = name.split(".")
            assert getattr(py[struct], member).offset == int(value), name
            seen.add(struct + "." + member)
        else:
            assert ctypes.sizeof(py[name]) == int(value), name
    # every member of every binding structure was checked
    for struct, cls in py.items():
        for field in cls._fields_:
            assert struct + "." + field[0] in seen, (struct, field[0])


def _prototypes():
    src = open(os.path.join(ROOT, "include", "vc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"#[^\n]*", "", src)
    protos = {}
    for m in re.finditer(r"([A-Za-z_][\w\s\*]*?)\b(vc_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", src):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        args = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        protos[name] = (ret, args)
    return protos


def _c_kind(decl):
    if "*" in decl or decl.startswith("vc_stream_t"):
        return "ptr"
    if decl.startswith("size_t"):
        return "size"
    if decl.startswith("float"):
        return "float"
    if re.match(r"(const\s+)?(int|int32_t|vc_status|vc_wfmt)\b", decl):
        return "int"
    raise AssertionError(decl)


def _ct_kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_float:
        return "float"
    if t is ctypes.c_int:
        return "int"
    raise AssertionError(t)


def test_binding_signatures_match_the_header():
    """each exported call's ctypes argument and return types agree with its vc.h prototype
    (pointer, int, size_t, float), so no argument is marshalled at the wrong width"""
    import attention_frame_decode_b200 as vc
    protos = _prototypes()
    for name in vc.EXPORTS:
        ret, args = protos[name]
        fn = getattr(vc.lib(), name)
        assert fn.argtypes is not None, name
        assert [_c_kind(a) for a in args] == [_ct_kind(t) for t in fn.argtypes], name
        if ret == "void":
            assert fn.restype is None, name
        elif ret.startswith("const char"):
            assert fn.restype is ctypes.c_char_p, name
        else:
            assert _c_kind(ret) == _ct_kind(fn.restype), name


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a host C compiler")
def test_plain_c_client_links_and_calls_the_library(tmp_path):
    """a C99 program that includes only vc.h links libvc.so and gets sizes and host-side
    rejections from it (no Python, no torch, no device)"""
    import attention_frame_decode_b200 as vc
    libdir = os.path.dirname(vc.LIB_PATH)
    exe = str(tmp_path / "abi_from_c")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-o", exe,
                    os.path.join(ROOT, "tests", "host", "abi_from_c.c"), "-L" + libdir, "-lvc",
                    "-Wl,-rpath," + libdir], check=True, capture_output=True, timeout=300)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout
    lines = out.stdout.splitlines()
    assert lines[-1] == "ok"
    ws = int(lines[0].split()[1])
    import synth
    cfg = synth.tiny_config()
    assert ws == vc.workspace_bytes(vc.make_config(cfg, 1, 128, 1))


def test_package_refuses_to_import_without_the_library(tmp_path):
    """no fallback: a copy of the package without libvc.so raises ImportError on import"""
    pkg = tmp_path / "attention_frame_decode_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "attention_frame_decode_b200", "__init__.py"), pkg / "__init__.py")
    code = "import attention_frame_decode_b200"
    out = subprocess.run([sys.executable, "-c", code], cwd=str(tmp_path), capture_output=True, text=True,
                         timeout=120)
    assert out.returncode != 0
    assert "ImportError" in out.stderr and "libvc.so not found" in out.stderr
