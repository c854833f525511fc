"""Boundary checks that need no GPU: the library loads, exports every entry
point the header declares, sizes its buffers correctly, and rejects bad
arguments on the host before any launch."""
import ctypes
import math
import os
import re
import subprocess
import sys

import pytest

from sparse_long_context_ffd_b200 import ffd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ffd.h")
PKG = os.path.join(ROOT, "sparse_long_context_ffd_b200")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ffd_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = ffd.load_library()
    declared = _declared_functions()
    assert sorted(ffd.EXPORTED) == declared
    out = subprocess.run(["nm", "-D", "--defined-only", ffd.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (ffd_\w+)", out))
    assert set(declared) <= exported
    for name in declared:
        assert getattr(lib, name) is not None


def test_build_targets_sm100a():
    from sparse_long_context_ffd_b200 import build
    assert build.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "--use_fast_math" not in build.NVCC_FLAGS  # the selector needs IEEE fp32


def test_abi_version_and_status_strings():
    assert ffd.abi_version() == 2
    assert ffd.status_string(ffd.FFD_OK) == "ok"
    for code in range(1, 7):
        assert ffd.status_string(code) not in ("ok", "unknown status")
    assert ffd.status_string(99) == "unknown status"


@pytest.mark.parametrize("B,Hq,Hkv,cap,T,S", [
    (1, 4, 1, 4096, 64, 16), (4, 32, 8, 32768, 64, 32), (1, 32, 8, 131072, 64, 64),
    (1, 32, 8, 262144, 128, 64), (16, 32, 8, 65536, 64, 32), (3, 8, 8, 640, 64, 3)])
def test_buffer_sizes(B, Hq, Hkv, cap, T, S):
    s = ffd.make_shape(B, Hq, Hkv, cap, T, S)
    assert ffd.packed_bytes(s) == B * Hkv * cap * 64
    assert ffd.scale_bytes(s) == B * Hkv * (cap // T) * 128 * 2
    assert ffd.mask_words(s) == B * Hkv * math.ceil(cap // T / 32)
    assert ffd.thumb_bytes(s) == B * Hkv * cap * 32
    assert ffd.residual_bytes(s) == B * Hkv * cap * 128
    nsplit = math.ceil(cap // T / S)
    # CTAs per split (documented with ffd_decode_workspace_bytes): the largest
    # power of two up to 8 and up to S for which B * Hkv * nsplit * R <= 296
    R = 1
    while R < 8 and 2 * R <= S and B * Hkv * nsplit * 2 * R <= 296:
        R *= 2
    assert R == {(1, 4096): 8, (4, 32768): 1, (1, 131072): 1, (1, 262144): 1, (16, 65536): 1,
                 (3, 640): 2}[(B, cap)]
    partials = B * Hkv * nsplit * R * (Hq // Hkv) * 132 * 4
    ws = ffd.decode_workspace_bytes(s)
    assert ws >= partials + B * Hkv * 4 + 4 and ws % 256 == 0
    assert ws <= partials + 4 * 256 + B * Hkv * 4 + B * Hkv * nsplit * math.ceil(S / 32) * 4


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, ffd.FFD_ERR_UNSUPPORTED), ("head_dim", 0, ffd.FFD_ERR_INVALID_ARG),
    ("block_size", 32, ffd.FFD_ERR_UNSUPPORTED), ("block_size", -1, ffd.FFD_ERR_INVALID_ARG),
    ("capacity", 4000, ffd.FFD_ERR_INVALID_ARG), ("capacity", -64, ffd.FFD_ERR_INVALID_ARG),
    ("split_blocks", 0, ffd.FFD_ERR_INVALID_ARG), ("split_blocks", 513, ffd.FFD_ERR_UNSUPPORTED),
    ("num_q_heads", 12, ffd.FFD_ERR_UNSUPPORTED), ("num_q_heads", 6, ffd.FFD_ERR_INVALID_ARG),
    ("num_kv_heads", 0, ffd.FFD_ERR_INVALID_ARG), ("batch", -1, ffd.FFD_ERR_INVALID_ARG),
])
def test_bad_shapes_rejected_on_host(field, value, status):
    s = ffd.make_shape(2, 16, 4, 4096, 64, 16)
    setattr(s, field, value)
    lib = ffd.load_library()
    assert ffd.packed_bytes(s) == 0 and ffd.decode_workspace_bytes(s) == 0
    fake = 1 << 20  # never dereferenced: the shape check fails first
    rc = lib.ffd_decode(ctypes.byref(s), fake, fake, fake, fake, fake, fake, 1.0, fake, fake, fake,
                        1 << 30, None)
    assert rc == status
    rc = lib.ffd_quantize_keys(ctypes.byref(s), fake, fake, 0, fake, fake, None)
    assert rc == status


def test_bad_arguments_rejected_on_host():
    lib = ffd.load_library()
    s = ffd.make_shape(2, 16, 4, 4096, 64, 16)
    ws = ffd.decode_workspace_bytes(s)
    a = 1 << 20  # 16-byte aligned, never dereferenced on these paths

    def dec(q=a, k=a, v=a, p=a, sc=a, ln=a, delta=1.0, out=a, mask=a, w=a, wb=ws):
        return lib.ffd_decode(ctypes.byref(s), q, k, v, p, sc, ln, delta, out, mask, w, wb, None)

    assert dec(delta=float("nan")) == ffd.FFD_ERR_INVALID_ARG
    assert dec(delta=-0.5) == ffd.FFD_ERR_INVALID_ARG
    assert dec(w=None) == ffd.FFD_ERR_WORKSPACE
    assert dec(wb=ws - 1) == ffd.FFD_ERR_WORKSPACE
    for name in ("q", "k", "v", "ln", "out", "mask"):
        assert dec(**{name: None}) == ffd.FFD_ERR_INVALID_ARG, name
        assert dec(**{name: a + 2}) == ffd.FFD_ERR_INVALID_ARG, name
    assert dec(p=None) == ffd.FFD_ERR_INVALID_ARG  # the scan needs the packed keys
    assert dec(sc=a + 8) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_quantize_keys(ctypes.byref(s), a, a, -2, a, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_quantize_keys(ctypes.byref(s), None, a, 0, a, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_quantize_keys(ctypes.byref(s), a, a, 0, a + 4, a, None) == ffd.FFD_ERR_INVALID_ARG
    # block_begin past the last block and an empty batch are no-ops
    assert lib.ffd_quantize_keys(ctypes.byref(s), a, a, 64, a, a, None) == ffd.FFD_OK
    s0 = ffd.make_shape(0, 16, 4, 4096, 64, 16)
    assert lib.ffd_quantize_keys(ctypes.byref(s0), None, None, 0, None, None, None) == ffd.FFD_OK
    assert lib.ffd_decode(ctypes.byref(s0), None, None, None, None, None, None, 1.0, None, None,
                          a, 1 << 20, None) == ffd.FFD_OK
    assert lib.ffd_workspace_init(ctypes.byref(s), a, ws - 1, None) == ffd.FFD_ERR_WORKSPACE
    assert lib.ffd_check_device_status(None, None, None) == ffd.FFD_ERR_INVALID_ARG
    # the fused step writes the int4 copy, so it needs it even in dense mode
    assert lib.ffd_decode_step(ctypes.byref(s), a, a, a, None, a, a, float("inf"), a, a, a, ws,
                               None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_decode_step(ctypes.byref(s), a, a, a, a, a, a, -1.0, a, a, a, ws,
                               None) == ffd.FFD_ERR_INVALID_ARG
    for bad in (ffd.DecodeOptions(3, 0), ffd.DecodeOptions(-1, 0), ffd.DecodeOptions(0, 2),
                ffd.DecodeOptions(0, 0, -1)):
        assert lib.ffd_decode_ex(ctypes.byref(s), ctypes.byref(bad), a, a, a, a, a, a, 1.0, a, a,
                                 a, ws, None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_decode_ex(ctypes.byref(s), None, a, a, a, a, a, a, 1.0, a, a, a, ws,
                             None) == ffd.FFD_ERR_INVALID_ARG


def test_thumb_resid_arguments_rejected_on_host():
    lib = ffd.load_library()
    s = ffd.make_shape(2, 16, 4, 4096, 64, 16)
    ws = ffd.decode_workspace_bytes(s)
    a = 1 << 20
    run = ffd.DecodeOptions(0, 0)
    step = ffd.DecodeOptions(0, 1)

    def dec(opt=run, q=a, k=a, v=a, th=a, re=a, sc=a, ln=a, delta=1.0, out=a, mask=a, w=a, wb=ws):
        o = None if opt is None else ctypes.byref(opt)
        return lib.ffd_decode_tr(ctypes.byref(s), o, q, k, v, th, re, sc, ln, delta, out, mask, w,
                                 wb, None)

    assert dec(opt=None) == ffd.FFD_ERR_INVALID_ARG
    assert dec(opt=ffd.DecodeOptions(0, 3)) == ffd.FFD_ERR_INVALID_ARG
    assert dec(delta=float("nan")) == ffd.FFD_ERR_INVALID_ARG
    assert dec(wb=ws - 1) == ffd.FFD_ERR_WORKSPACE
    for name in ("q", "v", "th", "re", "sc", "ln", "out", "mask"):
        assert dec(**{name: None}) == ffd.FFD_ERR_INVALID_ARG, name
        assert dec(**{name: a + 2}) == ffd.FFD_ERR_INVALID_ARG, name
    # the computer reconstructs keys from thumbnails and residuals, so they are
    # needed in dense mode too; bf16 K only when the last block is re-quantised
    assert dec(th=None, delta=float("inf")) == ffd.FFD_ERR_INVALID_ARG
    assert dec(opt=step, k=None) == ffd.FFD_ERR_INVALID_ARG
    assert dec(opt=step, k=a + 8) == ffd.FFD_ERR_INVALID_ARG
    q = lib.ffd_quantize_keys_tr
    assert q(ctypes.byref(s), a, a, 0, a, None, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert q(ctypes.byref(s), a, a, 0, a, a + 4, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert q(ctypes.byref(s), a, a, -2, a, a, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert q(ctypes.byref(s), a, a, 64, a, a, a, None) == ffd.FFD_OK  # past the last block
    s_bad = ffd.make_shape(2, 16, 4, 4096, 32, 16)
    assert q(ctypes.byref(s_bad), a, a, 0, a, a, a, None) == ffd.FFD_ERR_UNSUPPORTED
    assert ffd.thumb_bytes(s_bad) == 0 and ffd.residual_bytes(s_bad) == 0
    # context shards: both pseudo-max modes are rejected as for the int4 format
    for ref in (ffd.FFD_REFERENCE_SINK_LOCAL, ffd.FFD_REFERENCE_SINK_LOCAL_FIXED):
        sink = ffd.DecodeOptions(ref, 0)
        assert lib.ffd_decode_partials_tr(ctypes.byref(s), ctypes.byref(sink), a, a, a, a, a, a, a,
                                          1.0, a, ws, None) == ffd.FFD_ERR_UNSUPPORTED


def test_reference_codes_match_the_oracle_numbering():
    # the parity tests pass FFD_REFERENCE_* straight to the oracle
    import oracle
    assert ffd.FFD_REFERENCE_RUNNING_MAX == oracle.RUNNING_MAX == 0
    assert ffd.FFD_REFERENCE_SINK_LOCAL == oracle.PSEUDO_MAX_SEEDED == 1
    assert ffd.FFD_REFERENCE_SINK_LOCAL_FIXED == oracle.PSEUDO_MAX_FIXED == 2
    header = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                               "include", "ffd.h")).read()
    assert "#define FFD_REFERENCE_SINK_LOCAL_FIXED 2" in header


def test_append_arguments_rejected_on_host():
    lib = ffd.load_library()
    s = ffd.make_shape(2, 16, 4, 4096, 64, 16)
    ws = ffd.decode_workspace_bytes(s)
    a = 1 << 20

    def app(ref=0, q=a, kn=a, vn=a, k=a, v=a, p=a, sc=a, ln=a, delta=1.0):
        return lib.ffd_decode_append(ctypes.byref(s), ref, q, kn, vn, k, v, p, sc, ln, delta, a, a,
                                     a, ws, None)

    def app_tr(kn=a, vn=a, k=a, re=a):
        return lib.ffd_decode_append_tr(ctypes.byref(s), 0, a, kn, vn, k, a, a, re, a, a, 1.0, a, a,
                                        a, ws, None)

    for name in ("kn", "vn", "k", "v", "p", "sc"):
        assert app(**{name: None}) == ffd.FFD_ERR_INVALID_ARG, name
    assert app(kn=a + 4) == ffd.FFD_ERR_INVALID_ARG and app(vn=a + 2) == ffd.FFD_ERR_INVALID_ARG
    assert app(ref=3) == ffd.FFD_ERR_INVALID_ARG and app(ref=-1) == ffd.FFD_ERR_INVALID_ARG
    assert app(delta=float("nan")) == ffd.FFD_ERR_INVALID_ARG
    # the thumbnail form needs bf16 K here: the append writes it
    assert app_tr(k=None) == ffd.FFD_ERR_INVALID_ARG
    assert app_tr(vn=None) == ffd.FFD_ERR_INVALID_ARG and app_tr(re=None) == ffd.FFD_ERR_INVALID_ARG


def test_step_graph_rejects_bad_arguments_without_capturing():
    lib = ffd.load_library()
    s = ffd.make_shape(2, 16, 4, 4096, 64, 16)
    a = 1 << 20
    out = ctypes.c_void_p(None)

    def create(fmt=0, adv=0, hin=a, din=a, hres=a, mask_off=16384, shape=s, res_ptr=None):
        return lib.ffd_step_graph_create(ctypes.byref(shape), fmt, 0, 1.0, adv, hin, din, a, a, a,
                                         a, a, a, res_ptr, hres, mask_off, a, 1 << 30,
                                         ctypes.byref(out))

    assert lib.ffd_step_graph_create(ctypes.byref(s), 0, 0, 1.0, 0, a, a, a, a, a, a, a, a, a, a,
                                     16384, a, 1 << 30, None) == ffd.FFD_ERR_INVALID_ARG
    assert create(fmt=2) == ffd.FFD_ERR_INVALID_ARG
    assert create(adv=3) == ffd.FFD_ERR_INVALID_ARG
    assert create(hin=None) == ffd.FFD_ERR_INVALID_ARG
    assert create(din=a + 8) == ffd.FFD_ERR_INVALID_ARG
    assert create(hres=a + 4) == ffd.FFD_ERR_INVALID_ARG
    assert create(mask_off=100) == ffd.FFD_ERR_INVALID_ARG      # not a multiple of 16
    assert create(mask_off=16) == ffd.FFD_ERR_INVALID_ARG       # inside the output rows
    assert create(shape=ffd.make_shape(0, 16, 4, 4096, 64, 16)) == ffd.FFD_ERR_INVALID_ARG
    assert out.value is None
    lib.ffd_step_graph_destroy(None)  # a null graph is ignored
    assert lib.ffd_step_graph_run(None) == ffd.FFD_ERR_INVALID_ARG


def test_product_path_never_touches_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, re.M), f
                assert "ffd_oracle" not in text and "ffdo_" not in text, f


def test_binding_has_no_cpu_fallback():
    import torch
    s = ffd.make_shape(1, 4, 1, 128, 64, 2)
    t = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError):
        ffd.decode(s, t, t, t, t, t, t, 1.0, t, t, t)


def test_read_probe_rejects_bad_arguments_on_host():
    lib = ffd.load_library()
    a = 1 << 20  # never dereferenced: every call below fails its host checks
    assert lib.ffd_read_probe(None, 1024, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_read_probe(a, 1024, None, None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_read_probe(a, 0, a, None) == ffd.FFD_ERR_INVALID_ARG
    assert lib.ffd_read_probe(a, 1000, a, None) == ffd.FFD_ERR_INVALID_ARG  # not a multiple of 16
    assert lib.ffd_read_probe(a + 8, 1024, a, None) == ffd.FFD_ERR_INVALID_ARG  # misaligned


def test_debug_library_switch():
    # a fresh process may switch to the bounds-checking build before its first call;
    # a process that already loaded the product library may not
    code = ("from sparse_long_context_ffd_b200 import ffd; ffd.use_debug_library(); "
            "print(ffd.library_path())")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT,
                         check=True).stdout.strip()
    assert out.endswith("libffd_b200_debug.so")
    ffd.load_library()
    with pytest.raises(RuntimeError):
        ffd.use_debug_library()
    assert ffd.library_path().endswith("libffd_b200.so")
