"""The C ABI library on the host: it loads, exports every declared symbol,
computes the budget count, and rejects bad arguments before launching
anything (CPU only: every call below carries at least one invalid argument,
so no kernel is ever launched and the placeholder pointers are never used).
"""
import ctypes
import os
import re

import pytest
import torch

import token_level_dynamic_seq_b200 as logo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "logo.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "num_selected.txt")

# Placeholder device addresses: aligned, never dereferenced (each call fails validation first).
FAKE = ctypes.c_void_p(1 << 20)
FAKE2 = ctypes.c_void_p(2 << 20)

no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="placeholder pointers are only passed where no GPU exists")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LOGO_API\s+[^;]*?\b(logo_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = logo.load_library()
    names = declared_symbols()
    assert len(names) == 22, names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(logo.EXPORTED)


def test_num_selected_matches_golden_table():
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        r, n, k = line.split()[:3]
        assert logo.num_selected(float(r), int(n)) == int(k), line


def test_num_selected_edge_values():
    assert logo.num_selected(float("nan"), 10) == 0
    assert logo.num_selected(-0.5, 10) == 0
    assert logo.num_selected(2.0, 10) == 10
    assert logo.num_selected(0.5, -3) == 0


def test_status_strings():
    lib = logo.load_library()
    for code, name in logo._STATUS.items():
        assert lib.logo_status_string(code).decode() == name


def shape(B=1, Hq=4, Hkv=2, L=256, d=128, cu=None, nseq=1, max_seqlen=256):
    return logo.Shape(B, Hq, Hkv, L, d, cu, nseq, max_seqlen)


def test_workspace_size():
    lib = logo.load_library()
    assert lib.logo_workspace_size(ctypes.byref(shape()), 0.2) >= 256
    assert lib.logo_workspace_size(ctypes.byref(shape(d=96)), 0.2) == 0
    assert lib.logo_workspace_size(ctypes.byref(shape()), 1.5) == 0
    assert lib.logo_workspace_size(None, 0.2) == 0


def local(lib, sh, window=16, scale=0.0, q=FAKE, k=FAKE, v=FAKE, out=FAKE2, ws=FAKE, ws_bytes=256):
    return lib.logo_local_attn(q, k, v, ctypes.byref(sh) if sh is not None else None, window, scale, out, ws,
                               ws_bytes, None)


@no_gpu_only
@pytest.mark.parametrize("case,expect", [
    (dict(sh=shape(d=96)), 2),
    (dict(sh=shape(d=80)), 2),
    (dict(sh=shape(Hq=6, Hkv=4)), 1),
    (dict(sh=shape(Hkv=0)), 1),
    (dict(sh=shape(B=0)), 1),
    (dict(sh=shape(L=-1)), 1),
    (dict(sh=None), 1),
    (dict(sh=shape(), window=0), 1),
    (dict(sh=shape(), scale=float("nan")), 1),
    (dict(sh=shape(), scale=float("inf")), 1),
    (dict(sh=shape(), ws=None), 3),
    (dict(sh=shape(), ws_bytes=16), 3),
    (dict(sh=shape(), ws=ctypes.c_void_p((1 << 20) + 8)), 3),
    (dict(sh=shape(), q=None), 1),
    (dict(sh=shape(), out=ctypes.c_void_p((2 << 20) + 2)), 1),
    (dict(sh=shape(B=2, cu=0x1000, nseq=2)), 1),          # varlen needs B == 1
    (dict(sh=shape(cu=0x1000, nseq=0)), 1),
    (dict(sh=shape(cu=0x1000, nseq=2, max_seqlen=300)), 1),  # max_seqlen > T
])
def test_local_attn_rejects(case, expect):
    lib = logo.load_library()
    assert local(lib, **case) == expect
    assert lib.logo_last_error().decode() != ""


@no_gpu_only
def test_select_and_forward_reject():
    lib = logo.load_library()
    sh = shape()
    by = ctypes.byref(sh)
    # ratio outside [0, 1]
    assert lib.logo_select(FAKE, by, 1.5, FAKE, FAKE, FAKE, 256, None) == 1
    assert lib.logo_select(FAKE, by, float("nan"), FAKE, FAKE, FAKE, 256, None) == 1
    # missing cu_sel
    assert lib.logo_select(FAKE, by, 0.2, FAKE, None, FAKE, 256, None) == 1
    # workspace too small
    assert lib.logo_select(FAKE, by, 0.2, FAKE, FAKE, FAKE, 8, None) == 3
    # forward: bad window, bad ratio, null gate, bad d
    assert lib.logo_forward(FAKE, FAKE, FAKE, FAKE, by, 0, 0.2, 0.0, FAKE2, FAKE, FAKE, FAKE, 256, None) == 1
    assert lib.logo_forward(FAKE, FAKE, FAKE, FAKE, by, 8, -0.1, 0.0, FAKE2, FAKE, FAKE, FAKE, 256, None) == 1
    assert lib.logo_forward(FAKE, FAKE, FAKE, None, by, 8, 0.2, 0.0, FAKE2, FAKE, FAKE, FAKE, 256, None) == 1
    sh96 = shape(d=96)
    assert lib.logo_forward(FAKE, FAKE, FAKE, FAKE, ctypes.byref(sh96), 8, 0.2, 0.0, FAKE2, FAKE, FAKE, FAKE, 256,
                            None) == 2
    # global: max_selected beyond the sequence length, null sel_idx
    assert lib.logo_global_attn_sparse(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, by, 257, 0.0, 1, FAKE2, FAKE, 256,
                                       None) == 1
    assert lib.logo_global_attn_sparse(FAKE, FAKE, FAKE, FAKE, None, FAKE, by, 64, 0.0, 1, FAKE2, FAKE, 256,
                                       None) == 1
    # selftest: bad limits
    assert lib.logo_selftest_timeout(FAKE, 256, 0, None) == 1
    assert lib.logo_selftest_timeout(None, 256, 10, None) == 3


@no_gpu_only
def test_training_entry_points_reject():
    lib = logo.load_library()
    sh = shape()
    by = ctypes.byref(sh)
    assert lib.logo_backward_workspace_size(by, 64) > 256
    assert lib.logo_backward_workspace_size(by, -1) == 0
    assert lib.logo_backward_workspace_size(ctypes.byref(shape(d=96)), 64) == 0
    ft = lambda **kw: lib.logo_forward_train(
        FAKE, FAKE, FAKE, FAKE, kw.get("by", by), kw.get("window", 8), kw.get("ratio", 0.2), 0.0, FAKE2, FAKE, FAKE,
        kw.get("cap", 64), kw.get("lse", FAKE), FAKE, FAKE, FAKE, FAKE, 256, None)
    assert ft(window=0) == 1
    assert ft(ratio=1.5) == 1
    assert ft(cap=-1) == 1
    assert ft(cap=10) == 1          # below one sequence's count (52 of 256)
    assert ft(lse=None) == 1
    assert ft(by=ctypes.byref(shape(d=96))) == 2
    need = lib.logo_backward_workspace_size(by, 64)
    bw = lambda **kw: lib.logo_backward(
        FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("dout", FAKE), FAKE, FAKE, kw.get("cap", 64), kw.get("max_sel", 52),
        FAKE, FAKE, FAKE, FAKE, by, kw.get("window", 8), 0.0, FAKE2, FAKE2, FAKE2, FAKE2, FAKE,
        kw.get("ws_bytes", need),
        None)
    assert bw(window=0) == 1
    assert bw(max_sel=65) == 1      # above the capacity
    assert bw(max_sel=-1) == 1
    assert bw(ws_bytes=need - 1) == 3
    assert bw(dout=None) == 1
    assert lib.logo_last_error().decode() != ""


def test_host_forward_entry_rejects():
    """The host-buffer forward validates its arguments before touching the device."""
    lib = logo.load_library()
    sh = shape()
    by = ctypes.byref(sh)
    need = lib.logo_forward_host_buffer_size(by, 0.2)
    # arena = workspace + gate + selection + three slots of one kv-head group's Q, O, K, V
    assert need > 3 * 2 * (sh.B * (sh.Hq // sh.Hkv) * sh.L * sh.d * 2)
    assert lib.logo_forward_host_buffer_size(ctypes.byref(shape(d=96)), 0.2) == 0
    assert lib.logo_forward_host_buffer_size(by, 1.5) == 0
    fh = lambda **kw: lib.logo_forward_host(
        FAKE, FAKE, FAKE, kw.get("gate", FAKE), kw.get("by", by), kw.get("window", 8), kw.get("ratio", 0.2), 0.0,
        FAKE2, None, None, kw.get("buf", FAKE), kw.get("nbytes", need), None)
    assert fh(window=0) == 1
    assert fh(ratio=-0.5) == 1
    assert fh(by=ctypes.byref(shape(d=96))) == 2
    assert fh(buf=None) == 3
    assert fh(nbytes=need - 1) == 3
    assert fh(gate=None) == 1
