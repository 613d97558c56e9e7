"""CPU checks of the C ABI boundary (no GPU, no kernel launch).

The library must load, export every entry point include/cta.h declares, plan
workspace sizes, and reject bad arguments with a status code before it
touches the device.  Every call below fails a host-side check, so none of
them reaches a CUDA call (fake pointers are never dereferenced).
"""
import ctypes
import os
import re
import subprocess

import pytest

import certified_top_sparse_b200 as cta
from certified_top_sparse_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cta.h")

FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced
ODD = ctypes.c_void_p((1 << 20) + 4)   # misaligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w[\w\s\*]*?\b(cta_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    lib = cta.load()
    names = declared_functions()
    assert set(names) == set(cta.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", cta.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    for name in names:
        assert hasattr(lib, name)
        assert re.search(rf"\bT {name}$", out, re.M), name


def test_library_is_built_for_sm100a_only():
    """The build compiles one cubin for sm_100a and embeds no PTX, so a launch
    on any other architecture fails instead of JIT-compiling something else;
    every GPU test then exercises exactly this code (checked from the build
    recipe, without inspecting the binary)."""
    from certified_top_sparse_b200 import build as cta_build
    flags = " ".join(cta_build.FLAGS)
    assert "-gencode arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1 and "code=compute_" not in flags


def test_version_and_strings():
    assert cta.cta_version() >= 100
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert cta.cta_status_string(code)
    assert cta.cta_status_string(12345) == "unknown status"


def test_opts_layout_matches_header():
    # 4 int32, 3 pointers + size_t, 5 pointers on LP64 (gap_out appended last)
    assert ctypes.sizeof(_lib.cta_opts) == 16 + 8 * 8
    assert _lib.cta_opts.gap_out.offset == 16 + 8 * 7
    o = _lib.make_opts()
    assert (o.batch, o.m, o.dtype) == (1, 1, cta.CTA_BF16)


def test_workspace_size_plans():
    # logits of every row dominate: 4 * rows * n bytes
    n, d, h, kv = 131072, 128, 32, 8
    ws = cta.cta_workspace_size(n, d, h, kv)
    assert ws >= 4 * h * n and ws < 4 * h * n * 1.6
    assert cta.cta_workspace_size(1, 64, 1, 1) > 0
    assert cta.cta_workspace_size(512, 64, 12, 12, batch=8, m=512) >= 4 * 8 * 12 * 512 * 512
    # unsupported shapes plan to 0
    assert cta.cta_workspace_size(100, 96, 8, 8) == 0
    assert cta.cta_workspace_size(100, 64, 6, 4) == 0
    assert cta.cta_workspace_size(0, 64, 8, 8) == 0
    assert cta.cta_workspace_size((1 << 28) + 1, 64, 1, 1) == 0


def _call(q=FAKE, K=FAKE, V=FAKE, n=1024, d=64, h=8, kv=8, eps=0.01, out=FAKE, k=FAKE, idx=FAKE,
          tv=FAKE, opts="default", ws_bytes=None, dtype=cta.CTA_BF16):
    lib = cta.load()
    if opts == "default":
        o = _lib.make_opts(dtype=dtype)
        o.workspace = 1 << 20
        o.workspace_bytes = 0 if ws_bytes is None else ws_bytes
        optr = ctypes.byref(o)
    else:
        optr = None
    return lib.cta_certified_topk_attn(q, K, V, n, d, h, kv, eps, out, k, idx, tv, optr)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(K=None), -1), (dict(V=None), -1), (dict(out=None), -1),
    (dict(k=None), -1), (dict(idx=None), -1), (dict(tv=None), -1),
    (dict(eps=0.0), -1), (dict(eps=1.0), -1), (dict(eps=-0.5), -1), (dict(eps=float("nan")), -1),
    (dict(opts=None), -3), (dict(dtype=7), -1), (dict(q=ODD), -1), (dict(V=ODD), -1),
    (dict(d=96), -2), (dict(h=6, kv=4), -2), (dict(n=0), -2), (dict(n=(1 << 28) + 1), -2),
    (dict(), -3),                       # workspace too small (0 bytes)
    (dict(ws_bytes=1000), -3),
])
def test_bad_arguments_rejected_before_launch(kw, code):
    assert _call(**kw) == code


def test_dense_bad_arguments():
    lib = cta.load()
    assert lib.cta_dense_attn(None, FAKE, FAKE, 10, 64, 1, 1, FAKE, None) == -1
    assert lib.cta_dense_attn(FAKE, FAKE, FAKE, 10, 80, 1, 1, FAKE, None) == -2
    assert lib.cta_dense_attn(FAKE, FAKE, FAKE, 10, 64, 3, 2, FAKE, None) == -2


def test_binding_has_no_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib.load()
