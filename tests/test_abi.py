"""The C-ABI library loads, exports every symbol include/bifocal.h declares, and its
host-only logic (dynamic factor, workspace sizes, argument validation that returns
before any CUDA call) behaves as documented. No compute call is made here."""
import ctypes
import os
import re

import pytest

import rope_context_extension_bifocal_b200 as bfl
from tests import pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bifocal.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n.startswith(("bifocal_", "rope_causal_"))))


@pytest.fixture(scope="module")
def lib():
    from rope_context_extension_bifocal_b200 import build
    build.build()
    return bfl.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("bifocal_prefill", "bifocal_decode", "rope_causal_prefill", "rope_causal_decode", "bifocal_factor",
                 "bifocal_prefill_workspace_size", "bifocal_decode_workspace_size", "bifocal_status_string",
                 "bifocal_last_device_error", "bifocal_build_info"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_factor_matches_golden_table(lib):
    with open(os.path.join(pins.GOLDEN, "dynamic_factor.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                L, w, G = (int(x) for x in line.split())
                assert lib.bifocal_factor(L, w) == G, (L, w)
    assert lib.bifocal_factor(10, 0) == -1
    assert lib.bifocal_factor(-1, 4) == -1


def test_status_strings(lib):
    for code in range(0, 9):
        assert isinstance(lib.bifocal_status_string(code), bytes)
    assert b"invalid" in lib.bifocal_status_string(1)
    assert b"workspace" in lib.bifocal_status_string(5)
    assert b"fp16" in lib.bifocal_status_string(7)
    assert b"block-table" in lib.bifocal_status_string(8)
    assert b"unknown" in lib.bifocal_status_string(9)
    assert b"sm_100a" in lib.bifocal_build_info()


def test_status_codes_agree_with_the_header():
    import re
    hdr = open(os.path.join(ROOT, "include", "bifocal.h")).read()
    codes = dict((m.group(1), int(m.group(2))) for m in re.finditer(r"\b(BF_ERR_[A-Z_]+) = (\d+)", hdr))
    assert codes["BF_ERR_TIMEOUT"] == bfl.STATUS_TIMEOUT
    assert codes["BF_ERR_RANGE"] == bfl.STATUS_RANGE
    assert codes["BF_ERR_INDEX"] == bfl.STATUS_INDEX


def params(**kw):
    base = dict(hq=32, hkv=8, head_dim=128, w0=4096, w_pretrained=32768, theta=1e6)
    base.update(kw)
    return bfl.make_params(**base)


def test_workspace_sizes(lib):
    p = params()
    L = 131072
    s_bf = bfl.prefill_workspace_size(bfl.DTYPE_BF16, 1, L, p)
    s_fp = bfl.prefill_workspace_size(bfl.DTYPE_FP32, 1, L, p)
    # fp16 Qo/Ql [L, 32, 128] and Ko/Kl [L, 8, 128]
    assert s_bf == 2 * (L * 32 * 128 * 2) + 2 * (L * 8 * 128 * 2)
    assert s_fp == s_bf + L * 8 * 128 * 2
    assert bfl.prefill_workspace_size(7, 1, L, p) == 0
    assert bfl.prefill_workspace_size(bfl.DTYPE_BF16, 0, L, p) == 0
    d = bfl.decode_workspace_size(131200, p)
    assert 0 < d < 64 << 20
    assert bfl.decode_workspace_size(0, p) == 0
    assert bfl.prefill_workspace_size(bfl.DTYPE_BF16, 1, 64, params(head_dim=96)) == 0


FAKE = 1 << 20  # a 256-aligned non-null address; every case below fails validation before it is used


@pytest.mark.parametrize("fn", ["bifocal_prefill", "rope_causal_prefill"])
def test_prefill_validation_before_launch(lib, fn):
    f = getattr(lib, fn)

    def call(p, q=FAKE, L=128, batch=1, dtype=0, ws=FAKE, wsb=0):
        return f(q, FAKE, FAKE, dtype, batch, L, ctypes.byref(p), FAKE, None, None, None, ws, wsb, None)

    assert call(params(), q=None) == 1
    assert call(params(), L=0) == 1
    assert call(params(), batch=0) == 1
    assert call(params(hq=30)) == 1                  # hq % hkv != 0
    assert call(params(head_dim=96)) == 2
    assert call(params(), dtype=5) == 2
    assert call(params(theta=1.0)) == 1
    assert call(params(), ws=None) == 5
    assert call(params(), wsb=100) == 5
    assert call(params(), ws=FAKE + 8, wsb=1 << 40) == 5  # misaligned workspace
    assert call(params(), q=FAKE + 2) == 1                # misaligned input
    if fn == "bifocal_prefill":
        assert call(params(w0=-1)) == 1
        assert call(params(w_pretrained=0)) == 1
        p = params()
        p.mode = 7
        assert call(p) == 1
    else:  # the comparator ignores the bifocal parameters
        assert call(params(w0=-1)) == 5


@pytest.mark.parametrize("fn", ["bifocal_decode", "rope_causal_decode"])
def test_decode_validation_before_launch(lib, fn):
    f = getattr(lib, fn)

    def call(p, L=100, cap=200, kc=FAKE, ws=FAKE, wsb=0):
        return f(FAKE, FAKE, FAKE, kc, FAKE, cap, L, ctypes.byref(p), FAKE, None, ws, wsb, None)

    assert call(params(), kc=None) == 1
    assert call(params(), L=0) == 1
    assert call(params(), L=201) == 1   # L > cap
    assert call(params(hq=16, hkv=1)) == 2  # more than 8 query heads per kv head
    assert call(params(head_dim=32)) == 2
    assert call(params(), ws=None) == 5
    assert call(params(), wsb=16) == 5


def test_chunk_workspace_size(lib):
    p = params()
    P0, C = 126976, 4096
    L = P0 + C
    # fp16 Qo/Ql [C, 32, 128] and Ko/Kl [L, 8, 128]
    assert bfl.prefill_chunk_workspace_size(P0, C, p) == 2 * (C * 32 * 128 * 2) + 2 * (L * 8 * 128 * 2)
    assert bfl.prefill_chunk_workspace_size(-1, C, p) == 0
    assert bfl.prefill_chunk_workspace_size(P0, 0, p) == 0


def test_chunk_validation_before_launch(lib):
    f = lib.bifocal_prefill_chunk

    def call(p, P0=100, C=50, cap=200, kc=FAKE, ws=FAKE, wsb=1 << 30, dtype=0):
        return f(FAKE, FAKE, FAKE, dtype, P0, C, ctypes.byref(p), kc, FAKE, cap, FAKE, None, ws, wsb, None)

    assert call(params(), kc=None) == 1
    assert call(params(), P0=-1) == 1
    assert call(params(), C=0) == 1
    assert call(params(), P0=190, C=11) == 1       # P0 + C > cap
    assert call(params(head_dim=64)) == 2           # only the D = 128 ping-pong kernel takes a query offset
    assert call(params(hq=24, hkv=8)) == 2          # odd GQA group
    assert call(params(), dtype=4) == 2
    assert call(params(w0=-1)) == 1
    assert call(params(), ws=None) == 5
    assert call(params(), wsb=256) == 5


def test_window_flag_validation_before_launch(lib):
    W = bfl.FLAG_WINDOW

    def prefill(p):
        return lib.bifocal_prefill(FAKE, FAKE, FAKE, 0, 1, 128, ctypes.byref(p), FAKE, None, None, None, FAKE, 0, None)

    def decode(p):
        return lib.bifocal_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 200, 100, ctypes.byref(p), FAKE, None, FAKE, 0, None)

    assert prefill(params(w0=0, flags=W)) == 1             # an empty window
    assert prefill(params(w0=64, head_dim=64, flags=W)) == 2  # the window runs on the D = 128 ping-pong kernel
    assert prefill(params(w0=64, hq=24, flags=W)) == 2      # odd GQA group
    assert prefill(params(w0=64, flags=W)) == 5             # valid: stops at the (empty) workspace
    assert decode(params(w0=0, flags=W)) == 1
    assert decode(params(w0=64, flags=W)) == 5


def test_qknorm_validation_before_launch(lib):
    f = lib.bifocal_prefill_rope_qknorm

    def call(p, qw=FAKE, kw=FAKE, eps=1e-6, ws=FAKE, wsb=0):
        return f(FAKE, FAKE, FAKE, 0, 1, 128, ctypes.byref(p), qw, kw, ctypes.c_float(eps), None, None, ws, wsb, None)

    assert call(params(), qw=None) == 1
    assert call(params(), kw=None) == 1
    assert call(params(), eps=-1.0) == 1
    assert call(params(), eps=float("nan")) == 1
    assert call(params(), qw=FAKE + 2) == 1  # misaligned weights
    assert call(params()) == 5               # valid: stops at the (empty) workspace


def test_paged_decode_validation_before_launch(lib):
    f = lib.bifocal_decode_paged

    def call(p, pages=100, page=32, table=FAKE, max_pages=10, lens=FAKE, max_len=300, batch=2, ws=FAKE, wsb=0):
        return f(FAKE, FAKE, FAKE, FAKE, FAKE, pages, page, table, max_pages, lens, max_len, batch, ctypes.byref(p),
                 FAKE, None, ws, wsb, None)

    assert call(params(), table=None) == 1
    assert call(params(), lens=None) == 1
    assert call(params(), batch=0) == 1
    assert call(params(), page=24) == 1          # not a multiple of 16
    assert call(params(), max_pages=9) == 1      # 9 * 32 < 300
    assert call(params(flags=bfl.FLAG_WINDOW)) == 2
    assert call(params()) == 5                   # valid: stops at the (empty) workspace
    assert bfl.decode_paged_workspace_size(2, 300, params()) > 0
    assert bfl.decode_paged_workspace_size(0, 300, params()) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    mod = importlib.import_module("rope_context_extension_bifocal_b200")
    monkeypatch.setattr(mod, "_LIB", None)
    monkeypatch.setattr(mod, "lib_path", lambda: str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        mod.bifocal_factor(10, 4)
