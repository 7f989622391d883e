"""The C-ABI library loads, exports every symbol include/fa.h declares, and its host-side
argument validation rejects bad calls before any launch (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest

import tiled_exact_attention_fwd_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"FA_API\s+[^;(]*?\b(fa_\w+)\s*\(", text)
    return names


@pytest.fixture(scope="module")
def lib():
    from tiled_exact_attention_fwd_b200 import build
    build.build()
    return fa.lib()


def test_header_declares_the_boundary():
    names = set(_declared_symbols())
    for required in ("fa_fwd", "fa_varlen_fwd", "fa_unpad", "fa_pad"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in fa.STATUS.items():
        assert lib.fa_status_string(code).decode().startswith(name)
    assert b"unknown" in lib.fa_status_string(12345)
    assert b"sm_100a" in lib.fa_version()


# Host-side validation returns before any CUDA call, so it is exercised here without a GPU.
FAKE = 1 << 20  # a 16-byte aligned non-null address that is never dereferenced


def test_fwd_rejects_null(lib):
    assert lib.fa_fwd(None, FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 0.0, 0, 0, None) == -1
    assert lib.fa_fwd(FAKE, FAKE, FAKE, None, None, 1, 1, 128, 64, 0.0, 0, 0, None) == -1


def test_fwd_rejects_head_dim_dtype_shape_align(lib):
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 128, 96, 0.0, 0, 0, None) == -4
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 0.0, 0, 7, None) == -3
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, None, 0, 1, 128, 64, 0.0, 0, 0, None) == -2
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, None, 1, 0, 128, 64, 0.0, 0, 0, None) == -2
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, None, 1, 1, -5, 64, 0.0, 0, 0, None) == -2
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, None, 70000, 1, 128, 64, 0.0, 0, 0, None) == -2
    assert lib.fa_fwd(FAKE + 8, FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 0.0, 0, 0, None) == -5
    assert lib.fa_fwd(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 1, 1, 128, 64, 0.0, 0, 0, None) == -5


def test_varlen_validation(lib):
    # empty problems are a successful no-op
    assert lib.fa_varlen_fwd(None, None, None, None, 0, 0, 0, None, None, 4, 64, 0.0, 0, 1, None) == 0
    assert lib.fa_varlen_fwd(FAKE, FAKE, FAKE, FAKE, 3, 0, 10, FAKE, None, 4, 64, 0.0, 0, 1, None) == -2
    assert lib.fa_varlen_fwd(FAKE, FAKE, FAKE, None, 3, 8, 10, FAKE, None, 4, 64, 0.0, 0, 1, None) == -1
    assert lib.fa_varlen_fwd(FAKE, FAKE, FAKE, FAKE, 3, 8, 10, FAKE, None, 4, 48, 0.0, 0, 1, None) == -4
    assert lib.fa_varlen_fwd(FAKE, FAKE, FAKE, FAKE + 2, 3, 8, 10, FAKE, None, 4, 64, 0.0, 0, 1, None) == -5


def test_pad_unpad_validation(lib):
    assert lib.fa_unpad(None, None, 0, 10, 64, None, None) == 0
    assert lib.fa_unpad(FAKE, None, 4, 10, 64, FAKE, None) == -1
    assert lib.fa_unpad(FAKE, FAKE, -1, 10, 64, FAKE, None) == -2
    assert lib.fa_unpad(FAKE, FAKE + 4, 4, 10, 64, FAKE, None) == -5
    assert lib.fa_pad(FAKE, FAKE, 11, 10, 64, FAKE, None) == -2
    assert lib.fa_pad(None, None, 0, 0, 64, None, None) == 0
    assert lib.fa_pad(FAKE, FAKE, 4, 10, 0, FAKE, None) == -2
    assert lib.fa_pad(FAKE, FAKE, 4, 10, 64, None, None) == -1


def test_selftest_rejects_bad_limit(lib):
    assert lib.fa_selftest_bounded_wait(0, None) == -2


def test_fused_varlen_validation(lib):
    # all padding, nothing to attend: out is zero-filled (needs a device), here only shape checks
    assert lib.fa_varlen_fwd_padded(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 10, 5, FAKE, None, 2, 64, 0.0, 0, 1, None) == -2
    assert lib.fa_varlen_fwd_padded(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 10, 20, None, None, 2, 64, 0.0, 0, 1, None) == -1
    assert lib.fa_varlen_fwd_padded(FAKE, FAKE, FAKE, None, FAKE, 2, 8, 10, 20, FAKE, None, 2, 64, 0.0, 0, 1, None) == -1
    assert lib.fa_varlen_fwd_padded(FAKE, FAKE, FAKE, FAKE + 4, FAKE, 2, 8, 10, 20, FAKE, None, 2, 64, 0.0, 0, 1, None) == -5
    assert lib.fa_varlen_fwd_padded(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 10, 20, FAKE, None, 2, 48, 0.0, 0, 1, None) == -4
    assert lib.fa_varlen_fwd_padded(None, None, None, None, None, 0, 0, 0, 0, None, None, 2, 64, 0.0, 0, 1, None) == 0


def test_paged_validation(lib):
    f = lib.fa_fwd_paged
    # q, k_cache, v_cache, table, max_blocks, page_size, num_pages, out, lse, B, H, S, D, scale, causal, dtype
    ok = [FAKE, FAKE, FAKE, FAKE, 3, 64, 10, FAKE, None, 2, 4, 130, 128, 0.0, 0, 1, None]

    def call(**kw):
        a = list(ok)
        names = ["q", "k", "v", "table", "max_blocks", "page", "pages", "out", "lse", "B", "H", "S", "D",
                 "scale", "causal", "dtype", "stream"]
        for n, val in kw.items():
            a[names.index(n)] = val
        return f(*a)

    assert call(table=None) == -1
    assert call(out=None) == -1
    assert call(D=96) == -4
    assert call(dtype=5) == -3
    for bad_page in (0, 8, 24, 48, 96, 200, 384):
        assert call(page=bad_page) == -2, bad_page
    assert call(max_blocks=2) == -2          # 2 * 64 < 130 keys
    assert call(pages=0) == -2
    assert call(pages=1 << 26, page=64) == -2  # pool rows past 2^31
    assert call(table=FAKE + 2) == -5
    assert call(q=FAKE + 8) == -5
    assert call(B=0) == -2


def test_bwd_validation(lib):
    f = lib.fa_bwd
    # q, k, v, out, dout, lse, dq, dk, dv, delta, B, H, S, D, scale, causal, dtype, stream
    ok = [FAKE] * 10 + [2, 4, 130, 128, 0.0, 1, 1, None]

    def call(i=None, val=None):
        a = list(ok)
        if i is not None:
            a[i] = val
        return f(*a)

    for i in range(10):
        assert call(i, None) == -1, i
    assert call(13, 48) == -4
    assert call(13, 96) == -4
    assert call(16, 3) == -3
    assert call(10, 0) == -2
    assert call(12, 0) == -2
    assert call(0, FAKE + 8) == -5
    assert call(5, FAKE + 2) == -5
    assert call(9, FAKE + 2) == -5


def test_varlen_bwd_validation(lib):
    f = lib.fa_varlen_bwd
    # q, k, v, out, dout, lse, cu, num_seqs, max_seqlen, total, dq, dk, dv, delta, H, D, scale, causal, dtype, st
    ok = [FAKE] * 7 + [3, 64, 100] + [FAKE] * 4 + [2, 64, 0.0, 1, 1, None]

    def call(i=None, val=None):
        a = list(ok)
        if i is not None:
            a[i] = val
        return f(*a)

    assert call(9, 0) == 0      # no tokens: nothing to do
    assert call(6, None) == -1
    assert call(15, 48) == -4
    assert call(8, 0) == -2
    assert call(6, FAKE + 2) == -5
    assert call(18, 4) == -3


# The Python binding checks every caller-given buffer before the library sees it (the C entry
# points take sizes from q alone, so a smaller output would be written past its end).
def test_binding_rejects_wrong_output_shapes():
    import torch
    q = torch.zeros((1, 8, 2, 64), dtype=torch.bfloat16)
    lse = torch.zeros((1, 2, 8), dtype=torch.float32)
    good = torch.zeros_like(q)
    small = torch.zeros((1, 4, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="dq"):
        fa.fa_bwd_noalloc(q, q, q, q, q, lse, small, good, good)
    with pytest.raises(ValueError, match="dv"):
        fa.fa_bwd_noalloc(q, q, q, q, q, lse, good, good, good.float())
    with pytest.raises(ValueError, match="lse"):
        fa.fa_bwd_noalloc(q, q, q, q, q, lse[:, :1], good, good, good)
    with pytest.raises(ValueError, match="shape and dtype"):
        fa.fa_bwd_noalloc(q, small, q, q, q, lse, good, good, good)
    with pytest.raises(ValueError, match="dk"):
        fa.fa_bwd(q, q, q, q, q, lse, dk=small)
    with pytest.raises(ValueError, match="delta"):
        fa.fa_bwd(q, q, q, q, q, lse, delta=lse[:, :, :4])
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fa.fa_bwd_noalloc(q, q, q, q, q, lse, good, good, good)
