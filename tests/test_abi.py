"""C ABI checks that need no GPU: the library loads, exports every function
that include/attn.h declares, and rejects bad arguments on the host before
any CUDA call (status codes as documented in the header)."""

import ctypes
import os
import re

import pytest

from flashattention_attention_attn_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")

OK, INVALID, UNSUPPORTED = 0, -1, -2


@pytest.fixture(scope="module")
def lib():
    path = build.build()  # no-op when up to date; nvcc cross-compiles without a GPU
    from flashattention_attention_attn_b200 import _binding
    assert os.path.samefile(path, _binding.library_path)
    return _binding.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("attn_fwd", "paged_attn_decode", "attn_check_support", "attn_status_string",
              "attn_read_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in attn.h but not exported"


def test_status_strings(lib):
    for s in (OK, INVALID, UNSUPPORTED, -3, -4, 12345):
        assert isinstance(lib.attn_status_string(s), bytes)


def _fwd(lib, ptrs=(1 << 20,) * 4, B=1, Hq=32, Hkv=8, T=128, S=128, d=128, causal=1, scale=0.088):
    q, k, v, o = ptrs
    return lib.attn_fwd(q, k, v, o, None, B, Hq, Hkv, T, S, d, causal, ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=(None, 16, 16, 16)), INVALID),
    (dict(ptrs=(16, 16, 16, None)), INVALID),
    (dict(B=-1), INVALID),
    (dict(Hkv=0), INVALID),
    (dict(Hkv=7), INVALID),               # Hq % Hkv != 0
    (dict(scale=0.0), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(scale=float("inf")), INVALID),
    (dict(d=96), UNSUPPORTED),
    (dict(ptrs=(8, 16, 16, 16)), UNSUPPORTED),  # q not 16-byte aligned
    (dict(B=0), OK),                      # empty batch: nothing to do
    (dict(T=0), OK),                      # no queries: nothing to do
])
def test_attn_fwd_host_validation(lib, kw, expect):
    assert _fwd(lib, **kw) == expect


def _dec(lib, ptrs=(1 << 20,) * 6, B=2, Hq=32, Hkv=8, d=128, bs=16, maxb=8, splits=0):
    q, kc, vc, bt, sl, o = ptrs
    return lib.paged_attn_decode(q, kc, vc, bt, sl, B, Hq, Hkv, d, bs, maxb, splits, o, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=(16, 16, None, 16, 16, 16)), INVALID),
    (dict(ptrs=(16, 16, 16, None, 16, 16)), INVALID),
    (dict(maxb=0), INVALID),
    (dict(Hkv=5), INVALID),
    (dict(B=-3), INVALID),
    (dict(bs=32), UNSUPPORTED),           # only 16-token blocks
    (dict(d=80), UNSUPPORTED),
    (dict(Hq=72, Hkv=4), UNSUPPORTED),    # group of 18 query heads > 8
    (dict(ptrs=(16, 24, 16, 16, 16, 16)), UNSUPPORTED),
    (dict(B=0), OK),
])
def test_paged_decode_host_validation(lib, kw, expect):
    assert _dec(lib, **kw) == expect


def test_no_cpu_fallback_without_device(lib):
    """Valid arguments without a usable device fail loudly (no silent CPU path)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd(lib) < 0
    assert _dec(lib) < 0
    assert lib.attn_check_support(0) < 0
