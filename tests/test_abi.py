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
              "attn_read_device_status", "paged_attn_decode_partial", "attn_lse_merge"):
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


def _varlen(lib, ptrs=(1 << 20,) * 7, B=2, max_q=64, total_q=100, total_k=100, Hq=8, Hkv=2, d=128, scale=0.088):
    q, k, v, o, lse, cq, ck = ptrs
    return lib.attn_fwd_varlen(q, k, v, o, lse, cq, ck, B, max_q, total_q, total_k, Hq, Hkv, d, 1,
                               ctypes.c_float(scale), None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=(None,) + (1 << 20,) * 6), INVALID),          # q
    (dict(ptrs=(1 << 20,) * 5 + (None, 1 << 20)), INVALID),  # cu_seqlens_q
    (dict(ptrs=(1 << 20, None) + (1 << 20,) * 5), INVALID),  # k with keys present
    (dict(total_k=-1), INVALID),
    (dict(Hkv=3), INVALID),
    (dict(scale=-1.0), INVALID),
    (dict(d=256), UNSUPPORTED),
    (dict(ptrs=(1 << 20,) * 5 + (2 + (1 << 20), 1 << 20)), UNSUPPORTED),  # cu_seqlens_q not 4-byte aligned
    (dict(ptrs=(1 << 20,) * 4 + (1 + (1 << 20),) + (1 << 20,) * 2), UNSUPPORTED),  # lse not 4-byte aligned
    (dict(B=0), OK),
    (dict(total_q=0), OK),
    (dict(max_q=0), OK),
])
def test_attn_fwd_varlen_host_validation(lib, kw, expect):
    assert _varlen(lib, **kw) == expect


def _chunked(lib, ptrs=(1 << 20,) * 8, B=2, Hq=8, Hkv=2, d=128, bs=16, maxb=8, max_q=32, total_q=40, scale=0.088):
    q, kc, vc, bt, sl, cq, o, lse = ptrs
    return lib.paged_attn_prefill(q, kc, vc, bt, sl, cq, B, Hq, Hkv, d, bs, maxb, max_q, total_q, 1,
                                  ctypes.c_float(scale), o, lse, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=(1 << 20,) * 3 + (None,) + (1 << 20,) * 4), INVALID),  # block_table
    (dict(ptrs=(1 << 20,) * 6 + (None, 1 << 20)), INVALID),           # o
    (dict(maxb=0), INVALID),
    (dict(Hq=9), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(bs=8), UNSUPPORTED),
    (dict(d=32), UNSUPPORTED),
    (dict(ptrs=(1 << 20, 8 + (1 << 20)) + (1 << 20,) * 6), UNSUPPORTED),  # k_cache not 16-byte aligned
    (dict(B=0), OK),
    (dict(total_q=0), OK),
])
def test_paged_prefill_host_validation(lib, kw, expect):
    assert _chunked(lib, **kw) == expect


def _partial(lib, ptrs=(1 << 20,) * 7, B=2, Hq=32, Hkv=8, d=128, bs=16, maxb=8, nblk=64, splits=0):
    q, kc, vc, bt, sl, op, lp = ptrs
    return lib.paged_attn_decode_partial(q, kc, vc, bt, sl, B, Hq, Hkv, d, bs, maxb, nblk, splits, op, lp, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=(1 << 20,) * 5 + (None, 1 << 20)), INVALID),  # o_part
    (dict(ptrs=(1 << 20,) * 6 + (None,)), INVALID),          # lse_part
    (dict(ptrs=(None,) + (1 << 20,) * 6), INVALID),          # q
    (dict(nblk=0), INVALID),
    (dict(Hkv=6), INVALID),
    (dict(d=96), UNSUPPORTED),
    (dict(bs=8), UNSUPPORTED),
    (dict(ptrs=(1 << 20,) * 5 + (8 + (1 << 20), 1 << 20)), UNSUPPORTED),  # o_part not 16-byte aligned
    (dict(ptrs=(1 << 20,) * 6 + (2 + (1 << 20),)), UNSUPPORTED),          # lse_part not 4-byte aligned
    (dict(B=0), OK),
])
def test_paged_decode_partial_host_validation(lib, kw, expect):
    assert _partial(lib, **kw) == expect


def _merge(lib, ptrs=(1 << 20,) * 3, R=2, B=2, Hq=8, d=128):
    po, pl, o = ptrs
    return lib.attn_lse_merge(po, pl, R, B, Hq, d, o, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(R=0), INVALID),
    (dict(Hq=0), INVALID),
    (dict(B=-1), INVALID),
    (dict(ptrs=(1 << 20, None, 1 << 20)), INVALID),
    (dict(ptrs=(1 << 20, 1 << 20, None)), INVALID),
    (dict(d=32), UNSUPPORTED),
    (dict(R=70000), UNSUPPORTED),
    (dict(ptrs=(4 + (1 << 20), 1 << 20, 1 << 20)), UNSUPPORTED),  # o_parts not 16-byte aligned
    (dict(B=0), OK),
])
def test_lse_merge_host_validation(lib, kw, expect):
    assert _merge(lib, **kw) == expect


def _fp8(lib, ptrs=(1 << 20,) * 6, B=2, Hq=32, Hkv=8, d=128, bs=16, maxb=8, splits=0, ks=0.5, vs=2.0):
    q, kc, vc, bt, sl, o = ptrs
    return lib.paged_attn_decode_fp8(q, kc, vc, bt, sl, B, Hq, Hkv, d, bs, maxb, splits, ctypes.c_float(ks),
                                     ctypes.c_float(vs), o, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=(1 << 20,) * 4 + (None, 1 << 20)), INVALID),  # seq_lens
    (dict(ks=0.0), INVALID),
    (dict(vs=float("inf")), INVALID),
    (dict(maxb=-1), INVALID),
    (dict(d=64), UNSUPPORTED),       # the FP8 path is built for d = 128
    (dict(bs=32), UNSUPPORTED),
    (dict(Hq=80, Hkv=8), UNSUPPORTED),  # group of 10 query heads > 8
    (dict(B=0), OK),
])
def test_paged_decode_fp8_host_validation(lib, kw, expect):
    assert _fp8(lib, **kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(ptrs=(16, 16, None, 16, 16, 16)), INVALID),
    (dict(Hkv=5), INVALID),
    (dict(d=80), UNSUPPORTED),
    (dict(B=0), OK),
])
def test_paged_decode_noalloc_host_validation(lib, kw, expect):
    ptrs = kw.pop("ptrs", (1 << 20,) * 6)
    args = dict(B=2, Hq=32, Hkv=8, d=128, bs=16, maxb=8, splits=0)
    args.update(kw)
    q, kc, vc, bt, sl, o = ptrs
    rc = lib.paged_attn_decode_noalloc(q, kc, vc, bt, sl, args["B"], args["Hq"], args["Hkv"], args["d"], args["bs"],
                                       args["maxb"], args["splits"], o, None)
    assert rc == expect


def _dec_checked(lib, ptrs=(1 << 20,) * 6, B=2, Hq=32, Hkv=8, d=128, bs=16, maxb=8, nblocks=100, splits=0):
    q, kc, vc, bt, sl, o = ptrs
    return lib.paged_attn_decode_checked(q, kc, vc, bt, sl, B, Hq, Hkv, d, bs, maxb, nblocks, splits, o, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(nblocks=0), INVALID),                    # a pool needs at least one block
    (dict(nblocks=-4), INVALID),
    (dict(nblocks=1 << 27), UNSUPPORTED),          # token coordinates must fit in int32
    (dict(maxb=1 << 27), UNSUPPORTED),
    (dict(ptrs=(16, 16, None, 16, 16, 16)), INVALID),
    (dict(d=80), UNSUPPORTED),
    (dict(B=0, nblocks=0), OK),                    # empty batch: nothing to check
])
def test_paged_decode_checked_host_validation(lib, kw, expect):
    assert _dec_checked(lib, **kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(nblocks=0), INVALID),
    (dict(nblocks=1 << 27), UNSUPPORTED),
    (dict(ks=-1.0), INVALID),
    (dict(d=64), UNSUPPORTED),
])
def test_paged_decode_fp8_checked_host_validation(lib, kw, expect):
    a = dict(ptrs=(1 << 20,) * 6, B=2, Hq=32, Hkv=8, d=128, bs=16, maxb=8, nblocks=100, splits=0, ks=0.5, vs=2.0)
    a.update(kw)
    q, kc, vc, bt, sl, o = a["ptrs"]
    rc = lib.paged_attn_decode_fp8_checked(q, kc, vc, bt, sl, a["B"], a["Hq"], a["Hkv"], a["d"], a["bs"], a["maxb"],
                                           a["nblocks"], a["splits"], ctypes.c_float(a["ks"]),
                                           ctypes.c_float(a["vs"]), o, None)
    assert rc == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(nblocks=0), INVALID),
    (dict(nblocks=1 << 27), UNSUPPORTED),
    (dict(maxb=1 << 27), UNSUPPORTED),
    (dict(scale=0.0), INVALID),
    (dict(B=0), OK),
])
def test_paged_prefill_checked_host_validation(lib, kw, expect):
    a = dict(ptrs=(1 << 20,) * 8, B=2, Hq=8, Hkv=2, d=128, bs=16, maxb=8, nblocks=100, max_q=32, total_q=40,
             scale=0.088)
    a.update(kw)
    q, kc, vc, bt, sl, cq, o, lse = a["ptrs"]
    rc = lib.paged_attn_prefill_checked(q, kc, vc, bt, sl, cq, a["B"], a["Hq"], a["Hkv"], a["d"], a["bs"], a["maxb"],
                                        a["nblocks"], a["max_q"], a["total_q"], 1, ctypes.c_float(a["scale"]), o,
                                        lse, None)
    assert rc == expect


def test_unchecked_paged_calls_reject_tables_wider_than_int32_positions(lib):
    assert _dec(lib, maxb=1 << 27) == UNSUPPORTED
    assert _chunked(lib, maxb=1 << 27) == UNSUPPORTED
    assert _fp8(lib, maxb=1 << 27) == UNSUPPORTED


def test_no_cpu_fallback_without_device(lib):
    """Valid arguments without a usable device fail loudly (no silent CPU path)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd(lib) < 0
    assert _dec(lib) < 0
    assert _varlen(lib) < 0
    assert _chunked(lib) < 0
    assert _fp8(lib) < 0
    assert _dec_checked(lib) < 0
    assert lib.attn_check_support(0) < 0


def test_plain_c_client_compiles_links_and_runs(lib, tmp_path):
    """include/attn.h compiles as C99 and the library answers a C program."""
    import shutil
    import subprocess
    from flashattention_attention_attn_b200 import _binding
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = os.path.join(ROOT, "tests", "c_client", "abi_client.c")
    exe = str(tmp_path / "abi_client")
    libdir = os.path.dirname(_binding.library_path)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                    "-o", exe, "-L", libdir, "-lattn_b200", "-Wl,-rpath," + libdir], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "attn_check_support(0)" in r.stdout
