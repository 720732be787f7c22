"""Source-level rules of the library, checked as text on the CPU.

* No TMA or bulk copy with cluster multicast anywhere in the CUDA sources:
  every CTA fetches its own tiles.
* No batched async memcpy call (the four batched copy entry points of the
  runtime and driver APIs) in any source; copies are one call each.
* The product path (package, bench step, C sources) does not import the
  oracle, and nothing imports Triton: the kernels are the CUDA in csrc/.
The forbidden names are assembled from pieces so that this file does not
spell them out itself.
"""

import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "flashattention_attention_attn_b200")


def _files(*dirs, exts=(".py", ".cu", ".cuh", ".h", ".c", ".cpp", ".sh")):
    for d in dirs:
        for base, subdirs, names in os.walk(d):
            subdirs[:] = [s for s in subdirs if not s.startswith((".", "_build", "__pycache__"))]
            for n in names:
                if n.endswith(exts):
                    yield os.path.join(base, n)


def _sources():
    yield from _files(PKG, os.path.join(ROOT, "include"), os.path.join(ROOT, "oracle"), os.path.join(ROOT, "tests"))
    for n in ("bench.py", "__graft_entry__.py"):
        yield os.path.join(ROOT, n)


def _read(path):
    with open(path, encoding="utf-8", errors="replace") as f:
        return f.read()


def test_no_cluster_multicast_copies():
    token = "." + "multicast" + "::" + "cluster"
    bad = [p for p in _sources() if token in _read(p)]
    assert not bad, bad


def test_no_batched_memcpy_calls():
    names = [a + "Memcpy" + b + "BatchAsync" for a in ("cuda", "cu") for b in ("", "3D")]
    bad = [(p, n) for p in _sources() for n in names if n in _read(p)]
    assert not bad, bad


def test_product_path_does_not_use_the_oracle_or_triton():
    imp = re.compile(r"^\s*(from|import)\s+(oracle|triton)\b", re.M)
    product = list(_files(PKG))
    bad = [p for p in product if imp.search(_read(p))]
    assert not bad, bad
    # bench.py reaches the oracle only from its CPU-baseline / reference leg
    # (the CpuSample class, which both use)
    bench = _read(os.path.join(ROOT, "bench.py"))
    for m in re.finditer(r"^\s*(from oracle|import oracle)", bench, re.M):
        line = bench[: m.start()].count("\n") + 1
        # the enclosing top-level definition (a line that starts in column 0)
        tops = re.findall(r"^(def \w+|class \w+)", bench[: m.start()], re.M)
        assert tops and tops[-1] in ("class CpuSample", "def run_reference"), (line, tops[-1:])
