"""Parity of the sm_100a prefill kernel (attn_fwd through the C ABI) with the
fp64 oracle on the same seeded inputs."""

import numpy as np
import pytest
import torch

from flashattention_attention_attn_b200 import inputs
from tests._parity import check_close, f64, oracle_prefill, run_prefill

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, T, S, d, causal, seed):
    spec = inputs.PrefillSpec(B=B, Hq=Hq, Hkv=Hkv, T=T, S=S, d=d, causal=causal, seed=seed)
    q, k, v = inputs.make_prefill(spec)
    o, lse = run_prefill(q, k, v, causal, spec.scale)
    O, L = oracle_prefill(q, k, v, causal, spec.scale)
    return check_close(f64(o), O, lse.numpy(), L, what=f"B{B} Hq{Hq} Hkv{Hkv} T{T} S{S} d{d} c{causal}")


def test_tiny_causal_workload():
    spec = inputs.WORKLOADS["tiny_causal"]
    q, k, v = inputs.make_prefill(spec)
    o, lse = run_prefill(q, k, v, True, spec.scale)
    O, L = oracle_prefill(q, k, v, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what="tiny_causal")


def test_llama3_8b_prefill_workload():
    spec = inputs.WORKLOADS["llama3_8b_prefill"]
    q, k, v = inputs.make_prefill(spec)
    o, lse = run_prefill(q, k, v, True, spec.scale)
    O, L = oracle_prefill(q, k, v, True, spec.scale)
    check_close(f64(o), O, lse.numpy(), L, what="llama3_8b_prefill")


@pytest.mark.parametrize("B,Hq,Hkv,T,S,d,causal", [
    (1, 4, 1, 128, 128, 128, True),     # one tile, GQA 4:1
    (2, 8, 2, 300, 300, 128, True),     # ragged tail, several tiles
    (1, 8, 8, 777, 777, 64, True),      # MHA, d=64, ragged
    (1, 16, 2, 200, 333, 128, True),    # T < S: bottom-right causal
    (1, 4, 2, 333, 200, 128, True),     # T > S: leading rows see no key
    (2, 8, 1, 257, 391, 128, False),    # non-causal, GQA 8:1
    (1, 2, 2, 64, 1000, 64, False),     # short query block, long keys
    (3, 4, 4, 1, 1, 128, True),         # single row, single key
    (1, 4, 2, 513, 513, 128, True),     # one row past a 256-row CTA block
])
def test_prefill_shapes(B, Hq, Hkv, T, S, d, causal):
    _case(B, Hq, Hkv, T, S, d, causal, seed=7 + T + S)


def test_no_keys_gives_zero_and_minus_inf():
    q = torch.randn(1, 5, 4, 128).to(torch.bfloat16)
    k = torch.zeros(1, 0, 2, 128, dtype=torch.bfloat16)
    o, lse = run_prefill(q, k, k, True, 0.1)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_deterministic():
    spec = inputs.PrefillSpec(B=1, Hq=8, Hkv=2, T=700, S=700, d=128, causal=True, seed=3)
    q, k, v = inputs.make_prefill(spec)
    o1, l1 = run_prefill(q, k, v, True, spec.scale)
    o2, l2 = run_prefill(q, k, v, True, spec.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_long_prefill_workload_sampled_rows():
    """T = S = 16384: the full GPU output, checked on sampled rows (all heads)
    against the oracle, plus LSE on those rows."""
    spec = inputs.WORKLOADS["long_prefill_16k"]
    q, k, v = inputs.make_prefill(spec)
    o, lse = run_prefill(q, k, v, True, spec.scale)
    rng = np.random.default_rng(0)
    rows = sorted(set(rng.integers(0, spec.T, 40).tolist()) | {0, 1, 127, 128, 255, 256, spec.T - 1})
    O, L = oracle_prefill(q, k, v, True, spec.scale, rows=rows)
    check_close(f64(o)[:, rows], O[:, rows], lse.numpy()[:, :, rows], L[:, :, rows], what="long_prefill rows")
    assert torch.isfinite(o.float()).all()


def test_long_prefill_workload_all_rows():
    """T = S = 16384: every element of O and LSE (16384 rows x 32 heads)
    against the oracle, evaluated head by head in worker processes."""
    from tests._oracle_pool import attention_by_head
    spec = inputs.WORKLOADS["long_prefill_16k"]
    q, k, v = inputs.make_prefill(spec)
    o, lse = run_prefill(q, k, v, True, spec.scale)
    O, L = attention_by_head(f64(q), f64(k), f64(v), spec.scale, True)
    check_close(f64(o), O, lse.numpy(), L, what="long_prefill all rows")
