"""Host-side pieces of bench.py, checked without a GPU: the clock summary,
the per-workload traffic table and the algorithmic-work helpers it reports."""

import importlib.util
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_entries_name_known_workloads_and_kernels():
    b = _bench()
    for name, t in b.TRAFFIC.items():
        assert name in b.WORKLOAD_SETS, name
        assert set(t) <= {"prefill", "decode", "csrc"} and "csrc" in t, name
        for part in ("prefill", "decode"):
            if part in t:
                assert t[part] > 0, (name, part)


def test_traffic_applies_only_to_the_kernels_it_was_captured_on():
    b = _bench()
    h = b.csrc_hash()
    assert len(h) == 16 and h == b.csrc_hash()  # stable for the same sources
    b.TRAFFIC["long"] = {"prefill": 4.9e8, "decode": 5.4e8, "csrc": h}
    assert b.traffic_of("long", "prefill")[0] == 4.9e8
    b.TRAFFIC["long"]["csrc"] = "0" * 16  # captured on other kernels
    val, note = b.traffic_of("long", "prefill")
    assert val is None and "changed" in note
    assert b.traffic_of("no-such-set", "decode")[0] is None


def test_measured_decode_traffic_is_at_least_the_algorithmic_bytes():
    # a DRAM count below the bytes the method must read would mean a kernel
    # that skipped work (or a stale table)
    b = _bench()
    from flashattention_attention_attn_b200 import inputs, workloads
    for name, (pname, dname) in b.WORKLOAD_SETS.items():
        t = b.TRAFFIC.get(name)
        if not t or "decode" not in t:
            continue
        base, fp8 = b.decode_workload(dname)
        ds = inputs.WORKLOADS[base]
        d = inputs.make_paged(ds)
        algo = workloads.decode_bytes(d.seq_lens.tolist(), ds.Hq, ds.Hkv, ds.d, ds.block_size,
                                      kv_elem_bytes=1 if fp8 else 2)
        assert algo <= t["decode"] < 1.05 * algo, name  # K/V read once, partials small


def test_clock_summary_uses_samples_inside_the_window():
    b = _bench()
    cs = b.ClockSampler.__new__(b.ClockSampler)
    cs.samples = [(0.0, 1000, 0x0), (1.0, 1965, 0x4), (2.0, 1900, 0x0), (3.0, 1965, 0x0), (9.0, 700, 0x40)]
    cs.max_mhz = 1965
    cs.source = "test"
    s = cs.summary(0.5, 3.5)
    assert s["samples"] == 3 and s["samples_total"] == 5
    assert s["sm_mhz"] == 1965  # median of 1965, 1900, 1965
    assert s["reasons"] == ["sw_power_cap"]  # bits of the samples inside the window only
    assert "hw_thermal_slowdown" not in s["reasons"]


def test_clock_summary_without_samples_says_so():
    b = _bench()
    cs = b.ClockSampler.__new__(b.ClockSampler)
    cs.samples, cs.max_mhz, cs.source = [], None, None
    s = cs.summary(0.0, 1.0)
    assert s["sm_mhz"] is None and s["samples"] == 0 and s["reasons"]


def test_prefill_min_bytes_counts_inputs_once_and_outputs():
    from flashattention_attention_attn_b200 import workloads
    B, Hq, Hkv, T, S, d = 1, 32, 8, 16384, 16384, 128
    qo = 2 * B * T * Hq * d * 2          # Q read, O written (bf16)
    kv = 2 * B * S * Hkv * d * 2         # K and V read (bf16)
    lse = 4 * B * Hq * T
    assert workloads.prefill_min_bytes(B, Hq, Hkv, T, S, d) == qo + kv + lse
    # causal work: sum over rows of (row + 1) visible keys
    assert workloads.visible_pairs(T, S, True) == T * (T + 1) // 2
    assert math.isclose(workloads.prefill_flops(B, Hq, T, S, d, True), 4 * d * Hq * T * (T + 1) / 2)


def test_default_run_follows_the_timing_rules():
    # no flags: one GPU, >= 3 warm-up steps, the long-context pair (16k-token
    # prefill, 131k-token decode), both ops of a step concurrent, the
    # library's own split choice, end-to-end leg and CPU baseline on
    b = _bench()
    a = b.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1 and a.impl == "ours"
    assert b.WORKLOAD_SETS[a.workload] == ("long_prefill_16k", "long_decode_131k")
    assert a.streams == 2 and a.num_splits == 0
    assert a.e2e_steps > 0 and not a.no_cpu_baseline
    assert b.parse_args(["--streams", "1"]).streams == 1
