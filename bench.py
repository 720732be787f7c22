"""Benchmark of the fused-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input: a
causal GQA prefill and a one-token paged-KV decode.  The default step is the
long-context pair:
  * attn_fwd          causal GQA prefill, B=1, Hq=32, Hkv=8, T=S=16384, d=128
  * paged_attn_decode one-token decode of a 131072-token context through the
                      block table (8192 permuted 16-token blocks), split-KV
The metric is the fraction of the B200 roofline the step reaches: the ideal
step time is prefill FLOPs / measured bf16 tensor peak + decode bytes /
measured HBM bandwidth, and value = 100 * (sum over ranks of ideal time) /
(measured step time, max over ranks): percent of one B200's roofline,
summed over the GPUs of the job.  Each op is also timed alone (`parts`), and
`roofline` reports the dominant one (the prefill) against its own peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long|step|varlen|chunked|fp8]

`--workload step` times the Llama3-8B-shaped pair (T=S=512 prefill, B=2,
and a 64-sequence decode with contexts of 256-4096 tokens); `--workload
varlen` replaces that prefill by 16 packed sequences of U[64, 2048] tokens
(attn_fwd_varlen); `--workload chunked` by a 512-token chunk of each of 8
sequences against their paged cache of 1k-8k tokens (paged_attn_prefill);
`--workload fp8` keeps the Llama3-8B step but stores the decode cache as FP8
e4m3 (paged_attn_decode_fp8; decode bytes count 1 byte per cached element).
`--impl reference` times the fp64 CPU oracle (the only reference
implementation there is) on a bounded sample of the same step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attn TFLOP/s & paged-decode KV GB/s, % of B200 roofline"
UNIT = "% of 1xB200 roofline (summed over GPUs)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PART_MIN_MS = 20.0  # an op timed alone runs for at least this long (and at least K calls)
PART_TIMING = ("each op alone: back-to-back calls on the launching stream (at least K, and at least "
               f"{PART_MIN_MS:g} ms of them), CUDA events at the two ends, right after the timed step loop")

WORKLOAD_SETS = {
    "long": ("long_prefill_16k", "long_decode_131k"),
    "step": ("llama3_8b_prefill", "paged_decode_b64"),
    "varlen": ("varlen_prefill_16seq", "paged_decode_b64"),
    "chunked": ("chunked_prefill_paged", "paged_decode_b64"),
    "fp8": ("llama3_8b_prefill", "paged_decode_b64:fp8"),
}
DEFAULT_WORKLOAD = "long"

# DRAM bytes (read + write) per launch of each kernel of a step, from a
# one-pass ncu launch list of `bench.py --workload <set>` (dram__bytes_read.sum
# + dram__bytes_write.sum, mean over the captured launches of each kernel).
# `csrc` is the source hash (csrc_hash() below) of the kernels that were
# captured: when the kernels change, the figure no longer applies and the
# bench reports null until a new capture replaces it.
TRAFFIC = {
    # set: {"prefill": bytes per launch, "decode": bytes per call (split + combine), "csrc": hash}
    "long": {"prefill": 381.92e6, "decode": 539.75e6, "csrc": "c2db8360f1659fcb"},
    "step": {"prefill": 12.65e6, "decode": 604.99e6, "csrc": "c2db8360f1659fcb"},
    "fp8": {"prefill": 12.65e6, "decode": 306.29e6, "csrc": "c2db8360f1659fcb"},
    "varlen": {"prefill": 279.62e6, "decode": 605.21e6, "csrc": "c2db8360f1659fcb"},
    "chunked": {"prefill": 209.72e6, "decode": 605.10e6, "csrc": "c2db8360f1659fcb"},
}


def csrc_hash() -> str:
    """Hash of the CUDA sources (csrc/*.cu, *.cuh) the library is built from."""
    d = os.path.join(ROOT, "flashattention_attention_attn_b200", "csrc")
    h = hashlib.sha256()
    for n in sorted(os.listdir(d)):
        if n.endswith((".cu", ".cuh")):
            h.update(n.encode())
            with open(os.path.join(d, n), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def traffic_of(workload: str, part: str):
    """(bytes, note) for a kernel of a workload set, or (None, why not)."""
    t = TRAFFIC.get(workload)
    if not t or part not in t:
        return None, "no ncu capture of this workload"
    if t.get("csrc") != csrc_hash():
        return None, "kernels changed since the ncu capture"
    return t[part], "ncu DRAM read + write per launch, source hash %s" % t["csrc"]


def decode_workload(dname):
    """(spec name, FP8 cache?) of a decode workload name ("name" or "name:fp8")."""
    base, _, kind = dname.partition(":")
    return base, kind == "fp8"


def vars_of(spec):
    return {k: getattr(spec, k) for k in spec.__dataclass_fields__ if not k.startswith("_")}


def step_config(pname, dname, inputs, world, args, prefill_in_bytes, decode_bytes):
    """The `config` object of the JSON line; identical for both --impl arms."""
    pspec = (inputs.VARLEN_WORKLOADS.get(pname) or inputs.CHUNKED_WORKLOADS.get(pname) or inputs.WORKLOADS[pname])
    dbase, dfp8 = decode_workload(dname)
    return {"workload": f"{pname} + {dname}", "prefill": vars_of(pspec),
            "decode": {**vars_of(inputs.WORKLOADS[dbase]), "kv_cache": "fp8 e4m3" if dfp8 else "bf16"},
            "decode_num_splits": args.num_splits or "auto", "parallelism": f"replicas x{world} (no exchange)",
            "streams": ("prefill and decode concurrently on two streams (fork/join every step)"
                        if args.streams == 2 else "prefill then decode on one stream"),
            "l2": ("no flush between steps; per step the prefill moves %.0f MB (inputs read once, outputs written "
                   "once) and the decode reads %.0f MB (L2: 126 MB)" % (prefill_in_bytes / 1e6, decode_bytes / 1e6))}


class PrefillCase:
    """The prefill half of a step: dense (attn_fwd), packed (attn_fwd_varlen)
    or chunked against a paged cache (paged_attn_prefill)."""

    def __init__(self, name, seed, dev, fa, inputs, workloads):
        import torch
        self.name = name
        self.varlen = name in inputs.VARLEN_WORKLOADS
        self.chunked = name in inputs.CHUNKED_WORKLOADS
        if self.chunked:
            sp = self.spec = inputs.CHUNKED_WORKLOADS[name]
            ci = inputs.make_chunked(sp, seed=seed)
            c = ci.cache
            self.host_in = [ci.q, c.k_cache, c.v_cache, c.block_table, c.seq_lens, ci.cu_q]
            lens_q = (ci.cu_q[1:] - ci.cu_q[:-1]).tolist()
            ctx = c.seq_lens.tolist()
            self.flops = sum(workloads.prefill_flops(1, sp.Hq, t, s_, sp.d, sp.causal) for t, s_ in zip(lens_q, ctx))
            self.min_bytes = sum(workloads.prefill_min_bytes(1, sp.Hq, sp.Hkv, t, s_, sp.d) for t, s_ in zip(lens_q, ctx))
            self.max_q, self.total_q, self.max_blocks = ci.max_q, int(ci.cu_q[-1]), c.block_table.shape[1]
            self.dev_in = [t.to(dev) for t in self.host_in]
            self.o = torch.empty_like(self.dev_in[0])
            self.lse = torch.empty(sp.Hq, self.total_q, device=dev, dtype=torch.float32)
        elif self.varlen:
            sp = self.spec = inputs.VARLEN_WORKLOADS[name]
            vin = inputs.make_varlen(sp, seed=seed)
            self.host_in = [vin.q, vin.k, vin.v, vin.cu_q, vin.cu_k]
            lens_q = (vin.cu_q[1:] - vin.cu_q[:-1]).tolist()
            lens_k = (vin.cu_k[1:] - vin.cu_k[:-1]).tolist()
            self.flops = sum(workloads.prefill_flops(1, sp.Hq, t, s_, sp.d, sp.causal) for t, s_ in zip(lens_q, lens_k))
            self.min_bytes = sum(workloads.prefill_min_bytes(1, sp.Hq, sp.Hkv, t, s_, sp.d)
                                 for t, s_ in zip(lens_q, lens_k))
            self.max_q, self.total_q, self.total_k = vin.max_q, int(vin.cu_q[-1]), int(vin.cu_k[-1])
            self.dev_in = [t.to(dev) for t in self.host_in]
            self.o = torch.empty_like(self.dev_in[0])
            self.lse = torch.empty(sp.Hq, self.total_q, device=dev, dtype=torch.float32)
        else:
            sp = self.spec = inputs.WORKLOADS[name]
            q, k, v = inputs.make_prefill(sp, seed=seed)
            self.host_in = [q, k, v]
            self.flops = workloads.prefill_flops(sp.B, sp.Hq, sp.T, sp.S, sp.d, sp.causal)
            self.min_bytes = workloads.prefill_min_bytes(sp.B, sp.Hq, sp.Hkv, sp.T, sp.S, sp.d)
            self.dev_in = [t.to(dev) for t in self.host_in]
            self.o = torch.empty_like(self.dev_in[0])
            self.lse = torch.empty(sp.B, sp.Hq, sp.T, device=dev, dtype=torch.float32)
        self.fa = fa

    def call(self, stream):
        sp, fa = self.spec, self.fa
        if self.chunked:
            q, kc, vc, bt, sl, cq = self.dev_in
            fa.paged_attn_prefill(q, kc, vc, bt, sl, cq, sp.B, sp.Hq, sp.Hkv, sp.d, sp.block_size, self.max_blocks,
                                  self.max_q, self.total_q, sp.causal, sp.scale, self.o, self.lse, stream)
        elif self.varlen:
            q, k, v, cq, ck = self.dev_in
            fa.attn_fwd_varlen(q, k, v, self.o, self.lse, cq, ck, sp.B, self.max_q, self.total_q, self.total_k,
                               sp.Hq, sp.Hkv, sp.d, sp.causal, sp.scale, stream)
        else:
            q, k, v = self.dev_in
            fa.attn_fwd(q, k, v, self.o, self.lse, sp.B, sp.Hq, sp.Hkv, sp.T, sp.S, sp.d, sp.causal, sp.scale,
                        stream)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_SETS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--num-splits", type=int, default=0, help="decode splits (0 = library's choice)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--streams", type=int, choices=[1, 2], default=2,
                    help="1: prefill then decode on one stream; 2: the two run concurrently (fork/join per step)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------
# clocks during the timed regions (NVML reads only; nothing is changed)
# --------------------------------------------------------------------------
class ClockSampler:
    """Samples the SM clock and the clock-event reasons of one GPU every
    `period_s` through NVML, from a thread (NVML calls release the GIL), each
    sample stamped with time.perf_counter().  `summary(t0, t1)` reports the
    samples inside a window.  `nvidia-smi -lms` is the fallback when NVML
    cannot be used."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        # NVML numbers GPUs physically; CUDA_VISIBLE_DEVICES may not, so the
        # device is named by its UUID when torch reports one.
        self.ident = str(device_index)
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if uuid:
                self.ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self._stop = threading.Event()
        self._thr = None
        self._proc = None
        self.max_mhz = None
        self.source = None
        self._nv = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = (pynvml.nvmlDeviceGetHandleByUUID(self.ident.encode()) if self.ident.startswith("GPU-")
                       else pynvml.nvmlDeviceGetHandleByIndex(device_index))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            self._nv = None

    def _poll_nvml(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = self._reasons(self._h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def _read_smi(self):
        for line in self._proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            try:
                self.samples.append((time.perf_counter(), int(parts[0]), int(parts[2], 16)))
                if self.max_mhz is None:
                    self.max_mhz = int(parts[1])
            except (ValueError, IndexError):
                pass

    def start(self, wait_s: float = 5.0):
        if self._nv is not None:
            self._thr = threading.Thread(target=self._poll_nvml, daemon=True)
            self.source = "nvml polling every %g ms" % (self.period * 1000)
        else:
            import shutil
            import subprocess
            smi = shutil.which("nvidia-smi")
            if smi is not None:
                try:
                    self._proc = subprocess.Popen(
                        [smi, "-i", self.ident, "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                         "--format=csv,noheader,nounits", "-lms", "20"],
                        stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
                    self._thr = threading.Thread(target=self._read_smi, daemon=True)
                    self.source = "nvidia-smi -lms 20"
                except OSError:
                    self._proc = None
        if self._thr is not None:
            self._thr.start()
            t_end = time.perf_counter() + wait_s  # the timed regions start once samples flow
            while not self.samples and time.perf_counter() < t_end:
                time.sleep(0.01)

    def stop(self):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
        if self._thr is not None:
            self._thr.join(timeout=5)

    def summary(self, t0, t1):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no clock samples"], "samples": 0}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        use = inside or self.samples
        mhz = sorted(s[1] for s in use)
        bits = 0
        for s in use:
            bits |= int(s[2])
        reasons = [name for bit, name in self.REASONS.items() if bits & bit and name != "gpu_idle"]
        return {"sm_mhz": mhz[len(mhz) // 2] if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "samples_total": len(self.samples),
                "source": self.source}


def timed_region(torch, stream, body, K, sampler, world, dist):
    """K calls of `body` with CUDA events on `stream` at the two ends only,
    bracketed by a barrier and a device synchronisation on both sides.
    Returns (milliseconds per call, clock summary of the region)."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    start.record(stream)
    for _ in range(K):
        body()
    end.record(stream)
    while not end.query():  # the sampler thread records clocks meanwhile
        time.sleep(0.0005)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    return start.elapsed_time(end) / K, sampler.summary(t0, t1)


# --------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the same step
# --------------------------------------------------------------------------
class CpuSample:
    """The fp64 oracle on a bounded sample of one step's workloads.  The
    inputs are drawn once; `run()` times the oracle on the sample and scales
    that time to the whole step by visible (query, key) pairs for the
    prefill and by cached tokens for the decode."""

    def __init__(self, pname, dname, peaks, seed_offset=0, decode_budget_s=10.0):
        import torch

        from flashattention_attention_attn_b200 import inputs, workloads
        from oracle import fp64_attention as orc
        self.orc = orc
        f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:
            self.cores = 1
        self.decode_budget_s = decode_budget_s
        if pname in inputs.VARLEN_WORKLOADS:
            sp = inputs.VARLEN_WORKLOADS[pname]
            vin = inputs.make_varlen(sp, seed=sp.seed + seed_offset)
            lq = (vin.cu_q[1:] - vin.cu_q[:-1]).tolist()
            lk = (vin.cu_k[1:] - vin.cu_k[:-1]).tolist()
            n = 2
            cq, ck = vin.cu_q[:n + 1].numpy(), vin.cu_k[:n + 1].numpy()
            a = (f(vin.q[:cq[-1]]), f(vin.k[:ck[-1]]), f(vin.v[:ck[-1]]), cq, ck, sp.scale, sp.causal)
            self.prefill_fn = lambda: orc.attention_varlen(*a)
            pairs = [workloads.visible_pairs(t, s_, sp.causal) for t, s_ in zip(lq, lk)]
            self.prefill_scale = sum(pairs) / max(sum(pairs[:n]), 1)
            self.flops = sum(workloads.prefill_flops(1, sp.Hq, t, s_, sp.d, sp.causal) for t, s_ in zip(lq, lk))
            self.pdesc = f"sequences {n}/{sp.B} (all {sp.Hq} heads), scaled by visible pairs"
            self.prefill_bytes = sum(workloads.prefill_min_bytes(1, sp.Hq, sp.Hkv, t, s_, sp.d) for t, s_ in zip(lq, lk))
        elif pname in inputs.CHUNKED_WORKLOADS:
            sp = inputs.CHUNKED_WORKLOADS[pname]
            ci = inputs.make_chunked(sp, seed=sp.seed + seed_offset)
            c = ci.cache
            lq = (ci.cu_q[1:] - ci.cu_q[:-1]).tolist()
            ctx = c.seq_lens.tolist()
            a = (f(ci.q[:lq[0]]), f(c.k_cache), f(c.v_cache), c.block_table.numpy()[:1], ctx[:1], ci.cu_q.numpy()[:2],
                 c.block_size, sp.scale, sp.causal)
            self.prefill_fn = lambda: orc.paged_prefill(*a)
            pairs = [workloads.visible_pairs(t, s_, sp.causal) for t, s_ in zip(lq, ctx)]
            self.prefill_scale = sum(pairs) / max(pairs[0], 1)
            self.flops = sum(workloads.prefill_flops(1, sp.Hq, t, s_, sp.d, sp.causal) for t, s_ in zip(lq, ctx))
            self.pdesc = f"sequences 1/{sp.B} (all {sp.Hq} heads), scaled by visible pairs"
            self.prefill_bytes = sum(workloads.prefill_min_bytes(1, sp.Hq, sp.Hkv, t, s_, sp.d) for t, s_ in zip(lq, ctx))
        else:
            ps = inputs.WORKLOADS[pname]
            q, k, v = inputs.make_prefill(ps, seed=ps.seed + seed_offset)
            qd, kd, vd = f(q[:1]), f(k[:1]), f(v[:1])
            rows = list(range(0, ps.T, max(1, ps.T // 64)))
            self.prefill_fn = lambda: orc.attention(qd, kd, vd, ps.scale, ps.causal, rows=rows)
            # the oracle forms every row's full score row, so its cost goes with the rows
            self.prefill_scale = ps.B * ps.T / len(rows)
            self.flops = workloads.prefill_flops(ps.B, ps.Hq, ps.T, ps.S, ps.d, ps.causal)
            self.pdesc = f"rows {len(rows)}/{ps.T} of batch 0 (all {ps.Hq} heads), scaled by rows"
            self.prefill_bytes = workloads.prefill_min_bytes(ps.B, ps.Hq, ps.Hkv, ps.T, ps.S, ps.d)
        dbase, dfp8 = decode_workload(dname)
        ds = inputs.WORKLOADS[dbase]
        if dfp8:
            dinp = inputs.make_paged_fp8(ds, seed=ds.seed + seed_offset)
            self.kc = dinp.k_scale * orc.decode_e4m3(dinp.k_cache.numpy())
            self.vc = dinp.v_scale * orc.decode_e4m3(dinp.v_cache.numpy())
        else:
            dinp = inputs.make_paged(ds, seed=ds.seed + seed_offset)
            self.kc, self.vc = f(dinp.k_cache), f(dinp.v_cache)
        self.ds, self.q, self.table = ds, f(dinp.q), dinp.block_table.numpy()
        self.lens = dinp.seq_lens.numpy()
        self.dbytes = workloads.decode_bytes(self.lens, ds.Hq, ds.Hkv, ds.d, ds.block_size,
                                             kv_elem_bytes=1 if dfp8 else 2)
        self.ideal = self.flops / (peaks["bf16_tflops"] * 1e12) + self.dbytes / (peaks["hbm_gbs"] * 1e9)

    def run(self):
        """Oracle seconds for the whole step, estimated from the sample."""
        t0 = time.perf_counter()
        self.prefill_fn()
        t_prefill = (time.perf_counter() - t0) * self.prefill_scale
        done_tok, td, nseq = 0, 0.0, 0
        for b in range(len(self.lens)):  # leading sequences, until the budget or 4 sequences
            t0 = time.perf_counter()
            self.orc.paged_decode(self.q[b:b + 1], self.kc, self.vc, self.table[b:b + 1], self.lens[b:b + 1],
                                  self.ds.block_size, self.ds.scale)
            td += time.perf_counter() - t0
            done_tok += int(self.lens[b])
            nseq += 1
            if nseq >= 4 or td > self.decode_budget_s:
                break
        t_decode = td * float(self.lens.sum()) / max(done_tok, 1)
        self.sample = (f"fp64 oracle: prefill {self.pdesc}, decode {nseq}/{len(self.lens)} sequences "
                       f"({done_tok} tokens), scaled by tokens; the sum estimates the whole step")
        return t_prefill + t_decode

    def baseline(self):
        est = self.run()
        return {"value": 100.0 * self.ideal / est, "unit": UNIT, "cores": int(self.cores), "kind": "oracle",
                "sample": self.sample}


# --------------------------------------------------------------------------
def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    pname, dname = WORKLOAD_SETS[args.workload]
    peaks, peak_src = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return 0
        run_reference(args, pname, dname, peaks, peak_src, world)
        return 0

    import torch
    import torch.distributed as dist

    import flashattention_attention_attn_b200 as fa
    from flashattention_attention_attn_b200 import build as _build, dist_util, inputs, workloads

    if not os.path.exists(_build.LIB_PATH):
        _build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if fa.attn_check_support(local_rank) != 0:
        raise RuntimeError("device not supported by the library")

    dbase, dfp8 = decode_workload(dname)
    ds = inputs.WORKLOADS[dbase]
    # weak scaling: every rank runs its own batch (different seeds), no exchange
    pspec = (inputs.VARLEN_WORKLOADS.get(pname) or inputs.CHUNKED_WORKLOADS.get(pname)
             or inputs.WORKLOADS[pname])
    pre = PrefillCase(pname, dist_util.rank_seed(pspec.seed, rank), dev, fa, inputs, workloads)
    if dfp8:
        dinp = inputs.make_paged_fp8(ds, seed=dist_util.rank_seed(ds.seed, rank))
    else:
        dinp = inputs.make_paged(ds, seed=dist_util.rank_seed(ds.seed, rank))
    qd_, kc, vc = dinp.q.to(dev), dinp.k_cache.to(dev), dinp.v_cache.to(dev)
    bt, sl = dinp.block_table.to(dev), dinp.seq_lens.to(dev)
    od = torch.empty(ds.B, ds.Hq, ds.d, device=dev, dtype=torch.bfloat16)
    maxb = dinp.block_table.shape[1]
    # The prefill and the decode of one step touch disjoint data, so with
    # --streams 2 they run concurrently: the prefill on the current stream,
    # the decode on a second stream of the same priority that forks from it
    # and joins it again every step, so the decode's CTAs fill the SMs the
    # prefill leaves idle.  All timing events sit on the current stream.
    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev) if args.streams == 2 else stream
    fork_ev, join_ev = torch.cuda.Event(), torch.cuda.Event()

    flops = pre.flops
    dbytes = workloads.decode_bytes(dinp.seq_lens.tolist(), ds.Hq, ds.Hkv, ds.d, ds.block_size,
                                    kv_elem_bytes=1 if dfp8 else 2)
    splits = args.num_splits

    def decode_call(st):
        if dfp8:
            fa.paged_attn_decode_fp8(qd_, kc, vc, bt, sl, ds.B, ds.Hq, ds.Hkv, ds.d, ds.block_size, maxb, splits,
                                     dinp.k_scale, dinp.v_scale, od, st)
        else:
            fa.paged_attn_decode(qd_, kc, vc, bt, sl, ds.B, ds.Hq, ds.Hkv, ds.d, ds.block_size, maxb, splits, od,
                                 st)

    def step():
        if side is stream:
            pre.call(stream)
            decode_call(stream)
            return
        fork_ev.record(stream)
        side.wait_event(fork_ev)
        pre.call(stream)
        decode_call(side)
        join_ev.record(side)
        stream.wait_event(join_ev)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    K = args.steps
    sampler = ClockSampler(local_rank)
    sampler.start()
    # The timed step loop (the value).  Only its two ends are recorded: an
    # event between two kernels would cut the programmatic overlap of one
    # kernel's prologue with the previous one's tail.
    ms_step, clocks = timed_region(torch, stream, step, K, sampler, world, dist)
    # Each op alone (the per-op roofline fractions): at least K back-to-back
    # calls and at least PART_MIN_MS of them, so that a short op is timed in
    # steady state rather than over the first few calls after the step loop.
    def part_calls(body):
        t_est, _ = timed_region(torch, stream, body, 3, sampler, world, dist)
        (n,) = dist_util.max_over_ranks([max(K, math.ceil(PART_MIN_MS / max(t_est, 1e-3)))], device=dev)
        return int(n)

    pre_body, dec_body = (lambda: pre.call(stream)), (lambda: decode_call(stream))
    n_pre, n_dec = part_calls(pre_body), part_calls(dec_body)
    ms_pre, clocks_pre = timed_region(torch, stream, pre_body, n_pre, sampler, world, dist)
    ms_dec, clocks_dec = timed_region(torch, stream, dec_body, n_dec, sampler, world, dist)
    sampler.stop()
    status = fa.attn_read_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status}: a bounded wait timed out")
    ms_step, ms_pre, ms_dec = dist_util.max_over_ranks([ms_step, ms_pre, ms_dec], device=dev)

    ideal_pre = flops / (peaks["bf16_tflops"] * 1e12)
    ideal_dec = dbytes / (peaks["hbm_gbs"] * 1e9)
    ideal = ideal_pre + ideal_dec
    value = 100.0 * world * ideal / (ms_step * 1e-3)

    # ---------------- end to end through the public API, host buffers ----------------
    e2e = None
    if args.e2e_steps > 0:
        pin = lambda t: t.pin_memory()  # noqa: E731
        h_in = [pin(t) for t in pre.host_in] + [pin(dinp.q), pin(dinp.k_cache), pin(dinp.v_cache),
                                                pin(dinp.block_table), pin(dinp.seq_lens)]
        d_in = list(pre.dev_in) + [qd_, kc, vc, bt, sl]
        h_o = torch.empty(pre.o.shape, dtype=pre.o.dtype).pin_memory()
        h_lse = torch.empty(pre.lse.shape, dtype=pre.lse.dtype).pin_memory()
        h_od = torch.empty(od.shape, dtype=od.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in h_in)
        d2h = sum(t.numel() * t.element_size() for t in (h_o, h_lse, h_od))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        with torch.cuda.stream(stream):  # the copies go on the step's (joining) stream
            for _ in range(args.e2e_steps):
                for h, d_ in zip(h_in, d_in):
                    d_.copy_(h, non_blocking=True)
                step()
                h_o.copy_(pre.o, non_blocking=True)
                h_lse.copy_(pre.lse, non_blocking=True)
                h_od.copy_(od, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
        (e2e_ms,) = dist_util.max_over_ranks([e2e_ms], device=dev)
        e2e = {"value": 100.0 * world * ideal / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    dec_gbs = dbytes / (ms_dec * 1e-3) / 1e9
    pre_tflops = flops / (ms_pre * 1e-3) / 1e12
    # The burst GEMM peak applies to a kernel timed in short bursts; if the
    # power cap was active while it was timed, the sustained one.
    capped = "sw_power_cap" in clocks_pre.get("reasons", [])
    tpeak = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    tpeak_src = (f"{peak_src} (bf16_tflops_sustained: sw_power_cap active while the prefill was timed)"
                 if capped else f"{peak_src} (bf16_tflops, burst)")
    pre_traffic, pre_tnote = traffic_of(args.workload, "prefill")
    dec_traffic, dec_tnote = traffic_of(args.workload, "decode")
    parts = {
        "prefill": {"op": pre.name, "ms": ms_pre, "tflops": pre_tflops, "peak": tpeak, "frac": pre_tflops / tpeak,
                    "peak_source": tpeak_src, "flops": flops, "algorithmic_bytes": pre.min_bytes,
                    "traffic": pre_traffic, "traffic_note": pre_tnote, "calls": n_pre, "clocks": clocks_pre},
        "decode": {"op": dname, "ms": ms_dec, "gbs": dec_gbs, "peak": peaks["hbm_gbs"],
                   "frac": dec_gbs / peaks["hbm_gbs"], "peak_source": f"{peak_src} (hbm_gbs)", "bytes": dbytes,
                   "traffic": dec_traffic, "traffic_note": dec_tnote, "calls": n_dec, "clocks": clocks_dec},
    }
    if ms_pre >= ms_dec:  # the op that takes longer alone
        roofline = {"bound": "tensor", "achieved": pre_tflops, "peak": tpeak, "unit": "TFLOP/s",
                    "frac": pre_tflops / tpeak, "traffic": pre_traffic, "traffic_note": pre_tnote,
                    "algorithmic_bytes": pre.min_bytes, "kernel": f"prefill ({pre.name})",
                    "peak_source": tpeak_src, "duration": PART_TIMING}
    else:
        roofline = {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": dec_gbs / peaks["hbm_gbs"], "traffic": dec_traffic, "traffic_note": dec_tnote,
                    "algorithmic_bytes": dbytes, "kernel": f"paged decode ({dname}; split kernel + LSE combine)",
                    "peak_source": f"{peak_src} (hbm_gbs)", "duration": PART_TIMING}
    combine = 1 if (splits != 1) else 0  # the LSE combine runs whenever the decode uses more than one split
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16; random block-id permutations)",
        "config": step_config(pname, dname, inputs, world, args, pre.min_bytes, dbytes),
        "parts": parts,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": (2 + combine) * K,
        "clocks": clocks,
        "peaks": {**peaks, "source": peak_src},
        "csrc_hash": csrc_hash(),
    }
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = CpuSample(pname, dname, peaks).baseline()
    print(json.dumps(line))
    return 0


def run_reference(args, pname, dname, peaks, peak_src, world):
    """The fp64 CPU oracle, each step a bounded sample of the same workload."""
    from flashattention_attention_attn_b200 import inputs
    budget = max(0.5, 10.0 / max(1, args.steps))  # decode seconds per step: the run stays within minutes
    cs = CpuSample(pname, dname, peaks, decode_budget_s=budget)
    for _ in range(max(0, args.warmup)):
        cs.run()
    est = sum(cs.run() for _ in range(args.steps)) / max(1, args.steps)
    value = 100.0 * cs.ideal / est
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": est * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeds as ours)",
        "config": step_config(pname, dname, inputs, world, args, cs.prefill_bytes, cs.dbytes),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cs.cores, "kind": "oracle", "sample": cs.sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "peaks": {**peaks, "source": peak_src},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    sys.exit(main())
