"""Benchmark of the fused-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  * attn_fwd          Llama3-8B-shaped causal GQA prefill (B=2, Hq=32, Hkv=8,
                      T=S=512, d=128)
  * paged_attn_decode one-token decode of 64 sequences against a paged cache
                      (Hq=32, Hkv=8, d=128, block_size=16, context U[256,4096])
The metric is the fraction of the B200 roofline the step reaches: the ideal
step time is prefill FLOPs / measured bf16 tensor peak + decode bytes /
measured HBM bandwidth, and value = 100 * (sum over ranks of ideal time) /
(measured step time, max over ranks): percent of one B200's roofline,
summed over the GPUs of the job.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload step|long|varlen|chunked|fp8]

`--workload long` times the long-context pair (T=S=16384 prefill and a
131072-token split-KV decode) with the same accounting; `--workload varlen`
replaces the prefill by 16 packed sequences of U[64, 2048] tokens
(attn_fwd_varlen); `--workload chunked` by a 512-token chunk of each of 8
sequences against their paged cache of 1k-8k tokens (paged_attn_prefill);
`--workload fp8` keeps the step but stores the decode cache as FP8 e4m3
(paged_attn_decode_fp8; decode bytes count 1 byte per cached element).  `--impl reference`
times the fp64 CPU oracle (the only reference implementation there is) on a
bounded sample of the same step.
"""

from __future__ import annotations

import argparse
import json
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attn TFLOP/s & paged-decode KV GB/s, % of B200 roofline"
PART_TIMING = ("CUDA events around each part, on the launching stream, in a second K-step loop "
               "run right after the timed one")
UNIT = "% of 1xB200 roofline (summed over GPUs)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOAD_SETS = {
    "step": ("llama3_8b_prefill", "paged_decode_b64"),
    "long": ("long_prefill_16k", "long_decode_131k"),
    "varlen": ("varlen_prefill_16seq", "paged_decode_b64"),
    "chunked": ("chunked_prefill_paged", "paged_decode_b64"),
    "fp8": ("llama3_8b_prefill", "paged_decode_b64:fp8"),
}


# DRAM bytes (read + write) per launch of the dominant kernel of each step,
# from the one-pass ncu launch lists of the same command (`dram__bytes_read.sum`
# + `dram__bytes_write.sum`, mean over the captured launches), summarised in
# profiles/launches_<workload>.md.  A value is dropped (None) whenever the
# kernel changes after its capture.
#   step / fp8: decode split kernel + LSE combine of one paged_attn_decode call
#   long, varlen, chunked: the prefill launch
TRAFFIC_BYTES = {
    "step": 597.38e6 + 3.14e6 + 4.58e6,   # profiles/launches_llama3_8b_prefill_paged_decode_b64.md
    "fp8": 299.00e6 + 2.79e6 + 4.58e6,    # profiles/launches_llama3_8b_prefill_paged_decode_b64_fp8.md
    "long": 385.56e6 + 101.25e6,          # profiles/launches_long_prefill_16k_long_decode_131k.md
    "varlen": 247.64e6 + 89.08e6,         # profiles/launches_varlen_prefill_16seq_paged_decode_b64.md
    "chunked": 337.31e6 + 24.55e6,        # profiles/launches_chunked_prefill_paged_paged_decode_b64.md
}


def decode_workload(dname):
    """(spec name, FP8 cache?) of a decode workload name ("name" or "name:fp8")."""
    base, _, kind = dname.partition(":")
    return base, kind == "fp8"


class PrefillCase:
    """The prefill half of a step: dense (attn_fwd) or packed (attn_fwd_varlen); `--workload chunked` by a 512-token chunk of each of 8
sequences against their paged cache of 1k-8k tokens (paged_attn_prefill);
`--workload fp8` keeps the step but stores the decode cache as FP8 e4m3
(paged_attn_decode_fp8; decode bytes count 1 byte per cached element)."""

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
            self.config = {**vars_of(sp), "context_lengths": ctx, "query_counts": lens_q}
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
            self.config = {**vars_of(sp), "lengths": lens_q, "total_tokens": self.total_q}
        else:
            sp = self.spec = inputs.WORKLOADS[name]
            q, k, v = inputs.make_prefill(sp, seed=seed)
            self.host_in = [q, k, v]
            self.flops = workloads.prefill_flops(sp.B, sp.Hq, sp.T, sp.S, sp.d, sp.causal)
            self.min_bytes = workloads.prefill_min_bytes(sp.B, sp.Hq, sp.Hkv, sp.T, sp.S, sp.d)
            self.dev_in = [t.to(dev) for t in self.host_in]
            self.o = torch.empty_like(self.dev_in[0])
            self.lse = torch.empty(sp.B, sp.Hq, sp.T, device=dev, dtype=torch.float32)
            self.config = vars_of(sp)
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
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_SETS), default="step")
    ap.add_argument("--num-splits", type=int, default=0, help="decode splits (0 = library's choice)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--streams", type=int, choices=[1, 2], default=2,
                    help="1: prefill then decode on one stream; 2: the two run concurrently (fork/join per step)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# --------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock and clock-event reasons every 20 ms from an
    `nvidia-smi -lms` child process (independent of this process's GIL), with
    NVML polling in a thread as the fallback.  Each sample is stamped with
    time.perf_counter() when it arrives."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.period = period_s
        # nvidia-smi and NVML number GPUs physically; CUDA_VISIBLE_DEVICES may
        # not, so the device is named by its UUID when torch reports one.
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
        except Exception:
            self._nv = None

    def _read_smi(self):
        for line in self._proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            try:
                self.samples.append((time.perf_counter(), int(parts[0]), int(parts[2], 16)))
                if self.max_mhz is None:
                    self.max_mhz = int(parts[1])
            except (ValueError, IndexError):
                pass

    def _poll_nvml(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self, wait_s: float = 5.0):
        import shutil
        import subprocess
        smi = shutil.which("nvidia-smi")
        if smi is not None:
            try:
                self._proc = subprocess.Popen(
                    [smi, "-i", self.ident, "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                     "--format=csv,noheader,nounits", "-lms", str(int(self.period * 1000))],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
                self._thr = threading.Thread(target=self._read_smi, daemon=True)
                self.source = "nvidia-smi -lms %d" % int(self.period * 1000)
            except OSError:
                self._proc = None
        if self._proc is None and self._nv is not None:
            self._thr = threading.Thread(target=self._poll_nvml, daemon=True)
            self.source = "nvml polling"
        if self._thr is not None:
            self._thr.start()
            t_end = time.perf_counter() + wait_s  # the timed region starts once samples flow
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


# --------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the same step
# --------------------------------------------------------------------------
def _cpu_prefill_dense(pname, seed_offset, orc, inputs, workloads, f):
    """Oracle time of a dense prefill, from an evenly spread set of rows of
    batch 0 (all heads), scaled by visible pairs to the whole workload."""
    ps = inputs.WORKLOADS[pname]
    q, k, v = inputs.make_prefill(ps, seed=ps.seed + seed_offset)
    qd, kd, vd = f(q), f(k), f(v)
    T = ps.T
    rows = list(range(0, T, max(1, T // 64)))
    t0 = time.perf_counter()
    orc.attention(qd[:1], kd[:1], vd[:1], ps.scale, ps.causal, rows=rows)
    tp = time.perf_counter() - t0
    seen = sum(min(ps.S, i + ps.S - ps.T + 1) if ps.causal else ps.S for i in rows)  # cost ~ keys seen
    full_pairs = workloads.visible_pairs(ps.T, ps.S, ps.causal) * ps.B
    flops = workloads.prefill_flops(ps.B, ps.Hq, ps.T, ps.S, ps.d, ps.causal)
    return tp * full_pairs / max(seen, 1), flops, f"rows {len(rows)}/{T} of batch 0 (all {ps.Hq} heads)"


def _cpu_prefill_varlen(pname, seed_offset, orc, inputs, workloads, f):
    """Oracle time of a packed prefill, from its first two sequences, scaled
    by visible pairs to all sequences."""
    sp = inputs.VARLEN_WORKLOADS[pname]
    vin = inputs.make_varlen(sp, seed=sp.seed + seed_offset)
    lq = (vin.cu_q[1:] - vin.cu_q[:-1]).tolist()
    lk = (vin.cu_k[1:] - vin.cu_k[:-1]).tolist()
    n = 2
    cq, ck = vin.cu_q[:n + 1].numpy(), vin.cu_k[:n + 1].numpy()
    t0 = time.perf_counter()
    orc.attention_varlen(f(vin.q[:cq[-1]]), f(vin.k[:ck[-1]]), f(vin.v[:ck[-1]]), cq, ck, sp.scale, sp.causal)
    tp = time.perf_counter() - t0
    pairs = [workloads.visible_pairs(t, s_, sp.causal) for t, s_ in zip(lq, lk)]
    flops = sum(workloads.prefill_flops(1, sp.Hq, t, s_, sp.d, sp.causal) for t, s_ in zip(lq, lk))
    return tp * sum(pairs) / max(sum(pairs[:n]), 1), flops, f"sequences {n}/{sp.B} (all {sp.Hq} heads)"


def _cpu_prefill_chunked(pname, seed_offset, orc, inputs, workloads, f):
    """Oracle time of a chunked paged prefill, from its first sequence,
    scaled by visible pairs to all sequences."""
    sp = inputs.CHUNKED_WORKLOADS[pname]
    ci = inputs.make_chunked(sp, seed=sp.seed + seed_offset)
    c = ci.cache
    lq = (ci.cu_q[1:] - ci.cu_q[:-1]).tolist()
    ctx = c.seq_lens.tolist()
    t0 = time.perf_counter()
    orc.paged_prefill(f(ci.q[:lq[0]]), f(c.k_cache), f(c.v_cache), c.block_table.numpy()[:1], ctx[:1],
                      ci.cu_q.numpy()[:2], c.block_size, sp.scale, sp.causal)
    tp = time.perf_counter() - t0
    pairs = [workloads.visible_pairs(t, s_, sp.causal) for t, s_ in zip(lq, ctx)]
    flops = sum(workloads.prefill_flops(1, sp.Hq, t, s_, sp.d, sp.causal) for t, s_ in zip(lq, ctx))
    return tp * sum(pairs) / max(pairs[0], 1), flops, f"sequences 1/{sp.B} (all {sp.Hq} heads)"


def cpu_baseline(pname, dname, peaks, seed_offset=0, budget_s=20.0):
    import torch

    from flashattention_attention_attn_b200 import inputs, workloads
    from oracle import fp64_attention as orc

    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = 1
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    if pname in inputs.VARLEN_WORKLOADS:
        t_prefill, flops, pdesc = _cpu_prefill_varlen(pname, seed_offset, orc, inputs, workloads, f)
    elif pname in inputs.CHUNKED_WORKLOADS:
        t_prefill, flops, pdesc = _cpu_prefill_chunked(pname, seed_offset, orc, inputs, workloads, f)
    else:
        t_prefill, flops, pdesc = _cpu_prefill_dense(pname, seed_offset, orc, inputs, workloads, f)
    dbase, dfp8 = decode_workload(dname)
    ds = inputs.WORKLOADS[dbase]
    if dfp8:
        dinp = inputs.make_paged_fp8(ds, seed=ds.seed + seed_offset)
        kc = dinp.k_scale * orc.decode_e4m3(dinp.k_cache.numpy())
        vc = dinp.v_scale * orc.decode_e4m3(dinp.v_cache.numpy())
    else:
        dinp = inputs.make_paged(ds, seed=ds.seed + seed_offset)
        kc, vc = f(dinp.k_cache), f(dinp.v_cache)
    # decode sample: leading sequences until ~budget/2 spent or 4 sequences
    lens = dinp.seq_lens.numpy()
    qq = f(dinp.q)
    done_tok, td, nseq = 0, 0.0, 0
    for b in range(len(lens)):
        t0 = time.perf_counter()
        orc.paged_decode(qq[b:b + 1], kc, vc, dinp.block_table.numpy()[b:b + 1], lens[b:b + 1], 16, ds.scale)
        td += time.perf_counter() - t0
        done_tok += int(lens[b])
        nseq += 1
        if nseq >= 4 or td > budget_s / 2:
            break
    t_decode = td * float(lens.sum()) / max(done_tok, 1)
    dbytes = workloads.decode_bytes(lens, ds.Hq, ds.Hkv, ds.d, ds.block_size, kv_elem_bytes=1 if dfp8 else 2)
    ideal = flops / (peaks["bf16_tflops"] * 1e12) + dbytes / (peaks["hbm_gbs"] * 1e9)
    est = t_prefill + t_decode
    return {"value": 100.0 * ideal / est, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": (f"fp64 oracle: prefill {pdesc}, decode {nseq}/{len(lens)} sequences ({done_tok} tokens); "
                       f"time scaled by visible pairs / tokens to the full step"),
            "est_step_s": est}


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
    # prefill leaves idle.  All timing events sit on the current stream.  (A
    # higher priority for the prefill's stream measured slower on the default
    # and FP8 steps.)
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
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    # Only the two ends are recorded: an event between two kernels would cut
    # the programmatic overlap of one kernel's prologue with the previous tail.
    start.record(stream)
    for i in range(K):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    sampler.stop()
    total_ms = start.elapsed_time(end)

    # Per-part split (reported, not the value): K more steps with events
    # between the parts, both parts on one stream.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(K):
        ev[i][0].record(stream)
        pre.call(stream)
        ev[i][1].record(stream)
        decode_call(stream)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    status = fa.attn_read_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status}: a bounded wait timed out")

    t_pre = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)) / K
    t_dec = sum(ev[i][1].elapsed_time(ev[i][2]) for i in range(K)) / K
    ms_step = total_ms / K
    ms_step, t_pre, t_dec = dist_util.max_over_ranks([ms_step, t_pre, t_dec], device=dev)

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

    dec_gbs = dbytes / (t_dec * 1e-3) / 1e9
    pre_tflops = flops / (t_pre * 1e-3) / 1e12
    clocks = sampler.summary(t_wall0, t_wall1)
    dominant = "decode" if t_dec >= t_pre else "prefill"
    if dominant == "decode":
        roofline = {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": dec_gbs / peaks["hbm_gbs"], "traffic": TRAFFIC_BYTES.get(args.workload),
                    "traffic_unit": "bytes per call (ncu DRAM read + write)", "algorithmic_bytes": dbytes,
                    "kernel": "paged_attn_decode (split kernel + LSE combine)",
                    "peak_source": f"{peak_src} (hbm_gbs)", "duration": PART_TIMING}
    else:
        # The burst GEMM peak applies to a kernel that runs in short bursts; if
        # the power cap was active during the timed loop, the sustained one.
        capped = "sw_power_cap" in clocks.get("reasons", [])
        tpeak = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
        roofline = {"bound": "tensor", "achieved": pre_tflops, "peak": tpeak, "unit": "TFLOP/s",
                    "frac": pre_tflops / tpeak, "traffic": TRAFFIC_BYTES.get(args.workload),
                    "traffic_unit": "bytes per launch (ncu DRAM read + write)", "algorithmic_bytes": pre.min_bytes,
                    "kernel": "attn_fwd",
                    "peak_source": (f"{peak_src} (bf16_tflops_sustained: sw_power_cap active in the timed loop)"
                                    if capped else f"{peak_src} (bf16_tflops, burst)"),
                    "duration": PART_TIMING}
    launches_per_step = 1 + 1 + 1  # prefill, decode split kernel, LSE combine
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16; random block-id permutations)",
        "config": {"workload": f"{pname} + {dname}", "prefill": pre.config,
                   "decode": {**vars_of(ds), "kv_cache": "fp8 e4m3" if dfp8 else "bf16"},
                   "decode_num_splits": splits or "auto", "parallelism": f"replicas x{world} (no exchange)",
                   "streams": ("prefill and decode concurrently on two streams (fork/join every step)"
                               if args.streams == 2 else "prefill then decode on one stream"),
                   "l2": "inputs larger than L2 (decode KV cache %.0f MB per step)" % (dbytes / 1e6)},
        "parts": {"prefill": {"ms": t_pre, "tflops": pre_tflops, "frac": pre_tflops / peaks["bf16_tflops"],
                              "flops": flops},
                  "decode": {"ms": t_dec, "gbs": dec_gbs, "frac": dec_gbs / peaks["hbm_gbs"],
                             "bytes": dbytes}},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
        "peaks": {**peaks, "source": peak_src},
    }
    if not args.no_cpu_baseline and world == 1:
        cb = cpu_baseline(pname, dname, peaks)
        cb.pop("est_step_s", None)
        line["cpu_baseline"] = cb
    print(json.dumps(line))
    return 0


def vars_of(spec):
    return {k: getattr(spec, k) for k in spec.__dataclass_fields__ if not k.startswith("_")}


def run_reference(args, pname, dname, peaks, peak_src, world):
    """The fp64 CPU oracle, each step a bounded sample of the same workload."""
    steps = []
    info = None
    for i in range(max(0, args.warmup) + args.steps):
        budget = 20.0 / max(1, args.steps)
        r = cpu_baseline(pname, dname, peaks, budget_s=budget)
        if i >= args.warmup:
            steps.append(r["est_step_s"])
            info = r
    est = sum(steps) / len(steps)
    from flashattention_attention_attn_b200 import inputs
    value = info["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": est * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeds as ours)",
        "config": {"workload": f"{pname} + {dname}", "prefill": vars_of(inputs.VARLEN_WORKLOADS.get(pname) or inputs.CHUNKED_WORKLOADS.get(pname)
                                     or inputs.WORKLOADS[pname]),
                   "decode": vars_of(inputs.WORKLOADS[decode_workload(dname)[0]])},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                         "sample": info["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "peaks": {**peaks, "source": peak_src},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    sys.exit(main())
