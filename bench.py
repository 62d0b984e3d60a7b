#!/usr/bin/env python
"""Benchmark of MLA decode attention on B200: effective TB/s (KV + Q bytes) and TFLOPS.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3] [--impl ours|reference]
                    [--kv bf16|fp8]

One step = the whole decode path for one batch: split-KV metadata, the split kernel and
the combine kernel, on inputs already resident in HBM. Where the inputs are larger than
twice the L2 (126 MB) -- every workload but the tiny one -- no flush is needed between
steps; smaller inputs get a 256 MB write between steps, outside the timed steps. Rank 0
prints one JSON line.

Multi-GPU: one process per GPU (torchrun); every rank decodes its own batch of the same
shape (independent problems, no collective on the data path: weak scaling); the time is
the max over ranks and the value counts the bytes of all ranks.

``--kv fp8`` runs the same workload over the fp8 (E4M3) latent cache (640 bytes per token);
the bytes of the metric are then the fp8 cache's.

``--impl reference`` times the CPU oracle (the plain C fp64 implementation under
``oracle/``) on a bounded sample of the same workload; it is the deliberately slow
reference arm, run on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_decode_attention_14_b200 import workloads as W  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
SPEC_HBM_GBS = 8000.0         # B200 HBM3e, nominal (7.7 TB/s in HGX systems)
SPEC_BF16_TFLOPS = 2250.0     # B200 dense bf16/fp16 tensor peak, nominal
TARGET_HBM_FRAC = 0.80        # the split kernel's goal on the v3 workload
METRIC = "MLA decode effective TB/s and TFLOPS vs B200 roofline (bf16 paged KV)"
METRIC_FP8 = "MLA decode effective TB/s and TFLOPS vs B200 roofline (fp8 paged KV)"
METRIC_SPARSE = "MLA sparse decode effective TB/s and TFLOPS vs B200 roofline (bf16 paged KV, top-k lists)"
PROFILE_TRAFFIC = {"bf16": os.path.join(ROOT, "profiles", "decode_split_v3_traffic.txt"),
                   "fp8": os.path.join(ROOT, "profiles", "decode_split_fp8_v3_traffic.txt")}
L2_BYTES = 126 << 20


def describe(wl: W.Workload, kv: str = "bf16") -> str:
    n = wl.seqlens
    cache = ("bf16 N(0,1)" if kv == "bf16" else
             "fp8 cache: E4M3 latent (N(0,1) x 64, latent scale 2^-6) + bf16 N(0,1) rotary, 640 B/token; bf16 N(0,1) q")
    return ("%s: batch %d, h_q %d, s_q %d%s, seqlens %d..%d (mean %.0f), 64-token blocks, d_qk 576, d_v 512, "
            "%s, scale 192^-0.5" % (wl.name, wl.batch, wl.h_q, wl.s_q, " causal" if wl.causal else "",
                                    n.min(), n.max(), n.mean(), cache))


def kv_token_bytes(kv: str) -> int:
    return W.F8_REC if kv == "fp8" else 2 * W.D_QK


def oracle_decode(kv, inp, wl, tasks, nthreads):
    """The oracle over the run's cache format (test infrastructure: the CPU-baseline leg only)."""
    import oracle
    if kv == "fp8":
        return oracle.decode_fp8(inp["q"], inp["kv8"], inp["kv_scale"], inp["block_table"], inp["seqlens"],
                                 wl.scale, wl.causal, tasks=tasks, nthreads=nthreads)
    return oracle.decode(inp["q"], inp["kv"], inp["block_table"], inp["seqlens"], wl.scale, wl.causal,
                         tasks=tasks, nthreads=nthreads)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def _code_only(text: str) -> str:
    """C/CUDA source with comments removed and whitespace runs collapsed (string literals in these
    sources hold no comment markers), so that edits to comments do not change the hash."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


SPLIT_KERNEL_SOURCES = ("common.cuh", "decode_sm100.cu", "sm100_ptx.cuh", "schedule.cuh")  # the split kernel's device code


def kernel_source_hash() -> str:
    """Hash of the code (not the comments) of the split kernel's device sources."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_decode_attention_14_b200", "csrc")
    for name in SPLIT_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update((name + "\n" + _code_only(f.read())).encode())
    return h.hexdigest()[:16]


def profiled_traffic(cache: str = "bf16"):
    """DRAM bytes per split-kernel launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    try:
        kv = {}
        with open(PROFILE_TRAFFIC[cache]) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel_sources_sha256_16") != kernel_source_hash():
            return None
        return float(kv["dram_bytes_per_launch_full_size"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 50):
        self.index, self.period = index, period_ms
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", str(self.period)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() in ("active", "1"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(values, device=None):
    """Elementwise max of per-rank timings over all ranks (identity without a process group).

    Every rank must call this the same number of times, in the same order."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(bytes_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job TB/s: every rank decodes its own batch of the same shape (weak scaling)."""
    return bytes_per_rank * world / (ms_per_step * 1e-3) / 1e12


# --------------------------------------------------------------------------- reference arm
def run_reference(args, wl, inp, counts):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    # calibrate: one row of the longest sequence
    b_long = int(np.argmax(wl.seqlens))
    t0 = time.perf_counter()
    oracle_decode(args.kv, inp, wl, np.array([[b_long, 0, 0]], np.int32), 1)
    per_row = max(time.perf_counter() - t0, 1e-4) * float(wl.seqlens.mean()) / float(wl.seqlens.max())
    budget = min(10.0, 150.0 / max(1, args.steps + args.warmup))      # seconds of wall time per step
    nrows = int(max(1, min(wl.h_q * wl.s_q, budget * cores / per_row)))
    seq = int(rng.integers(0, wl.batch))
    heads = np.arange(nrows) % wl.h_q
    tasks = np.array([[seq, (i // wl.h_q) % wl.s_q, h] for i, h in enumerate(heads)], np.int32)
    n = int(wl.seqlens[seq])
    # algorithmic bytes of this sample: the sequence's KV once, plus its sampled query rows
    sample_bytes = n * kv_token_bytes(args.kv) + nrows * 1152
    for _ in range(args.warmup):
        oracle_decode(args.kv, inp, wl, tasks, cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_decode(args.kv, inp, wl, tasks, cores)
    dt = (time.perf_counter() - t0) / args.steps
    tbs = sample_bytes / dt / 1e12
    sample = "%d of %d query rows of sequence %d (%d tokens), all its keys, per step" % (nrows, wl.rows, seq, n)
    line = {"metric": METRIC_FP8 if args.kv == "fp8" else METRIC, "value": tbs, "unit": "TB/s",
            "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": describe(wl, args.kv), "kv": args.kv, "sample": sample},
            "cpu_baseline": {"value": tbs, "unit": "TB/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": tbs, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- our arm
def cpu_baseline(wl, inp, target_s=12.0, kv="bf16"):
    """The oracle, as it stands, on a bounded sample of the workload (rank 0, N = 1): whole
    sequences (every query row, every key) in a seeded order until ~target_s of CPU work."""
    cores = os.cpu_count() or 1
    order = np.random.default_rng(0).permutation(wl.batch)

    def rows_of(seqs):
        return np.array([[s, t, h] for s in seqs for t in range(wl.s_q) for h in range(wl.h_q)], np.int32)

    t0 = time.perf_counter()
    oracle_decode(kv, inp, wl, rows_of([int(order[0])]), cores)
    per_token = max(time.perf_counter() - t0, 1e-6) / max(1, int(wl.seqlens[order[0]]))
    chosen, est = [], 0.0
    for s in order:
        chosen.append(int(s))
        est += per_token * max(1, int(wl.seqlens[s]))
        if est >= target_s:
            break
    t0 = time.perf_counter()
    oracle_decode(kv, inp, wl, rows_of(chosen), cores)
    dt = time.perf_counter() - t0
    n = int(sum(int(wl.seqlens[s]) for s in chosen))
    # the metric's unit: algorithmic bytes (each sampled sequence's KV once + its query rows) per second
    val = (n * kv_token_bytes(kv) + len(chosen) * wl.rows * 1152) / dt / 1e12
    return {"value": val, "unit": "TB/s", "cores": cores, "kind": "oracle",
            "sample": "%d of %d sequences (%d tokens, all %d query rows each), %.1f s on %d threads"
                      % (len(chosen), wl.batch, n, wl.rows, dt, cores),
            "seconds": dt}


def neighbour_steps(mla, wl, dev, stream, iters=50):
    """The steps either side of decode, timed on their own (not part of the step): the per-head
    projections q_nope W_UK -> q and o_latent W_UV -> o (tcgen05 GEMMs, random weights) and a
    one-token append into a scratch cache. Each: CUDA-event time per call, algorithmic bytes
    (weights + activations read once, results written once) and the HBM fraction."""
    import torch
    hbm = measured_peaks()[0]
    b, s_q, h = wl.batch, wl.s_q, wl.h_q
    g = torch.Generator(device=dev).manual_seed(0)

    def rnd(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g, device=dev) * scale).to(torch.bfloat16)

    def timed(fn):
        # `iters` calls captured in one CUDA graph and replayed: the kernels' own time, without the
        # host's launch gaps between calls
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(iters):
                fn()
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del graph
        return e0.elapsed_time(e1) / iters

    res = {}
    q_nope, w_uk = rnd(b, s_q, h, 128), rnd(h, 128, 512, scale=128 ** -0.5)
    q = torch.zeros((b, s_q, h, 576), dtype=torch.bfloat16, device=dev)
    o_lat, w_uv = rnd(b, s_q, h, 512), rnd(h, 512, 128, scale=512 ** -0.5)
    rows = b * s_q * h
    for name, fn, nbytes, flops in (
            ("absorb_q", lambda: mla.absorb_q(q_nope, w_uk, q), 2 * (h * 128 * 512 + rows * 128 + rows * 512),
             2 * rows * 128 * 512),
            ("absorb_o", lambda: mla.absorb_o(o_lat, w_uv), 2 * (h * 512 * 128 + rows * 512 + rows * 128),
             2 * rows * 512 * 128)):
        ms = timed(fn)
        res[name] = {"us": ms * 1e3, "bytes": nbytes, "flops": flops, "GBps": nbytes / (ms * 1e-3) / 1e9,
                     "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / hbm}
    new_kv = rnd(b, 1, 576)
    cache = torch.zeros((b, 64, 1, 576), dtype=torch.bfloat16, device=dev)
    table = torch.arange(b, dtype=torch.int32, device=dev).reshape(b, 1)
    lens = torch.zeros((b,), dtype=torch.int32, device=dev)
    ms = timed(lambda: mla.append_kv(new_kv, cache, table, lens))
    res["append_kv"] = {"us": ms * 1e3, "bytes": 2 * b * 1152, "GBps": 2 * b * 1152 / (ms * 1e-3) / 1e9}
    st = mla.check_status()
    if st != 0:
        raise SystemExit("device error status %d in the neighbour steps" % st)
    res["note"] = ("per call: %d calls captured in one CUDA graph, its replay timed with CUDA events; "
                   "the HBM fraction is of the measured copy peak" % iters)
    return res


# --------------------------------------------------------------------------- every workload
CONFIG_SET = [("tiny", "bf16", None), ("v2lite", "bf16", None), ("multitoken", "bf16", None),
              ("skewed", "bf16", None), ("v2lite", "fp8", None), ("v3", "fp8", None),
              ("multitoken", "fp8", None), ("skewed", "fp8", None), ("v3", "bf16", 2048)]


def roofline_fracs(nbytes: int, flops: int, seconds: float, peaks):
    hbm, tfl_burst, _, _ = peaks
    gbs, tf = nbytes / seconds / 1e9, flops / seconds / 1e12
    ridge = tfl_burst * 1e12 / (hbm * 1e9)
    return {"bound": "hbm" if flops / nbytes < ridge else "tensor",
            "hbm_frac": gbs / hbm, "tensor_frac": tf / tfl_burst,
            "hbm_frac_spec": gbs / SPEC_HBM_GBS, "tensor_frac_spec": tf / SPEC_BF16_TFLOPS}


def measure_config(mla, name, kv, topk, dev, stream, peaks, target_s=0.4, warmup=5):
    """One workload at 1 GPU: whole step (metadata + split + combine) and split kernel, CUDA events."""
    import torch
    wl = W.workload(name)
    fp8 = kv == "fp8"
    inp = W.make_inputs_fp8(wl, seed=0, tail="normal") if fp8 else W.make_inputs(wl, seed=0, tail="normal")
    q = torch.from_numpy(inp["q"]).view(torch.bfloat16).to(dev)
    kvt = (torch.from_numpy(inp["kv8"]) if fp8 else torch.from_numpy(inp["kv"]).view(torch.bfloat16)).to(dev)
    bt = torch.from_numpy(inp["block_table"]).to(dev)
    sl = torch.from_numpy(inp["seqlens"]).to(dev)
    out = torch.empty((wl.batch, wl.s_q, wl.h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.batch, wl.h_q, wl.s_q), dtype=torch.float32, device=dev)
    if topk:
        ixh = W.sparse_indices(wl.seqlens, wl.s_q, topk, seed=0)
        ix = torch.from_numpy(ixh).to(dev)
        counts = W.sparse_counts(wl, ixh)
        parts = mla.default_num_parts(wl.h_q, 1, dev)
        ws = torch.empty((mla.workspace_bytes(wl.batch * wl.s_q, 1, wl.h_q, parts),), dtype=torch.uint8, device=dev)

        def step(ev=None):
            meta = mla.get_metadata_sparse(wl.batch, wl.s_q, wl.h_q, topk, num_parts=parts)
            if ev is not None:
                ev[0].record(stream)
            mla.decode_sparse(q, kvt, bt, sl, ix, wl.scale, meta, out=out, lse=lse, workspace=ws)
            if ev is not None:
                ev[1].record(stream)
    else:
        counts = W.algorithmic_counts(wl, kv)
        parts = mla.default_num_parts(wl.h_q, wl.s_q, dev)
        ws = torch.empty((mla.workspace_bytes(wl.batch, wl.s_q, wl.h_q, parts),), dtype=torch.uint8, device=dev)

        def dec(meta, phase):
            if fp8:
                mla.decode_fp8(q, kvt, bt, sl, wl.scale, inp["kv_scale"], wl.causal, meta, out=out, lse=lse,
                               workspace=ws, phase=phase)
            else:
                mla.decode(q, kvt, bt, sl, wl.scale, wl.causal, meta, out=out, lse=lse, workspace=ws, phase=phase)

        def step(ev=None):
            meta = mla.get_metadata(sl, wl.h_q, wl.s_q, num_parts=parts)
            if ev is not None:
                ev[0].record(stream)
            dec(meta, "split")
            if ev is not None:
                ev[1].record(stream)
            dec(meta, "combine")

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if mla.check_status() != 0:
        raise SystemExit("device error status after warm-up of %s/%s" % (name, kv))
    t0 = time.perf_counter()
    step()
    torch.cuda.synchronize()
    steps = int(min(5000, max(20, target_s / max(time.perf_counter() - t0, 1e-6))))
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev) if counts["bytes"] < 2 * L2_BYTES else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    whole = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            whole[i][0].record(stream)
            step(evs[i])
            whole[i][1].record(stream)
        torch.cuda.synchronize()
    if mla.check_status() != 0:
        raise SystemExit("device error status in the timed region of %s/%s" % (name, kv))
    step_ms = statistics.mean(a.elapsed_time(b) for a, b in whole)
    split_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    rec = {"workload": describe(wl, kv) + (", top-%d sparse lists (uniform, sorted)" % topk if topk else ""),
           "kv": kv, "sparse_topk": topk, "steps": steps, "ms_per_step": step_ms,
           "value": counts["bytes"] / (step_ms * 1e-3) / 1e12, "unit": "TB/s",
           "tflops": counts["flops"] / (step_ms * 1e-3) / 1e12,
           "algorithmic_bytes": counts["bytes"], "algorithmic_flops": counts["flops"],
           "l2": "flushed between steps (256 MB write, untimed)" if flush is not None else "inputs larger than L2",
           "clocks": clk.summary()}
    if topk:  # one call launches both kernels: the step time stands for the kernel
        rec["split_ms"] = None
        rec["roofline"] = dict(roofline_fracs(counts["bytes"], counts["flops"], step_ms * 1e-3, peaks),
                               basis="whole sparse call (split + combine)")
    else:
        rec["split_ms"] = split_ms
        rec["roofline"] = dict(roofline_fracs(counts["bytes"], counts["flops"], split_ms * 1e-3, peaks),
                               basis="split kernel")
    del q, kvt, bt, sl, out, lse, ws, flush
    torch.cuda.empty_cache()
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="v3", choices=W.NAMES)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="cache format: bf16 (576 dims) or fp8 (E4M3 latent + bf16 rotary, 640 B/token)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--graph-steps", type=int, default=-1,
                    help="replays of the step captured in a CUDA graph, reported under 'graph' "
                         "(default: as many as --steps; 0: skip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip timing the other workloads (1 GPU only)")
    ap.add_argument("--no-neighbours", action="store_true", help="skip timing the projections and the append")
    ap.add_argument("--max-batch", type=int, default=0,
                    help="keep only the first N sequences (for profiler captures of a smaller slice)")
    ap.add_argument("--topk", type=int, default=0,
                    help="sparse decode (bf16 cache): every query token attends to K positions drawn "
                         "uniformly from its sequence (sorted lists); the headline becomes mla_decode_sparse")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.topk and (args.kv != "bf16" or args.impl != "ours"):
        ap.error("--topk runs the library's sparse decode over the bf16 cache only")

    wl = W.workload(args.workload)
    if args.max_batch and args.max_batch < wl.batch:
        wl = W.custom(args.max_batch, wl.h_q, wl.s_q, wl.seqlens[:args.max_batch], wl.causal, wl.scale,
                      name="%s[:%d]" % (wl.name, args.max_batch))
    counts = W.algorithmic_counts(wl, kv=args.kv)
    fp8 = args.kv == "fp8"
    topk = args.topk
    if topk:
        ixh = W.sparse_indices(wl.seqlens, wl.s_q, topk, seed=0)
        counts = W.sparse_counts(wl, ixh)

    def make_inputs():
        return W.make_inputs_fp8(wl, seed=0, tail="normal") if fp8 else W.make_inputs(wl, seed=0, tail="normal")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        inp = make_inputs()
        run_reference(args, wl, inp, counts)
        return

    import torch
    import mla_decode_attention_14_b200 as mla

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    inp = make_inputs()
    dev = torch.device("cuda", local)
    q = torch.from_numpy(inp["q"]).view(torch.bfloat16).to(dev)
    kv = (torch.from_numpy(inp["kv8"]) if fp8 else torch.from_numpy(inp["kv"]).view(torch.bfloat16)).to(dev)
    bt = torch.from_numpy(inp["block_table"]).to(dev)
    sl = torch.from_numpy(inp["seqlens"]).to(dev)
    num_parts = mla.default_num_parts(wl.h_q, 1 if topk else wl.s_q, dev)
    fixed_cost = mla.default_fixed_cost(wl.h_q, 1 if topk else wl.s_q)
    ws_shape = (wl.batch * wl.s_q, 1) if topk else (wl.batch, wl.s_q)
    ws = torch.empty((mla.workspace_bytes(ws_shape[0], ws_shape[1], wl.h_q, num_parts),), dtype=torch.uint8,
                     device=dev)
    ix = torch.from_numpy(ixh).to(dev) if topk else None
    out = torch.empty((wl.batch, wl.s_q, wl.h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.batch, wl.h_q, wl.s_q), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def decode(q, kv, bt, sl, meta, out, lse, ws, phase):
        if fp8:
            return mla.decode_fp8(q, kv, bt, sl, wl.scale, inp["kv_scale"], wl.causal, meta, out=out, lse=lse,
                                  workspace=ws, phase=phase)
        return mla.decode(q, kv, bt, sl, wl.scale, wl.causal, meta, out=out, lse=lse, workspace=ws, phase=phase)

    def step(ev=None):
        if topk:  # one call launches both kernels: the events bracket the whole call
            meta = mla.get_metadata_sparse(wl.batch, wl.s_q, wl.h_q, topk, num_parts=num_parts, fixed_cost=fixed_cost)
            if ev is not None:
                ev[0].record(stream)
            mla.decode_sparse(q, kv, bt, sl, ix, wl.scale, meta, out=out, lse=lse, workspace=ws)
            if ev is not None:
                ev[1].record(stream)
            return
        meta = mla.get_metadata(sl, wl.h_q, wl.s_q, num_parts=num_parts, fixed_cost=fixed_cost)
        if ev is not None:
            ev[0].record(stream)
        decode(q, kv, bt, sl, meta, out, lse, ws, "split")
        if ev is not None:
            ev[1].record(stream)
        decode(q, kv, bt, sl, meta, out, lse, ws, "combine")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = mla.check_status()
    if st != 0:
        raise SystemExit("device error status %d after warm-up" % st)

    # Inputs smaller than twice the L2 (126 MB) would be served from L2 from the second step on:
    # then every step is timed on its own and a 256 MB write flushes L2 between steps, untimed.
    in_bytes = counts["kv_bytes"] + q.numel() * 2
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)] if flush is not None else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = mla.launch_count()
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
                steps_ev[i][0].record(stream)
            step(evs[i])
            if flush is not None:
                steps_ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    launches = mla.launch_count() - launches0
    if dist is not None:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end) if flush is None else sum(a.elapsed_time(b) for a, b in steps_ev)
    split_ms = [a.elapsed_time(b) for a, b in evs]
    st = mla.check_status()
    if st != 0:
        raise SystemExit("device error status %d in the timed region" % st)

    total_ms, split_avg_ms = max_over_ranks([total_ms, statistics.mean(split_ms)], dev)
    ms_per_step = total_ms / args.steps
    bytes_all = counts["bytes"] * world
    value = job_throughput(counts["bytes"], world, ms_per_step)
    tflops = counts["flops"] * world / (ms_per_step * 1e-3) / 1e12

    # the same step captured once in a CUDA graph and replayed (launch overhead removed); reported
    # beside the eager numbers, which stay the headline (they are the library's own launches)
    graph_ms = None
    graph_steps = args.steps if args.graph_steps < 0 else args.graph_steps
    if flush is None and graph_steps > 0:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        g0.record(stream)
        for _ in range(graph_steps):
            graph.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks([g0.elapsed_time(g1) / graph_steps], dev)[0]
        del graph
        st = mla.check_status()
        if st != 0:
            raise SystemExit("device error status %d in the graph replays" % st)

    # end to end through the host entry point: pinned host inputs in, host outputs out
    e2e = None
    if args.e2e_steps > 0 and not topk:  # the host entry point is the dense decode's
        hd = mla.HostDecoder(wl.batch, wl.s_q, wl.h_q, kv.shape[0], bt.shape[1], device=dev,
                             num_parts=num_parts, fixed_cost=fixed_cost, kv_scale=inp["kv_scale"] if fp8 else None)
        qh = torch.from_numpy(inp["q"]).view(torch.bfloat16).pin_memory()
        kvh = (torch.from_numpy(inp["kv8"]) if fp8 else torch.from_numpy(inp["kv"]).view(torch.bfloat16)).pin_memory()
        bth = torch.from_numpy(inp["block_table"]).pin_memory()
        slh = torch.from_numpy(inp["seqlens"]).pin_memory()
        oh = torch.empty(tuple(out.shape), dtype=torch.bfloat16).pin_memory()
        lh = torch.empty(tuple(lse.shape), dtype=torch.float32).pin_memory()
        for _ in range(2):
            hd(qh, kvh, bth, slh, wl.scale, wl.causal, oh, lh)
        if dist is not None:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            hd(qh, kvh, bth, slh, wl.scale, wl.causal, oh, lh)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / args.e2e_steps], dev)[0]
        h2d = sum(x.numel() * x.element_size() for x in (qh, kvh, bth, slh))
        d2h = oh.numel() * 2 + lh.numel() * 4
        e2e = {"value": bytes_all / (e2e_ms * 1e-3) / 1e12, "unit": "TB/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    neighbours = None if args.no_neighbours or fp8 or topk else neighbour_steps(mla, wl, dev, stream)

    # every other workload (and cache format), 1 GPU only: the same step, timed on its own
    configs = None
    if world == 1 and not args.no_configs and not topk:
        peaks = measured_peaks()
        configs = {}
        for name, kvk, ck in CONFIG_SET:
            if name == args.workload and kvk == args.kv and ck is None:
                continue
            key = "%s_%s" % (name, kvk) + ("_sparse_top%d" % ck if ck else "")
            configs[key] = measure_config(mla, name, kvk, ck, dev, stream, peaks)

    if rank == 0:
        hbm, tfl_burst, tfl_sust, src = measured_peaks()
        ai = counts["flops"] / counts["bytes"]
        ridge = tfl_burst * 1e12 / (hbm * 1e9)
        split_s = split_avg_ms * 1e-3
        ach_gbs = counts["bytes"] / split_s / 1e9
        ach_tf = counts["flops"] / split_s / 1e12
        bound = "hbm" if ai < ridge else "tensor"
        if bound == "hbm":
            roof = {"bound": "hbm", "achieved": ach_gbs, "peak": hbm, "unit": "GB/s", "frac": ach_gbs / hbm}
        else:
            roof = {"bound": "tensor", "achieved": ach_tf, "peak": tfl_burst, "unit": "TFLOP/s",
                    "frac": ach_tf / tfl_burst}
        roof.update({"traffic": None if topk else profiled_traffic(args.kv),
                     "kernel": ("mla sparse decode (split + combine kernels, one call)" if topk else
                                "mla decode split kernel" + (" (fp8 cache)" if fp8 else "")),
                     "peak_source": src + " (MEASURED_PEAKS.json)" if src == "measured" else "fallback",
                     "algorithmic_bytes_per_launch": counts["bytes"], "algorithmic_flops_per_launch": counts["flops"],
                     "launch_ms": split_avg_ms, "hbm_frac": ach_gbs / hbm, "tensor_frac": ach_tf / tfl_burst,
                     "tensor_frac_sustained": ach_tf / tfl_sust,
                     "hbm_frac_spec": ach_gbs / SPEC_HBM_GBS, "tensor_frac_spec": ach_tf / SPEC_BF16_TFLOPS,
                     "spec_peaks": {"hbm_gbs": SPEC_HBM_GBS, "bf16_tflops": SPEC_BF16_TFLOPS}})
        line = {"metric": METRIC_SPARSE if topk else (METRIC_FP8 if fp8 else METRIC), "value": value, "unit": "TB/s", "tflops": tflops,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f16 (fp8 E4M3 cache)" if fp8 else "bf16", "data": "synthetic",
                "config": {"workload": describe(wl, args.kv) + (", top-%d sparse lists (uniform, sorted)" % topk
                                                                 if topk else ""), "kv": args.kv, "topk": topk or None, "batch": wl.batch, "h_q": wl.h_q, "s_q": wl.s_q,
                           "causal": wl.causal, "num_parts": num_parts, "fixed_cost": fixed_cost,
                           "l2": ("inputs larger than L2 (KV cache %.0f MB > 126 MB); no flush" % (counts["kv_bytes"] / 1e6)
                                  if flush is None else "inputs (%.1f MB) fit in L2: a 256 MB write flushes L2 between "
                                  "steps, outside the timed steps" % (in_bytes / 1e6)),
                           "parallelism": "independent batch per GPU" if world > 1 else "1 GPU"},
                "roofline": roof, "clocks": clk.summary(), "e2e": e2e, "gpu_launches": launches,
                "target": {"what": "split kernel >= %.2f of the measured HBM peak on v3" % TARGET_HBM_FRAC,
                           "hbm_frac": ach_gbs / hbm,
                           "met": bool(args.workload == "v3" and ach_gbs / hbm >= TARGET_HBM_FRAC)},
                "configs": configs,
                "neighbours": neighbours,
                "graph": None if graph_ms is None else {
                    "ms_per_step": graph_ms, "value": job_throughput(counts["bytes"], world, graph_ms), "unit": "TB/s",
                    "note": "the same step (metadata + split + combine) captured once in a CUDA graph and replayed"}}
        if world == 1 and not args.no_cpu_baseline and not topk:
            line["cpu_baseline"] = cpu_baseline(wl, inp, kv=args.kv)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
