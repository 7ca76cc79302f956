"""Benchmark of the TurboQuant decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W]
                    [--workload serving|gqa|qjl|long|tiny|affine]
                    [--impl ours|reference] [--no-dense] [--no-cpu-baseline]
                    [--no-long-context] [--lutmm]

A step is one pass of the whole hot path over one batch: tq_quantize_append of
one new token per (batch row, KV head), then tq_decode_attention of every query
head over the compressed cache.  Caches are pre-filled (bulk append, outside
the timed region) with seeded synthetic K/V of the workload's shape.  Timing:
W untimed warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, measured with CUDA events on the launching stream;
steps rotate over cache replicas whose total size exceeds 4x L2, so every step
reads its cache from HBM.  Steps are replayed from CUDA graphs (one per
replica) so that host launch latency does not leak into the device time.

The JSON line reports `value` = algorithmic bytes of the step (packed cache
read by the decode, queries, outputs, appended K/V and their codes) / device
time, in GB/s, plus ctx-tokens/s, the decode call's roofline against the
measured HBM copy bandwidth, bulk quantize Mvec/s, an end-to-end figure through
host buffers, the FP16/BF16 dense decode baselines on the same GPU, and the CPU
oracle timed on the host as a baseline.  That oracle leg also checks the
benchmark's own inputs: the unit it encodes and decodes goes through the
library too, and `cpu_baseline.parity` reports the largest per-row error of
the GPU output against the oracle's (bar: 2e-3 of the row's largest value).
`cpu_baseline.rates_by_workload` gives the oracle's quantize and decode rates
for every workload, on one thread and on all, each on a bounded sample.  The default workload is `serving`
(32 ragged rows of 8k-64k tokens); the line also carries `long_context`: the
decode calls of the 131k-token `qjl` and 524k-token `long` workloads with their
own roofline fractions and dense baselines.  `roofline.traffic` (ncu DRAM
bytes) and `roofline.issue` (issue utilisation) come from committed ncu
summaries and read null once the decode sources differ from the captured ones.

With several GPUs (torchrun) every rank runs an independent replica of the
workload ("replicas only": the path has no exchange step); `value` is the sum
over ranks divided by the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from turboquant_kv_cache_rht_b200 import workloads as wl  # noqa: E402

METRIC = "fused TQ decode-attention GB/s & % HBM peak; ctx-tokens/s; quantize Mvec/s"
FALLBACK_HBM_GBS = 6650.0


# DRAM bytes (read + write) of one tq_decode_attention call (decode + combine
# launches), per workload, from one ncu capture of `bench.py --workload <name>`
# (dram__bytes_read.sum + dram__bytes_write.sum of both kernels).  Each entry
# carries the digest of the decode sources it was taken with; once the kernel
# sources change the figure no longer describes them and is reported as null.
DECODE_SOURCES = ("tq_internal.cuh", "tq_decode_impl.cuh", "tq_decode.cu", "tq_decode_d64.cu", "tq_decode_d128.cu",
                  "tq_decode_d256.cu", "tq_decode_affine_d64.cu", "tq_decode_affine_d128.cu",
                  "tq_decode_affine_d256.cu")
DECODE_TRAFFIC: dict[str, tuple[int, str]] = {
    "gqa": (31446272, "fb0b4675e697c407"),
    "qjl": (566612992, "fb0b4675e697c407"),
    "long": (352942080, "fb0b4675e697c407"),
    "serving": (1102108672, "fb0b4675e697c407"),
    "affine": (38473728, "fb0b4675e697c407"),
}


def decode_sources_digest() -> str:
    """Digest of the decode sources' code.  Comments and blank space are
    dropped first, so that an edit of the documentation alone keeps the
    recorded traffic (the sources hold no string with a comment marker)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "turboquant_kv_cache_rht_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = "\n".join(ln.strip() for ln in text.splitlines() if ln.strip())
        h.update(name.encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


def decode_traffic(workload: str):
    entry = DECODE_TRAFFIC.get(workload)
    if entry is None or entry[1] != decode_sources_digest():
        return None
    return entry[0]


# Issue utilisation of the decode kernel per workload, from the ncu --set full
# capture summarised in profiles/decode_kernel_<workload>.md: issue-active %
# of active cycles, warp instructions per (token, KV head), warps active %.
# Keyed, like the traffic, to the digest of the decode sources it describes.
DECODE_PROFILE: dict[str, tuple[dict, str]] = {
    "affine": ({"issue_active_pct": 38.1, "warp_inst_per_token_head": 32.16, "warps_active_pct": 12.3}, "fb0b4675e697c407"),
    "gqa": ({"issue_active_pct": 41.4, "warp_inst_per_token_head": 33.09, "warps_active_pct": 17.6}, "fb0b4675e697c407"),
    "long": ({"issue_active_pct": 55.9, "warp_inst_per_token_head": 41.47, "warps_active_pct": 12.3}, "fb0b4675e697c407"),
    "qjl": ({"issue_active_pct": 64.3, "warp_inst_per_token_head": 35.04, "warps_active_pct": 17.3}, "fb0b4675e697c407"),
    "serving": ({"issue_active_pct": 65.2, "warp_inst_per_token_head": 23.64, "warps_active_pct": 17.0}, "fb0b4675e697c407"),
}


def decode_profile(workload: str):
    entry = DECODE_PROFILE.get(workload)
    if entry is None or entry[1] != decode_sources_digest():
        return None
    return dict(entry[0], source=f"profiles/decode_kernel_{workload}.md")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# byte model (algorithmic bytes; see the design notes)
# ---------------------------------------------------------------------------
def meta_bytes(w: wl.Workload) -> int:
    """fp16 metadata per stored vector: the norm, or the affine codec's
    (scale, bias) per group of 64 channels."""
    return 4 * (w.head_dim // 64) if w.codebook == "affine" else 2


def token_bytes(w: wl.Workload) -> int:
    """Packed bytes one decode reads per (token, KV head)."""
    d = w.head_dim
    b = w.k_bits * d // 8 + w.v_bits * d // 8 + 2 * meta_bytes(w)
    if w.qjl:
        b += d // 8 + 2
    return b


def step_bytes(w: wl.Workload, lengths) -> dict:
    esz = {"f32": 4, "bf16": 2, "f16": 2}[w.dtype]
    d = w.head_dim
    cache = sum(lengths) * w.kv_heads * token_bytes(w)
    q_out = w.batch * w.q_heads * d * (esz + 4)
    vec_out = (w.k_bits + w.v_bits) * d // 8 + 2 * meta_bytes(w) + ((d // 8 + 2) if w.qjl else 0)
    append = w.batch * w.kv_heads * (2 * d * esz + vec_out)
    return {"decode": cache + q_out, "append": append, "total": cache + q_out + append}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.out = None
        try:
            bus = torch.cuda.get_device_properties(device_index).pci_bus_id
            sel = ["--id=" + bus] if bus else ["-i", "0"]
        except Exception:
            sel = ["-i", "0"]
        self.cmd = ["nvidia-smi", *sel, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                    "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self) -> dict:
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        rows = []
        for ln in self.out.strip().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, p in rows for i in range(4) if p[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def replica_plan(w: wl.Workload, steps_total: int, l2_bytes: int) -> dict:
    """Cache replicas (total above 4x L2), appends per replica, capacity and
    the decode's max_ctx for a run of `steps_total` appended steps."""
    lengths = wl.context_lengths(w)
    per_replica = sum(lengths) * w.kv_heads * token_bytes(w)
    replicas = max(1, math.ceil(4 * l2_bytes / max(per_replica, 1)) + (0 if per_replica > 4 * l2_bytes else 1))
    replicas = min(replicas, 64)
    visits = math.ceil(steps_total / replicas) + 8
    return {"lengths": lengths, "replicas": replicas,
            "capacity": (max(lengths) + visits + 15) // 16 * 16, "max_ctx": max(lengths) + visits}


def default_steps_total(steps: int = 200, warmup: int = 10) -> int:
    """Appends one bench run makes per workload (timed + e2e steps + warm-up)."""
    return 2 * steps + warmup


def reduce_over_ranks(ms: float, byts: float, tokens: float, device) -> tuple[float, float, float]:
    """Max of the device times and sums of the work over all ranks."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms, byts, tokens
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    u = torch.tensor([byts, tokens], device=device, dtype=torch.float64)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u[0].item()), float(u[1].item())


class State:
    """Caches (replicas), per-step inputs and outputs of one workload on one GPU."""

    def __init__(self, w: wl.Workload, steps_total: int, device):
        from turboquant_kv_cache_rht_b200 import tq
        self.tq = tq
        self.w = w
        self.dev = device
        self.cb = tq.Codebook(w.head_dim, w.k_bits, w.v_bits, w.qjl, w.rht_seed, codebook=w.codebook)
        plan = replica_plan(w, steps_total, torch.cuda.get_device_properties(device).L2_cache_size)
        self.lengths = plan["lengths"]
        self.replicas = plan["replicas"]
        self.capacity = plan["capacity"]
        self.max_ctx = plan["max_ctx"]
        self.caches = [tq.Cache(self.cb, w.batch, w.kv_heads, self.capacity, device)
                       for _ in range(self.replicas)]
        self._prefill()
        self.q = wl.queries(w, 0).to(device)
        kn, vn = wl.kv_step(w, 0)
        self.k_new, self.v_new = kn.to(device).contiguous(), vn.to(device).contiguous()
        self.out = torch.empty(w.batch, w.q_heads, w.head_dim, dtype=torch.float32, device=device)
        ws = tq.tq_decode_workspace_bytes(self.cb, w.batch, w.q_heads, w.kv_heads, self.max_ctx)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)

    def _prefill(self):
        tq, w = self.tq, self.w
        first = self.caches[0]
        # bulk append one KV head at a time on the host side to bound host memory,
        # then set each row's length (rows shorter than the longest keep zeros past it)
        tmax = max(self.lengths)
        for h in range(w.kv_heads):
            kh = torch.zeros(w.batch, 1, tmax, w.head_dim, dtype=w.torch_dtype)
            vh = torch.zeros_like(kh)
            for b in range(w.batch):
                k, v = wl.kv_unit(w, b, h, self.lengths[b])
                kh[b, 0, :self.lengths[b]] = k
                vh[b, 0, :self.lengths[b]] = v
            tmp = tq.Cache(self.cb, w.batch, 1, self.capacity, self.dev)
            tq.tq_quantize_append(self.cb, tmp, kh.to(self.dev), vh.to(self.dev))
            for name in ("k_codes", "v_codes", "k_signs", "k_norm", "v_norm", "k_rnorm"):
                src = getattr(tmp, name)
                if src is not None:
                    getattr(first, name)[:, h].copy_(src[:, 0])
            del tmp
        first.seq_lens.copy_(torch.tensor(self.lengths, dtype=torch.int32))
        for c in self.caches[1:]:
            for name in ("k_codes", "v_codes", "k_signs", "k_norm", "v_norm", "k_rnorm", "seq_lens"):
                src = getattr(first, name)
                if src is not None:
                    getattr(c, name).copy_(src)
        torch.cuda.synchronize(self.dev)

    def step(self, r: int, stream=None):
        tq = self.tq
        c = self.caches[r]
        tq.tq_quantize_append(self.cb, c, self.k_new, self.v_new, stream=stream)
        tq.tq_decode_attention(self.cb, c, self.q, out=self.out, max_ctx=self.max_ctx,
                               workspace=self.ws, stream=stream)


def run_gpu(args, rank: int, world: int) -> dict | None:
    import torch.distributed as dist
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = wl.WORKLOADS[args.workload]
    K, W = args.steps, args.warmup
    st = State(w, default_steps_total(K, W), dev)
    tq = st.tq
    stream = torch.cuda.current_stream(dev)

    # warm-up (also configures kernels before capture)
    for i in range(W):
        st.step(i % st.replicas)
    torch.cuda.synchronize(dev)

    graphs = []
    cap_stream = torch.cuda.Stream(dev)
    for r in range(st.replicas):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            st.step(r)
        graphs.append(g)
    torch.cuda.synchronize(dev)
    for r in range(st.replicas):   # one graph replay each before timing
        graphs[r].replay()
    torch.cuda.synchronize(dev)

    lengths_before = [int(x) for x in st.caches[0].seq_lens.cpu()]
    visit = [0] * st.replicas
    for r in range(st.replicas):
        visit[r] = int(st.caches[r].seq_lens[0].item()) - st.lengths[0]

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda._sleep(2_000_000)          # let the host queue ahead of the device
        e0.record(stream)
        for s in range(K):
            graphs[s % st.replicas].replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    # bytes of the timed steps: replica r's contexts grew by one token per visit
    total_bytes = 0
    ctx_tokens = 0
    for s in range(K):
        r = s % st.replicas
        grow = visit[r] + 1 + s // st.replicas
        lens = [L + grow for L in st.lengths]
        total_bytes += step_bytes(w, lens)["total"]
        ctx_tokens += sum(lens)
    ms_max, bytes_all, tokens_all = reduce_over_ranks(ms, float(total_bytes), float(ctx_tokens), dev)

    # ---- each call alone, back to back on the launching stream (host queued
    #      ahead): one append per replica, then decode calls over the replicas
    n_dec = max(st.replicas, 16)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    torch.cuda._sleep(2_000_000)
    ev[0].record(stream)
    for r in range(st.replicas):
        tq.tq_quantize_append(st.cb, st.caches[r], st.k_new, st.v_new)
    ev[1].record(stream)
    ev[2].record(stream)
    for i in range(n_dec):
        tq.tq_decode_attention(st.cb, st.caches[i % st.replicas], st.q, out=st.out,
                               max_ctx=st.max_ctx, workspace=st.ws)
    ev[3].record(stream)
    torch.cuda.synchronize(dev)
    app_us = 1e3 * ev[0].elapsed_time(ev[1]) / st.replicas
    dec_us = 1e3 * ev[2].elapsed_time(ev[3]) / n_dec
    lens_now = [int(x) for x in st.caches[0].seq_lens.cpu()]
    dec_bytes = step_bytes(w, lens_now)["decode"]

    # ---- bulk quantize throughput (prefill-style append of a whole context)
    q_mvec = bulk_quantize_mvec(st, dev)

    # ---- end to end through host buffers: pinned inputs in, result out, every step
    e2e = end_to_end(st, dev, K, stream)

    dense = None
    if not args.no_dense and world == 1:
        dense = dense_baselines(w, st, dev)
    lutmm = lut_matmul_bench(dev, peaks()[0]) if (args.lutmm and world == 1) else None

    del graphs
    peak, peak_kind = peaks()
    long_ctx = None
    if world == 1 and not args.no_long_context:
        del st.caches
        torch.cuda.empty_cache()
        long_ctx = {name: long_context_leg(name, dev, peak, dense=not args.no_dense)
                    for name in ("qjl", "long") if name != w.name}
    achieved = dec_bytes / (dec_us * 1e-6) / 1e9
    hbm_frac = achieved / peak
    res = {
        "metric": METRIC,
        "value": round(bytes_all / (ms_max * 1e-3) / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_max / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8 codes, f32 accumulate",
        "data": "synthetic (seeded Gaussian K/V with outlier channels)",
        "config": {"workload": w.name, "description": w.description, "batch": w.batch,
                   "q_heads": w.q_heads, "kv_heads": w.kv_heads, "head_dim": w.head_dim,
                   "context": st.lengths[0] if w.context else "ragged", "k_bits": w.k_bits,
                   "v_bits": w.v_bits, "qjl": w.qjl, "codebook": w.codebook,
                   "parallelism": f"replicas x{world}",
                   "l2": f"{st.replicas} rotating cache replicas "
                         f"({st.replicas * sum(st.lengths) * w.kv_heads * token_bytes(w) / 1e6:.0f} MB, > 4x L2)"},
        "ctx_tokens_per_s": round(tokens_all / (ms_max * 1e-3), 1),
        "hbm_frac_of_step": round(bytes_all / (ms_max * 1e-3) / 1e9 / peak / world, 4),
        "decode_us": round(dec_us, 3),
        "append_us": round(app_us, 3),
        "quantize_mvec_s": q_mvec,
        "roofline": {"bound": "hbm", "kernel": "tq_decode_attention (decode + combine launches)",
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(hbm_frac, 4), "traffic": decode_traffic(w.name),
                     "algorithmic_bytes_per_launch": dec_bytes,
                     "issue": decode_profile(w.name)},
        "e2e": e2e,
        "gpu_launches": 3 * K,
        "clocks": clk.summary(),
    }
    if dense is not None:
        res["dense_baseline"] = dense
    if lutmm is not None:
        res["lut_matmul"] = lutmm
    if long_ctx:
        res["long_context"] = long_ctx
    return res


def long_context_leg(name: str, dev, peak: float, dense: bool = True) -> dict:
    """Decode-call time of one long-context workload (caches prefilled as in
    the main leg, calls back to back over replicas > 4x L2), its fraction of
    the HBM roofline, and the dense bf16 decode kernels on the same shape."""
    w = wl.WORKLOADS[name]
    st = State(w, 64, dev)
    st_decode_us(st, dev, n=4)        # first calls configure the kernel of this shape
    us = st_decode_us(st, dev, n=max(st.replicas, 16))
    lens = [int(x) for x in st.caches[0].seq_lens.cpu()]
    byts = step_bytes(w, lens)["decode"]
    gbs = byts / (us * 1e-6) / 1e9
    res = {"description": w.description, "decode_us": round(us, 2), "gb_s": round(gbs, 1),
           "frac": round(gbs / peak, 4), "ctx_tokens_per_s": round(sum(lens) / (us * 1e-6), 1),
           "algorithmic_bytes_per_launch": byts}
    if dense:
        d = dense_baselines(w, st, dev)
        res["dense_baseline"] = d
    del st
    torch.cuda.empty_cache()
    return res


def bulk_quantize_mvec(st: State, dev) -> dict:
    """Append one full context of K/V (all heads) into a fresh cache; Mvec/s."""
    tq, w = st.tq, st.w
    n = min(max(st.lengths), 32768)
    k, v = wl.kv_unit(w, 0, 0, n)
    kk = k.to(dev)[None, None].expand(w.batch, w.kv_heads, n, w.head_dim).contiguous()
    vv = v.to(dev)[None, None].expand(w.batch, w.kv_heads, n, w.head_dim).contiguous()
    cap = (n + 15) // 16 * 16
    c = tq.Cache(st.cb, w.batch, w.kv_heads, cap, dev)
    times = []
    for i in range(4):
        c.seq_lens.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        tq.tq_quantize_append(st.cb, c, kk, vv)
        e1.record()
        torch.cuda.synchronize(dev)
        if i:
            times.append(e0.elapsed_time(e1))
    vecs = 2 * w.batch * w.kv_heads * n
    ms = statistics.median(times)
    esz = kk.element_size()
    lay = st.cb.layout
    byts = vecs // 2 * (2 * w.head_dim * esz + lay.k_code_bytes + lay.v_code_bytes + 2 * meta_bytes(w) +
                        (lay.k_sign_bytes + 2 if w.qjl else 0))
    return {"vectors": vecs, "ms": round(ms, 4), "mvec_s": round(vecs / (ms * 1e-3) / 1e6, 1),
            "gb_s": round(byts / (ms * 1e-3) / 1e9, 1)}


def end_to_end(st: State, dev, K: int, stream) -> dict:
    """Same step through the public API with pinned host buffers copied in and out."""
    tq, w = st.tq, st.w
    hk = st.k_new.cpu().pin_memory()
    hv = st.v_new.cpu().pin_memory()
    hq = st.q.cpu().pin_memory()
    hout = torch.empty(st.out.shape, dtype=torch.float32).pin_memory()
    dk, dv, dq = torch.empty_like(st.k_new), torch.empty_like(st.v_new), torch.empty_like(st.q)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    tokens = 0
    byts = 0
    for s in range(K):
        r = s % st.replicas
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dq.copy_(hq, non_blocking=True)
        c = st.caches[r]
        tq.tq_quantize_append(st.cb, c, dk, dv)
        tq.tq_decode_attention(st.cb, c, dq, out=st.out, max_ctx=st.max_ctx, workspace=st.ws)
        hout.copy_(st.out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    lens = [int(x) for x in st.caches[0].seq_lens.cpu()]
    byts = K * step_bytes(w, lens)["total"]
    ms = e0.elapsed_time(e1)
    h2d = hk.numel() * hk.element_size() + hv.numel() * hv.element_size() + hq.numel() * hq.element_size()
    d2h = hout.numel() * hout.element_size()
    return {"value": round(byts / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms / K, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def lut_matmul_bench(dev, peak_gbs: float, rows: int = 16384, k: int = 8192, bits: int = 4,
                     head_dim: int = 128, replicas: int = 8) -> dict:
    """The weights-regime LUT matmul on a synthetic [rows, k] layer (seeded N(0,1)
    weights): packed bytes per call over the back-to-back call time, for 1 and 16
    inputs, beside torch's dense bf16 product with the same weights.  The codes are
    replicated (replicas x codes > 4x L2) and calls rotate over them."""
    from turboquant_kv_cache_rht_b200 import tq
    g = torch.Generator(device=dev).manual_seed(20250)
    wt = torch.randn(rows, k, generator=g, device=dev).bfloat16()
    cb = tq.Codebook(head_dim, bits, bits, seed=5)
    qw = tq.QuantizedWeights(cb, wt)
    copies = [qw] + [qw.copy() for _ in range(replicas - 1)]
    packed = qw.codes.numel() + qw.norms.numel() * 2

    def timed(fn, n):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize(dev)
        torch.cuda._sleep(1_000_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n):
            fn(i)
        e1.record()
        torch.cuda.synchronize(dev)
        return 1e3 * e0.elapsed_time(e1) / n

    res = {"shape": [rows, k], "bits": bits, "head_dim": head_dim, "packed_bytes": packed}
    dense_w = [wt] + [wt.clone() for _ in range(2)]   # 3 x 256 MB bf16 copies, > 4x L2
    for m in (1, 16):
        x = torch.randn(m, k, generator=g, device=dev).bfloat16()
        us = timed(lambda i: copies[i % replicas].matmul(x), 4 * replicas)
        dus = timed(lambda i: torch.matmul(x, dense_w[i % 3].T), 12)
        gbs = (packed + x.numel() * 2 + m * rows * 4) / (us * 1e-6) / 1e9
        res[f"m{m}"] = {"us": round(us, 2), "gb_s": round(gbs, 1), "frac_of_peak": round(gbs / peak_gbs, 4),
                        "dense_bf16_us": round(dus, 2), "speedup_vs_dense": round(dus / us, 2)}
    del copies, dense_w, wt
    torch.cuda.empty_cache()
    return res


def dense_baselines(w: wl.Workload, st: State, dev) -> dict:
    """Unquantized bf16 decode attention on the same GPU: flash-attn's KV-cache
    kernel and torch SDPA, on dense caches of the same shape (replicated past L2)."""
    if w.batch * w.kv_heads * max(st.lengths) * w.head_dim * 2 * 2 > 40e9:
        return {"skipped": "dense cache too large"}
    res = {}
    T = max(st.lengths)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    one = (torch.randn(w.batch, T, w.kv_heads, w.head_dim, generator=g)).to(torch.bfloat16).to(dev)
    dense_bytes = one.numel() * 2 * 2
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    reps = max(1, min(8, math.ceil(4 * l2 / dense_bytes) + 1)) if dense_bytes < 4 * l2 else 1
    ks = [one] + [one.clone() for _ in range(reps - 1)]
    vs = [one.clone() for _ in range(reps)]
    q = st.q.to(torch.bfloat16).reshape(w.batch, 1, w.q_heads, w.head_dim)
    seqlens = torch.tensor(st.lengths, dtype=torch.int32, device=dev)

    def timeit(fn, n=20):
        for i in range(3):
            fn(i % reps)
        torch.cuda.synchronize(dev)
        torch.cuda._sleep(2_000_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n):
            fn(i % reps)
        e1.record()
        torch.cuda.synchronize(dev)
        return 1e3 * e0.elapsed_time(e1) / n

    try:
        from flash_attn import flash_attn_with_kvcache
        res["flash_attn_us"] = round(timeit(lambda i: flash_attn_with_kvcache(
            q, ks[i], vs[i], cache_seqlens=seqlens)), 2)
    except Exception as e:  # library baseline only
        res["flash_attn_error"] = repr(e)[:200]
    try:
        qs = q.transpose(1, 2).contiguous()
        kt = [k.transpose(1, 2).contiguous() for k in ks]
        vt = [v.transpose(1, 2).contiguous() for v in vs]
        if len(set(st.lengths)) == 1:
            res["sdpa_us"] = round(timeit(lambda i: torch.nn.functional.scaled_dot_product_attention(
                qs, kt[i], vt[i], enable_gqa=True)), 2)
    except Exception as e:
        res["sdpa_error"] = repr(e)[:200]
    times = [v for k, v in res.items() if k.endswith("_us")]
    if times:
        best = min(times)
        res["best_dense_us"] = best
        res["dense_bytes"] = dense_bytes
        res["tq_decode_us"] = round(st_decode_us(st, dev), 2)
        res["tq_speedup_vs_best_dense"] = round(best / res["tq_decode_us"], 3)
    return res


def st_decode_us(st: State, dev, n=None) -> float:
    tq = st.tq
    n = n or max(st.replicas, 8)
    torch.cuda.synchronize(dev)
    torch.cuda._sleep(2_000_000)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        tq.tq_decode_attention(st.cb, st.caches[i % st.replicas], st.q, out=st.out,
                               max_ctx=st.max_ctx, workspace=st.ws)
    e1.record()
    torch.cuda.synchronize(dev)
    return 1e3 * e0.elapsed_time(e1) / n


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and the reference arm)
# ---------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


class OracleUnit:
    """One (batch row 0, KV head 0) unit of the workload, encoded by the oracle."""

    def __init__(self, w: wl.Workload):
        import numpy as np

        import oracle as o
        self.o, self.np, self.w = o, np, w
        self.T = wl.context_lengths(w)[0]
        d = w.head_dim
        self.affine = w.codebook == "affine"
        if w.codebook == "sphere":
            self.ck, self.bk = o.sphere_codebook(w.k_bits, d)
            self.cv, self.bv = o.sphere_codebook(w.v_bits, d)
        elif not self.affine:
            self.ck, self.bk = o.codebook(w.k_bits)
            self.cv, self.bv = o.codebook(w.v_bits)
        self.s1 = o.rotation_signs(w.rht_seed, d)
        self.s2 = o.rotation_signs(w.rht_seed, d, second=True) if w.qjl else None
        k, v = wl.kv_unit(w, 0, 0, self.T)
        self.ek, self.ev = self._encode(k.float().numpy(), v.float().numpy())
        kn, vn = wl.kv_step(w, 0)
        self.k_new = kn[0, 0].float().numpy()
        self.v_new = vn[0, 0].float().numpy()
        self.q = wl.queries(w, 0)[0, :w.group].float().numpy().astype(np.float64)

    def _encode(self, k, v):
        o, w = self.o, self.w
        if self.affine:
            return o.affine_encode(k, w.k_bits, self.s1, self.s2), o.affine_encode(v, w.v_bits)
        return (o.encode(k, self.s1, self.ck, self.bk, w.k_bits, self.s2),
                o.encode(v, self.s1, self.cv, self.bv, w.v_bits))

    def step(self):
        """Append one token (encode K and V) and decode the unit's G heads."""
        o, np = self.o, self.np
        ek1, ev1 = self._encode(self.k_new, self.v_new)
        if self.affine:
            cat = lambda a, b: {key: np.concatenate([a[key], b[key]]) for key in a if key in b}
            return o.affine_decode_attention(self.q, self.s1, cat(self.ek, ek1), cat(self.ev, ev1),
                                             s2=self.s2)
        kw = {}
        if self.s2 is not None:
            kw = dict(s2=self.s2, k_sign_bits=np.concatenate([self.ek["sign_bits"], ek1["sign_bits"]]),
                      k_rnorm16=np.concatenate([self.ek["rnorm16"], ek1["rnorm16"]]))
        return o.decode_attention(self.q, self.s1, np.concatenate([self.ek["idx"], ek1["idx"]]),
                                  np.concatenate([self.ek["norm16"], ek1["norm16"]]), self.ck,
                                  np.concatenate([self.ev["idx"], ev1["idx"]]),
                                  np.concatenate([self.ev["norm16"], ev1["norm16"]]), self.cv, **kw)

    def bytes_per_step(self) -> int:
        w = self.w
        esz = {"f32": 4, "bf16": 2, "f16": 2}[w.dtype]
        d = w.head_dim
        vec_out = (w.k_bits + w.v_bits) * d // 8 + 2 * meta_bytes(w) + ((d // 8 + 2) if w.qjl else 0)
        return (self.T + 1) * token_bytes(w) + w.group * d * (esz + 4) + 2 * d * esz + vec_out


def unit_parity(u: "OracleUnit", ref) -> dict:
    """The benchmark's own inputs checked against the oracle: the unit the
    oracle leg encodes (batch row 0, KV head 0: its whole context, then the
    first step's appended token) goes through the library on the GPU as well,
    and each of the G output rows must be within the decode tolerance of the
    oracle's (max |gpu - oracle| <= 2e-3 * max |oracle| per row).  A failure
    is reported in the line and on stderr; it does not stop the benchmark."""
    import numpy as np
    from turboquant_kv_cache_rht_b200 import tq
    w = u.w
    try:
        dev = torch.device("cuda", torch.cuda.current_device())
        cb = tq.Codebook(w.head_dim, w.k_bits, w.v_bits, w.qjl, w.rht_seed, codebook=w.codebook)
        cache = tq.Cache(cb, 1, 1, (u.T + 1 + 15) // 16 * 16, dev)
        k, v = wl.kv_unit(w, 0, 0, u.T)
        tq.tq_quantize_cache(cb, cache, k[None, None].to(dev), v[None, None].to(dev))
        kn, vn = wl.kv_step(w, 0)
        tq.tq_quantize_append(cb, cache, kn[0:1, 0:1].contiguous().to(dev),
                              vn[0:1, 0:1].contiguous().to(dev))
        q = wl.queries(w, 0)[0:1, :w.group].contiguous().to(dev)
        got = tq.tq_decode_attention(cb, cache, q)[0].double().cpu().numpy()
        status = int(cache.status.item())
        ref = np.asarray(ref, np.float64)
        err = max(float(np.abs(got[r] - ref[r]).max() / np.abs(ref[r]).max()) for r in range(ref.shape[0]))
        res = {"unit": "batch row 0, KV head 0", "tokens": u.T + 1, "rows": int(ref.shape[0]),
               "max_rel_err": float(f"{err:.3g}"), "tol": 2e-3, "status": status,
               "ok": bool(err <= 2e-3 and status == 0)}
    except Exception as e:  # the check must not cost the measurement
        res = {"error": f"{type(e).__name__}: {e}", "ok": False}
    if not res["ok"]:
        print(f"bench: parity check against the oracle failed: {res}", file=sys.stderr, flush=True)
    return res


def cpu_baseline(w: wl.Workload, budget_s: float = 10.0) -> dict:
    u = OracleUnit(w)
    parity = unit_parity(u, u.step())
    t0 = time.perf_counter()
    n = 0
    while True:
        u.step()
        n += 1
        el = time.perf_counter() - t0
        if el > budget_s or n >= 200:
            break
    res = {"value": round(n * u.bytes_per_step() / el / 1e9, 4), "unit": "GB/s",
           "cores": blas_threads(), "kind": "oracle",
           "sample": f"{n} steps of one (batch row, KV head) unit: encode 1 appended K and V, "
                     f"decode {w.group} query heads over {u.T + 1} tokens (numpy, float64 attention)",
           "host_cpus": os.cpu_count()}
    res.update(oracle_rates(u))
    res["rates_by_workload"] = oracle_rates_by_workload()
    res["parity"] = parity
    return res


def oracle_rates_by_workload(context: int = 8192, budget_s: float = 0.3) -> dict:
    """The oracle's quantize and decode rates (as ``oracle_rates``) for every
    workload, each on a bounded sample: batch row 0, KV head 0 at `context`
    tokens (the workload's own context when shorter).  Per-token and
    per-vector costs do not depend on the context length beyond that."""
    out = {}
    for name, w in sorted(wl.WORKLOADS.items()):
        try:  # a reported baseline: a failure here must not cost the line
            u = OracleUnit(wl.with_sizes(w, context=min(context, w.context or context)))
            out[name] = dict(oracle_rates(u, budget_s), sample_tokens=u.T + 1)
        except Exception as e:
            out[name] = {"error": f"{type(e).__name__}: {e}"}
    return out


def oracle_rates(u: "OracleUnit", budget_s: float = 2.0) -> dict:
    """The oracle's quantize rate (Mvec/s: K and V vectors, keys with the QJL
    sketch when the workload has it) and decode rate (ctx-tokens/s of one KV
    head's G query heads), on all BLAS threads and on one thread."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        threadpool_limits = None
    w = u.w
    k, v = wl.kv_unit(w, 0, 0, 1024)
    kf, vf = k.float().numpy(), v.float().numpy()

    def rate(fn, units):
        fn()
        t0, n = time.perf_counter(), 0
        while True:
            fn()
            n += 1
            el = time.perf_counter() - t0
            if el > budget_s:
                return n * units / el

    def measure():
        return {"quantize_mvec_s": round(rate(lambda: u._encode(kf, vf), 2 * len(kf)) / 1e6, 5),
                "decode_ctx_tokens_s": round(rate(u.step, u.T + 1), 1)}

    out = {"all_threads": measure()}
    if threadpool_limits is not None:
        with threadpool_limits(limits=1):
            out["one_thread"] = measure()
    return out


def run_reference(args, rank: int) -> dict | None:
    if rank != 0:
        return None
    w = wl.WORKLOADS[args.workload]
    u = OracleUnit(w)
    for _ in range(args.warmup):
        u.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        u.step()
    el = time.perf_counter() - t0
    value = args.steps * u.bytes_per_step() / el / 1e9
    cores = blas_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 codec, f64 attention", "data": "synthetic",
        "config": {"workload": w.name, "description": w.description,
                   "sample": "one (batch row, KV head) unit of the workload per step"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: encode 1 appended K and V, decode {w.group} query heads "
                                   f"over {u.T + 1} tokens of one KV head",
                         "rates_by_workload": oracle_rates_by_workload()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="serving", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-long-context", action="store_true",
                    help="skip the decode-call timing of the qjl and long workloads")
    ap.add_argument("--lutmm", action="store_true",
                    help="also time the weights-regime LUT matmul on a 16384 x 8192 layer")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.gpus == 1 else 1)))

    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_gpu(args, rank, world)
    if rank == 0 and res is not None:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(wl.WORKLOADS[args.workload])
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
