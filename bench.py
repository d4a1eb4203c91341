"""Benchmark of the MXFP4 MoE block-verify step on B200.

One step = the whole hot path over one drafted batch: moe_route_permute ->
mxfp4_moe_ffn -> moe_combine (per MoE layer; stacked layers add a
moe_rms_norm before and the residual in the combine) -> block acceptance
(block_accept_greedy and/or block_accept_rejection).  The headline line is
the batch-1 verify workload (1 sequence x 8-token block, one MoE layer of
hidden 7168, expert intermediate 2048, 256 experts, top-8; greedy acceptance
over a 152064-token vocabulary).  Metric: verified tokens/s (= S*K / step
time), with the expert FFN's roofline beside it.  On one GPU the same line
carries `per_config`: the other seeded workloads (tiny, serving batch, DFlash
block-16 with rejection acceptance, the 8-layer stack) each timed the same
way with its own roofline, plus the MXFP4 weight quantiser.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--no-per-config] [--no-cpu-baseline]

Multi-GPU: every rank verifies its own independent batch (the path has no
exchange step); value = all ranks' tokens / the slowest rank's time.
--impl reference times the CPU oracle (the reference arm of this repository)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mxfp4_moe_block_b200 import synth  # noqa: E402

METRIC = "verified tokens/s (MXFP4 MoE block-verify step)"
UNIT = "tokens/s"
PER_CONFIG = ("tiny", "serving", "dflash16", "multilayer")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="batch1", choices=list(synth.SHAPES))
    ap.add_argument("--variant", type=int, default=0,
                    help="FFN kernel: 0 auto, 1 FMA, 2 tensor, 3 kind::mxf8f6f4, 4 kind::mxf4, "
                         "5 fused, 6 kind::mxf8f6f4 on CTA pairs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches only")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--per-config", default=",".join(PER_CONFIG),
                    help="comma-separated workloads for the per_config object (the "
                         "quantiser is always measured; 'none' for it alone)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the expert count (smaller cases for profiler captures)")
    return ap.parse_args(argv)


def load_peaks():
    """Roofline denominators: the machine's measured copy bandwidth and dense bf16
    GEMM rate (MEASURED_PEAKS.json), else the earlier measurement on this machine."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def kernel_source_tag():
    """Hash of the CUDA sources' code (comments and blank lines left out), so a
    committed traffic figure stays attached to the kernels it was taken on."""
    import hashlib
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "mxfp4_moe_block_b200", "csrc")
    for f in sorted(os.listdir(d)):
        text = open(os.path.join(d, f), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        lines = [ln.split("//", 1)[0].rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def _profile_value(fname, key):
    """A `key: value` line of a committed ncu summary in profiles/, if the
    summary was taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", fname)
    try:
        kv = {}
        for line in open(p):
            if ":" in line and not line.startswith(("#", "|", " ")):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("source_tag") != kernel_source_tag():
            return None
        return float(kv[key])
    except Exception:
        return None


VARIANT_NAMES = {0: "auto", 1: "fma", 2: "tensor", 3: "mxf8f6f4", 4: "mxf4", 5: "fused", 6: "pair"}


def load_traffic(workload, variant_name):
    """DRAM bytes per FFN call from the committed ncu summary (None if it was
    taken on other kernel sources)."""
    return _profile_value(f"ffn_{variant_name}_{workload}_traffic.txt", "dram_bytes_per_ffn_call")


def workload_config(sh, world):
    """The `config` object of the JSON line (identical for both arms)."""
    acc = " + ".join(sh.accept)
    layers = (f"{sh.layers} stacked MoE layers (RMSNorm, residual)" if sh.layers > 1
              else "one MoE layer")
    return {
        "workload": f"{sh.name}: {layers} H={sh.H} I={sh.I} E={sh.E} top-{sh.k} SwiGLU, "
                    f"S={sh.S} x K={sh.K} block, {acc} acceptance over V={sh.V}",
        "global_batch_tokens": sh.T * world,
        "parallelism": f"replicas x{world} (independent batches, no collective)",
        "l2": l2_statement(sh),
    }


L2_BYTES = 126 * 2**20


def l2_statement(sh):
    """Whether a step's expert weights alone exceed the 126 MB L2 (the bench
    does not flush L2 between steps; it relies on that)."""
    # expected distinct experts when P pairs pick among E uniformly
    experts = sh.E * (1.0 - (1.0 - 1.0 / sh.E) ** sh.P)
    gb = experts * sh.expert_bytes() * sh.layers / 1e9
    if experts * sh.expert_bytes() > L2_BYTES:
        return f"inputs larger than L2: ~{gb:.2f} GB of MXFP4 expert weights read per step"
    return (f"inputs smaller than L2 (~{gb * 1e3:.1f} MB of expert weights, no flush): "
            "L2-warm timing, not a bench number")


def rank_shape(sh, rank):
    """Each rank verifies its own batch: same weights, different activations,
    router logits and drafts."""
    return synth.Shape(**{**sh.__dict__, "seed": sh.seed + 7919 * rank})


def sum_over_ranks(value, world, device):
    """All ranks' total (all-reduce SUM); identity on one rank."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(value, world, device):
    """Slowest rank's value (all-reduce MAX); identity on one rank."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clock samples, taken only while a timed region runs
    (start/stop may be called several times; the samples accumulate)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.sm, self.mx, self.reasons = [], 0.0, set()

    def start(self):
        if shutil.which("nvidia-smi") is None:
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.f = open(self.path, "w")
        self.proc = subprocess.Popen(
            ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
             "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
            stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.proc = None
        self.f.close()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                self.sm.append(float(parts[1]))
                self.mx = max(self.mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(self.NAMES, parts[5:9]):
                if v.lower().startswith("active"):
                    self.reasons.add(n)
        os.unlink(self.path)

    def summary(self):
        if not self.sm:
            return None
        return {"sm_mhz": statistics.median(self.sm), "sm_max_mhz": self.mx,
                "reasons": sorted(self.reasons), "samples": len(self.sm)}


# ------------------------------------------------------------------ workload --

def _i32(n, device):
    return torch.empty(n, dtype=torch.int32, device=device)


class Workload:
    """Seeded inputs and buffers of one verify step, resident in HBM.

    Layer l of a stack: xn = rms_norm(residual) (layer 0 reads x), route and
    permute its router logits, the expert FFN, and a combine that adds the
    residual; a single layer combines without residual.  Then the block
    acceptance the workload names."""

    def __init__(self, sh, device, rank):
        import mxfp4_moe_block_b200 as mm
        self.mm = mm
        self.sh = sh
        self.dev = device
        s = self.sh_r = rank_shape(sh, rank)
        T, k, E, H, I, L = s.T, s.k, s.E, s.H, s.I, s.layers
        self.x_bits = synth.x_bf16_bits(s)
        self.x = torch.from_numpy(self.x_bits.view(np.int16)).to(device).view(torch.bfloat16)
        self.logits_np = [synth.router_logits(s, l) for l in range(L)]
        self.logits = [torch.from_numpy(a).to(device) for a in self.logits_np]
        self.w = [synth.weights_torch(sh, l, device) for l in range(L)]   # same on every rank
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.tw = torch.empty((T, k), dtype=torch.float32, device=device)
        self.off = [_i32(E + 1, device) for _ in range(L)]
        self.sp = _i32(T * k, device)
        self.pr = _i32(T * k, device)
        self.y = torch.empty((T * k, H), dtype=torch.float32, device=device)
        self.ws = mm.alloc_workspace(T, k, H, I, device)
        self.xn = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        # outputs the caller reads back, packed in one buffer: the combined
        # hidden states, then accept lengths and next tokens per acceptance
        self.greedy = "greedy" in s.accept
        self.rejection = "rejection" in s.accept
        nacc = int(self.greedy) + int(self.rejection)
        out_bytes = T * H * 2
        self.result = torch.empty(out_bytes + nacc * 2 * s.S * 4, dtype=torch.uint8, device=device)
        self.out = self.result[:out_bytes].view(torch.bfloat16).view(T, H)
        acc_views = self.result[out_bytes:].view(torch.int32).view(nacc, 2, s.S)
        j = 0
        if self.greedy:
            self.block_np = synth.block_logits(s)
            self.draft_np = synth.greedy_drafts(s, self.block_np)
            self.block = torch.from_numpy(self.block_np).to(device)
            self.draft = torch.from_numpy(self.draft_np).to(device)
            self.acc_g, self.nxt_g = acc_views[j, 0], acc_views[j, 1]
            j += 1
        if self.rejection:
            ri = synth.rejection_inputs(s)
            self.rej = [torch.from_numpy(np.ascontiguousarray(a)).to(device)
                        for a in (ri.p, ri.q, ri.draft, ri.u_accept, ri.u_resample)]
            self.acc_r, self.nxt_r = acc_views[j, 0], acc_views[j, 1]

    def step(self, variant, ev=None):
        """One verify step; `ev` (optional) = CUDA events: ev['ffn'][l] a
        (start, end) pair around layer l's FFN, ev['start'] / ev['end']."""
        mm, s = self.mm, self.sh_r
        L = s.layers
        if ev is not None:
            ev["start"].record()
        for l in range(L):
            if L > 1:
                mm.moe_rms_norm(self.x if l == 0 else self.out, out=self.xn)
                xin = self.xn
            else:
                xin = self.x
            mm.moe_route_permute(self.logits[l], s.k, s.E, self.idx, self.tw, self.off[l],
                                 self.sp, self.pr)
            if ev is not None:
                ev["ffn"][l][0].record()
            mm.mxfp4_moe_ffn(xin, s.k, *self.w[l], self.off[l], self.sp, y=self.y,
                             workspace=self.ws, variant=variant)
            if ev is not None:
                ev["ffn"][l][1].record()
            if L > 1:
                mm.moe_combine(self.y, self.pr, self.tw, residual=self.x if l == 0 else self.out,
                               out=self.out)
            else:
                mm.moe_combine(self.y, self.pr, self.tw, out=self.out)
        if self.greedy:
            mm.block_accept_greedy(self.block, self.draft, self.acc_g, self.nxt_g)
        if self.rejection:
            mm.block_accept_rejection(*self.rej, self.acc_r, self.nxt_r)
        if ev is not None:
            ev["end"].record()

    def active_experts(self):
        return [int((np.diff(o.cpu().numpy()) > 0).sum()) for o in self.off]

    def accepted(self):
        """Draft tokens accepted in the last step, per acceptance kind."""
        out = {}
        if self.greedy:
            out["greedy"] = int(self.acc_g.sum().item())
        if self.rejection:
            out["rejection"] = int(self.acc_r.sum().item())
        return out

    def ffn_flops(self):
        return 2.0 * self.sh_r.P * 3 * self.sh.H * self.sh.I


def count_launches(wl, variant):
    """Kernels one eager step launches, counted by the CUDA profiler (CUPTI)."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        wl.step(variant)
        torch.cuda.synchronize()
    names = [ev.name for ev in prof.events()
             if ev.device_type == torch.autograd.DeviceType.CUDA
             and not ev.name.lower().startswith(("memcpy", "memset"))]
    return len(names), sorted(set(names))


def capture_graph(wl, variant):
    """One step captured as a CUDA graph (launch gaps removed)."""
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        wl.step(variant)
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        wl.step(variant)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    return graph


def time_steps(wl, variant, steps, warmup, use_graph, clocks=None, barrier=lambda: None):
    """Device time of `steps` steps (CUDA events on the launching stream,
    synchronised on both sides), then an eager pass with events around each
    FFN call for the per-call breakdown."""
    for _ in range(max(3, warmup)):
        wl.step(variant)
    torch.cuda.synchronize()
    graph = capture_graph(wl, variant) if use_graph else None
    if clocks:
        clocks.start()
    barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        if graph is not None:
            graph.replay()
        else:
            wl.step(variant)
    b.record()
    torch.cuda.synchronize()
    barrier()
    ms = a.elapsed_time(b) / steps
    L = wl.sh.layers
    evs = [{"start": torch.cuda.Event(enable_timing=True), "end": torch.cuda.Event(enable_timing=True),
            "ffn": [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(L)]} for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        wl.step(variant, evs[i])
    torch.cuda.synchronize()
    if clocks:
        clocks.stop()
    eager_ms = statistics.mean(e["start"].elapsed_time(e["end"]) for e in evs)
    ffn_ms = [statistics.mean(e["ffn"][l][0].elapsed_time(e["ffn"][l][1]) for e in evs)
              for l in range(L)]
    del graph
    return {"ms": ms, "eager_ms": eager_ms, "ffn_ms": ffn_ms,
            "timing": "CUDA graph replay" if use_graph else "eager"}


def roofline(wl, ffn_ms, peaks, variant_name):
    """The expert FFN against its two rooflines (per layer, averaged): the
    active experts' MXFP4 bytes over the measured copy bandwidth, and the
    FFN's FLOPs over the measured dense bf16 GEMM rate.  `bound` is the
    roofline with the longer time; frac = that time / the measured time."""
    sh = wl.sh
    act = wl.active_experts()
    bytes_l = [n * sh.expert_bytes() for n in act]
    flops = wl.ffn_flops()
    ms = statistics.mean(ffn_ms)
    byts = statistics.mean(bytes_l)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9) * 1e3
    t_tc = flops / (peaks["bf16_tflops"] * 1e12) * 1e3
    hbm = {"achieved_gbs": byts / (ms * 1e-3) / 1e9, "peak_gbs": peaks["hbm_gbs"],
           "frac": t_hbm / ms, "algorithmic_bytes": byts, "active_experts": act}
    tc = {"achieved_tflops": flops / (ms * 1e-3) / 1e12, "peak_tflops": peaks["bf16_tflops"],
          "frac": t_tc / ms, "flops": flops,
          "peak_note": "dense bf16 (activations are bf16; the MMAs run block-scaled "
                       "fp8/fp4 kinds on exact narrow terms of them)"}
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    traffic = load_traffic(sh.name, variant_name)
    return {"bound": bound,
            "achieved": hbm["achieved_gbs"] if bound == "hbm" else tc["achieved_tflops"],
            "peak": hbm["peak_gbs"] if bound == "hbm" else tc["peak_tflops"],
            "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": max(t_hbm, t_tc) / ms, "traffic": traffic,
            "kernel": "mxfp4_moe_ffn (every launch of one FFN call: activation encodes and the "
                      "expert GEMMs, fused or GEMM-1+SwiGLU then GEMM-2)",
            "ffn_ms": ms, "hbm": hbm, "tensor": tc,
            "peak_source": f"{peaks['source']} hbm_gbs / bf16_tflops"}


# --------------------------------------------------------------- CPU oracle --

class OracleSample:
    """The oracle on a bounded sample of one verify step: the first `n_tok`
    tokens of the batch through every layer -- their routing over all E
    experts, the permutation, the SwiGLU FFN of each of their (token, expert)
    pairs, the combine and, for stacked layers, the RMSNorm and residual --
    then the acceptance of the sequences those tokens belong to.  Tokens are
    independent inside an MoE layer (router logits are given), so this is
    exactly the step's work for those tokens.  Inputs, expert weights
    included, are drawn before timing.  `workers` > 1 runs the (token,
    expert) FFNs of a layer on a thread pool (numpy releases the GIL) with one
    BLAS thread each; 1 is the plain single-thread oracle."""

    def __init__(self, sh, n_tok, workers=1):
        from oracle import moe as omoe
        self.sh = sh
        self.n_tok = n_tok = max(1, min(n_tok, sh.T))
        self.workers = workers
        self.toks = np.arange(n_tok)
        self.seqs = (0, (n_tok - 1) // sh.K + 1)
        x = synth.bf16_bits_to_f32(synth.x_bf16_bits(sh)).astype(np.float64)
        self.x64 = x[self.toks]
        self.logits = [synth.router_logits(sh, l)[self.toks] for l in range(sh.layers)]
        self.W = []
        for l in range(sh.layers):
            idx, _, _ = omoe.route_topk(self.logits[l], sh.k)
            self.W.append({int(e): (synth.weight_codes_np(sh, "w13", int(e), l),
                                    synth.weight_scales_np(sh, "w13", int(e), l),
                                    synth.weight_codes_np(sh, "w2", int(e), l),
                                    synth.weight_scales_np(sh, "w2", int(e), l))
                           for e in np.unique(idx)})
        if "greedy" in sh.accept:
            self.block = synth.block_logits(sh, seqs=self.seqs)
            self.draft = synth.greedy_drafts(sh, self.block, seqs=self.seqs)
        if "rejection" in sh.accept:
            self.ri = synth.rejection_inputs(sh, seqs=self.seqs)

    def run(self):
        from threadpoolctl import threadpool_limits

        from oracle import accept as oacc
        from oracle import moe as omoe
        sh = self.sh
        pool = (concurrent.futures.ThreadPoolExecutor(max_workers=self.workers)
                if self.workers > 1 else None)
        try:
            with threadpool_limits(limits=1):
                t0 = time.perf_counter()
                r = self.x64
                for l in range(sh.layers):
                    xn = omoe.rms_norm(r) if sh.layers > 1 else r
                    idx, w, _ = omoe.route_topk(self.logits[l], sh.k)
                    off, sp, pr = omoe.permute(idx, sh.E)
                    y = np.zeros((len(sp), sh.H))
                    jobs = [(e, int(off[e]), int(off[e + 1])) for e in range(sh.E)
                            if off[e + 1] > off[e]]

                    def one(job, xn=xn, sp=sp, l=l):
                        e, r0, r1 = job
                        _, ye = omoe.expert_ffn(xn[sp[r0:r1] // sh.k], *self.W[l][e], sh.I)
                        return r0, r1, ye
                    for r0, r1, ye in (pool.map(one, jobs) if pool else map(one, jobs)):
                        y[r0:r1] = ye
                    r, _ = omoe.combine(y, pr, w, r if sh.layers > 1 else None)
                if "greedy" in sh.accept:
                    oacc.greedy(self.block, self.draft)
                if "rejection" in sh.accept:
                    ri = self.ri
                    oacc.rejection(ri.p, ri.q, ri.draft, ri.u_accept, ri.u_resample)
                return time.perf_counter() - t0
        finally:
            if pool:
                pool.shutdown()

    def text(self):
        seq = self.seqs[1] - self.seqs[0]
        return (f"{self.n_tok} of the step's {self.sh.T} tokens through all {self.sh.layers} "
                f"layer(s) (routing, permutation, every expert FFN of those tokens, combine) "
                f"and the acceptance of their {seq} sequence(s); inputs drawn before timing")


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def sample_tokens(sh, cores):
    """Tokens in an oracle sample: the whole batch where its experts are small
    (the tiny shape), else as many tokens as give every core one (token,
    expert) FFN -- at least one."""
    if sh.H * sh.I <= 1 << 20:
        return sh.T
    return max(1, min(sh.T, cores // sh.k))


def cpu_baseline(sh):
    """Oracle tokens/s on the host: single thread, and all cores."""
    cores = host_cores()
    one = OracleSample(sh, sample_tokens(sh, 1), workers=1)
    t1 = one.run()
    many = OracleSample(sh, sample_tokens(sh, cores), workers=cores)
    tn = many.run()
    return {"value": many.n_tok / tn, "unit": UNIT, "cores": min(cores, many.n_tok * sh.k),
            "kind": "oracle", "sample": many.text(), "seconds": tn,
            "single_core": {"value": one.n_tok / t1, "unit": UNIT, "cores": 1, "kind": "oracle",
                            "sample": one.text(), "seconds": t1},
            "host_cores": cores}


# ---------------------------------------------------------------------- e2e --

def parse_cpulist(text):
    """CPU numbers of a Linux cpulist string ("0-3,8,10-11")."""
    cpus = set()
    for part in text.strip().split(","):
        if part:
            a, _, b = part.partition("-")
            cpus.update(range(int(a), int(b or a) + 1))
    return cpus


def gpu_local_cpus(dev):
    """The CPUs of the GPU's own NUMA node (its PCI device's local_cpulist in
    sysfs) that this process may run on, or None where that is unknown."""
    try:
        p = torch.cuda.get_device_properties(dev)
        bdf = f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        with open(f"/sys/bus/pci/devices/{bdf}/local_cpulist") as f:
            cpus = parse_cpulist(f.read())
    except (AttributeError, OSError, ValueError):
        return None
    return (cpus & os.sched_getaffinity(0)) or None


def pinned_near_gpu(n, dev):
    """A pinned host buffer whose pages are placed on the GPU's NUMA node: the
    allocating thread runs on that node's CPUs while the pages are allocated
    and first written, then gets its former CPUs back (pages on a far node
    would make every copy cross the socket link)."""
    local, old = gpu_local_cpus(dev), os.sched_getaffinity(0)
    if local:
        os.sched_setaffinity(0, local)
    try:
        buf = torch.empty(n, dtype=torch.uint8).pin_memory()
        buf.zero_()
    finally:
        if local:
            os.sched_setaffinity(0, old)
    return buf, (len(local) if local else None)


def e2e_time(wl, variant, steps, warmup):
    """The same step through the public API with host buffers, as a serving
    loop runs it: every step's inputs (x, router logits, block logits, drafts;
    one pinned staging buffer) are copied in with one copy and its results
    (combined hidden states, accept lengths, next tokens; one packed buffer)
    copied out with one copy, inside the timed region.  Each step (its kernels
    and the copy out) is one CUDA graph; the copy in of step i+1 runs on a
    second stream into the other of two input buffer sets while step i
    computes.  Also measures the host-to-device copy rate alone."""
    arrays = [wl.x_bits.view(np.uint8), wl.logits_np[0].view(np.uint8),
              wl.block_np.view(np.uint8), wl.draft_np.view(np.uint8)]
    offs, o = [], 0
    for a in arrays:
        offs.append(o)
        o += (a.nbytes + 255) // 256 * 256
    host_in, node_cpus = pinned_near_gpu(o, wl.dev)
    for a, off in zip(arrays, offs):
        host_in[off:off + a.nbytes] = torch.from_numpy(np.ascontiguousarray(a).reshape(-1))
    h2d = sum(a.nbytes for a in arrays)
    host_out, _ = pinned_near_gpu(wl.result.numel(), wl.dev)
    d2h = wl.result.numel()
    s = wl.sh_r

    def views(buf):
        x = buf[offs[0]:offs[0] + arrays[0].nbytes].view(torch.bfloat16).view(s.T, s.H)
        lg = buf[offs[1]:offs[1] + arrays[1].nbytes].view(torch.float32).view(s.T, s.E)
        blk = buf[offs[2]:offs[2] + arrays[2].nbytes].view(torch.float32).view(s.S, s.K, s.V)
        dr = buf[offs[3]:offs[3] + arrays[3].nbytes].view(torch.int32).view(s.S, s.K)
        return x, lg, blk, dr
    bufs = [torch.empty(o, dtype=torch.uint8, device=wl.dev) for _ in range(2)]
    sets = [views(b) for b in bufs]
    saved = (wl.x, wl.logits[0], wl.block, wl.draft)

    def use(i):
        wl.x, wl.logits[0], wl.block, wl.draft = sets[i]

    def step_out(i):
        use(i)
        wl.step(variant)
        host_out.copy_(wl.result, non_blocking=True)

    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    for i in (0, 1):
        bufs[i].copy_(host_in, non_blocking=True)
        step_out(i)
    torch.cuda.synchronize()
    graphs = []
    for i in (0, 1):
        side = torch.cuda.Stream()
        side.wait_stream(compute)
        with torch.cuda.stream(side):
            step_out(i)
        compute.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step_out(i)
        graphs.append(g)
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_done = [torch.cuda.Event(), torch.cuda.Event()]

    def run(n):
        copy.wait_stream(compute)
        with torch.cuda.stream(copy):
            bufs[0].copy_(host_in, non_blocking=True)
            ev_in[0].record(copy)
        for i in range(n):
            cur, nxt = i % 2, 1 - i % 2
            if i + 1 < n:
                if i >= 1:
                    copy.wait_event(ev_done[nxt])     # step i-1 has read set nxt
                with torch.cuda.stream(copy):
                    bufs[nxt].copy_(host_in, non_blocking=True)
                    ev_in[nxt].record(copy)
            compute.wait_event(ev_in[cur])
            graphs[cur].replay()
            ev_done[cur].record(compute)

    run(warmup)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(compute)
    run(steps)
    b.record(compute)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # the host link alone: the step's input copy, and a large pinned copy
    link = {"host_buffers_on_gpu_node_cpus": node_cpus}
    for name, n in (("step_input", o), ("256MiB", 256 << 20)):
        hsrc = host_in if n == o else pinned_near_gpu(n, wl.dev)[0]
        dst = torch.empty(n, dtype=torch.uint8, device=wl.dev)
        with torch.cuda.stream(copy):
            for _ in range(3):
                dst.copy_(hsrc, non_blocking=True)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(copy)
            for _ in range(10):
                dst.copy_(hsrc, non_blocking=True)
            e1.record(copy)
        torch.cuda.synchronize()
        link[f"h2d_gbs_{name}"] = 10 * n / (e0.elapsed_time(e1) * 1e-3) / 1e9
    wl.x, wl.logits[0], wl.block, wl.draft = saved
    del graphs
    return ms, h2d, d2h, link


# ---------------------------------------------------------------- quantiser --

def measure_quantize(device, peaks, reps=10):
    """mxfp4_quantize on 16 experts' worth of W13 rows ([16*4096, 7168] bf16,
    0.94 GB, larger than L2) against the copy-bandwidth roofline."""
    import mxfp4_moe_block_b200 as mm
    R, K = 16 * 4096, 7168
    g = torch.Generator(device=device)
    g.manual_seed(1234)
    w = (torch.randn((R, K), generator=g, device=device, dtype=torch.float32) * 0.02).to(torch.bfloat16)
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((R, K // 32), dtype=torch.uint8, device=device)
    for _ in range(3):
        mm.mxfp4_quantize(w, codes, scales)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        mm.mxfp4_quantize(w, codes, scales)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    byts = R * K * (2 + 0.5 + 1 / 32)
    gbs = byts / (ms * 1e-3) / 1e9
    del w, codes, scales
    return {"kernel": "mxfp4_quantize_kernel", "shape": [R, K], "ms": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes": byts,
                         "traffic": _profile_value("mxfp4_quantize_traffic.md",
                                                   "dram_bytes_per_launch")}}


# --------------------------------------------------------------- per config --

def measure_config(name, variant, steps, warmup, device, peaks, clocks, with_cpu):
    sh = synth.SHAPES[name]
    wl = Workload(sh, device, 0)
    t = time_steps(wl, variant, steps, warmup, True, clocks)
    n_launch, _ = count_launches(wl, variant)
    acc = wl.accepted()
    vname = VARIANT_NAMES.get(variant, str(variant))
    entry = {
        "config": workload_config(sh, 1),
        "ms_per_step": t["ms"], "timing": t["timing"],
        "verified_tokens_per_s": sh.T / (t["ms"] * 1e-3),
        "accepted_tokens_per_s": {k: v / (t["ms"] * 1e-3) for k, v in acc.items()},
        "ffn_ms_per_layer": statistics.mean(t["ffn_ms"]),
        "eager_ms_per_step": t["eager_ms"],
        "roofline": roofline(wl, t["ffn_ms"], peaks, vname),
        "launches_per_step": n_launch,
    }
    del wl
    torch.cuda.empty_cache()
    if with_cpu:
        entry["cpu_baseline"] = cpu_baseline(sh)
    return entry


# ---------------------------------------------------------------- reference --

def reference_arm(args, sh):
    """The oracle as the reference arm, on the host cores: every step is a
    real, timed bounded sample of the workload (OracleSample with all cores)."""
    cores = host_cores()
    samp = OracleSample(sh, sample_tokens(sh, cores), workers=cores)
    times = []
    for i in range(args.warmup + args.steps):
        t = samp.run()
        if i >= args.warmup:
            times.append(t)
    ms = 1e3 * statistics.mean(times)
    value = samp.n_tok / (ms / 1e3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded counter-based generator)",
        "config": workload_config(sh, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(cores, samp.n_tok * sh.k),
                         "kind": "oracle", "sample": samp.text()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------- main --

def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    sh = synth.SHAPES[args.workload]
    if args.experts:
        sh = synth.Shape(**{**sh.__dict__, "E": args.experts, "name": f"{sh.name}-E{args.experts}"})

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args, sh)))
        return

    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import mxfp4_moe_block_b200 as mm
    mm.lib()
    peaks = load_peaks()
    variant = args.variant
    vname = VARIANT_NAMES.get(variant, str(variant))

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    clocks = ClockSampler(local)
    wl = Workload(sh, dev, rank)
    t = time_steps(wl, variant, args.steps, args.warmup, not args.no_graph, clocks, barrier)
    ms = max_over_ranks(t["ms"], world, dev)
    acc = wl.accepted()
    accepted = sum_over_ranks(sum(acc.values()), world, dev)

    # the host-buffer path is staged for the single-layer greedy workloads
    e2e_ok = wl.sh.layers == 1 and wl.greedy and not wl.rejection
    if args.no_e2e or not e2e_ok:
        e2e_ms, h2d, d2h, link = float("nan"), 0, 0, {}
    else:
        e2e_ms, h2d, d2h, link = e2e_time(wl, variant, args.steps, 3)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    tokens = sh.T * world
    launches_per_step, kernel_names = count_launches(wl, variant)
    line = {
        "metric": METRIC, "value": tokens / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "mxfp4 weights, bf16 activations, f32 accumulate",
        "data": "synthetic (seeded counter-based generator; random MXFP4 weights)",
        "config": workload_config(sh, world),
        "ffn_variant": vname, "timing": t["timing"],
        "roofline": roofline(wl, t["ffn_ms"], peaks, vname),
        "breakdown_ms": {"ffn": statistics.mean(t["ffn_ms"]) * sh.layers,
                         "rest": t["eager_ms"] - sum(t["ffn_ms"]),
                         "eager_step": t["eager_ms"], "graph_step": t["ms"]},
        "ffn_tflops": wl.ffn_flops() / (statistics.mean(t["ffn_ms"]) * 1e-3) / 1e12,
        "accepted_tokens_per_s": accepted / (ms * 1e-3),
        "e2e": {"value": tokens / (e2e_ms * 1e-3) if e2e_ms == e2e_ms else None,
                "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "timing": "CUDA graph per step, one copy in (overlapped with the previous step) "
                          "and one copy out per step", **link},
        "gpu_launches": launches_per_step * args.steps,
        "launches_per_step": launches_per_step,
        "kernels": [n.split("(")[0].split("<")[0].replace("void ", "") for n in kernel_names],
    }
    del wl
    torch.cuda.empty_cache()
    if world == 1:
        if not args.no_per_config:
            pc = {}
            for name in [n for n in args.per_config.split(",")
                         if n in synth.SHAPES and n != sh.name]:
                pc[name] = measure_config(name, variant, min(args.steps, 20), args.warmup, dev,
                                          peaks, clocks, not args.no_cpu_baseline)
            pc["quantize"] = measure_quantize(dev, peaks)
            line["per_config"] = pc
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(sh)
    line["clocks"] = clocks.summary()
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
