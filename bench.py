"""Benchmark of the MXFP4 MoE block-verify step on B200.

One step = the whole hot path over one drafted batch: moe_route_topk ->
moe_permute -> mxfp4_moe_ffn -> moe_combine -> block_accept_greedy (the
batch-1 verify workload: 1 sequence x 8-token block, one MoE layer of
hidden 7168, expert intermediate 2048, 256 experts, top-8; greedy acceptance
over a 152064-token vocabulary).  Metric: verified tokens/s (= S*K / step
time), with the HBM roofline of the expert FFN beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload batch1|serving|tiny]

Multi-GPU: every rank verifies its own independent batch (the path has no
exchange step); value = all ranks' tokens / the slowest rank's time.
--impl reference times the CPU oracle (the reference arm of this repository)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    # the step times one MoE layer with greedy acceptance: the configurations
    # of that form; the others (rejection acceptance, stacked layers) are
    # parity-test cases
    ap.add_argument("--workload", default="batch1",
                    choices=[n for n, s in synth.SHAPES.items()
                             if s.layers == 1 and s.accept == ("greedy",)])
    ap.add_argument("--variant", type=int, default=0, help="FFN kernel: 0 auto, 1 FMA, 2 tensor")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches only")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the expert count (smaller cases for profiler captures)")
    return ap.parse_args()


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


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


def load_traffic(workload, variant_name):
    """DRAM bytes per FFN call from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", f"ffn_{variant_name}_{workload}_traffic.txt")
    try:
        kv = {}
        for line in open(p):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("source_tag") != kernel_source_tag():
            return None
        return float(kv["dram_bytes_per_ffn_call"])
    except Exception:
        return None


def workload_config(sh, world):
    """The `config` object of the JSON line (identical for both arms)."""
    acc = " + ".join(sh.accept)
    layers = f"{sh.layers} stacked MoE layers" if sh.layers > 1 else "one MoE layer"
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
    gb = experts * sh.expert_bytes() / 1e9
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
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

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
            return None
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ workload --

class Workload:
    """Seeded inputs of one verify step, resident in HBM."""

    def __init__(self, sh, device, rank):
        import mxfp4_moe_block_b200 as mm
        self.mm = mm
        self.sh = sh
        self.dev = device
        self.sh_r = rank_shape(sh, rank)
        s = self.sh_r
        self.x_bits = synth.x_bf16_bits(s)
        self.logits_np = synth.router_logits(s)
        self.block_np = synth.block_logits(s)
        self.draft_np = synth.greedy_drafts(s, self.block_np)
        self.x = torch.from_numpy(self.x_bits.view(np.int16)).to(device).view(torch.bfloat16)
        self.logits = torch.from_numpy(self.logits_np).to(device)
        self.block = torch.from_numpy(self.block_np).to(device)
        self.draft = torch.from_numpy(self.draft_np).to(device)
        self.w = synth.weights_torch(sh, 0, device)      # model weights: same on every rank
        T, k, E, H, I = s.T, s.k, s.E, s.H, s.I
        i32 = dict(dtype=torch.int32, device=device)
        self.idx = torch.empty((T, k), **i32)
        self.tw = torch.empty((T, k), dtype=torch.float32, device=device)
        self.off = torch.empty(E + 1, **i32)
        self.sp = torch.empty(T * k, **i32)
        self.pr = torch.empty(T * k, **i32)
        self.y = torch.empty((T * k, H), dtype=torch.float32, device=device)
        self.ws = mm.alloc_workspace(T, k, H, I, device)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        self.acc = torch.empty(s.S, **i32)
        self.nxt = torch.empty(s.S, **i32)

    def step(self, variant, ev=None):
        mm, s = self.mm, self.sh_r
        if ev is not None:
            ev[0].record()
        mm.moe_route_permute(self.logits, s.k, s.E, self.idx, self.tw, self.off, self.sp, self.pr)
        if ev is not None:
            ev[1].record()
        mm.mxfp4_moe_ffn(self.x, s.k, *self.w, self.off, self.sp, y=self.y, workspace=self.ws,
                         variant=variant)
        if ev is not None:
            ev[2].record()
        mm.moe_combine(self.y, self.pr, self.tw, out=self.out)
        mm.block_accept_greedy(self.block, self.draft, self.acc, self.nxt)
        if ev is not None:
            ev[3].record()

    def activated_bytes(self):
        off = self.off.cpu().numpy()
        n_act = int((np.diff(off) > 0).sum())
        return n_act * self.sh.expert_bytes(), n_act

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


def e2e_time(wl, variant, steps, warmup):
    """The same step through the public API with host buffers, as a serving
    loop runs it: every step's inputs are copied in from pinned host memory
    and its results (combined hidden states, accept lengths, next tokens)
    copied out, inside the timed region.  Each step (its kernels and the
    copies out) is one CUDA graph; the copy in of step i+1 runs on a second
    stream into the other of two input buffer sets while step i computes."""
    hx = torch.from_numpy(wl.x_bits.view(np.int16)).pin_memory()
    hl = torch.from_numpy(wl.logits_np).pin_memory()
    hb = torch.from_numpy(wl.block_np).pin_memory()
    hd = torch.from_numpy(wl.draft_np).pin_memory()
    ho = torch.empty(wl.out.shape, dtype=torch.bfloat16).pin_memory()
    ha = torch.empty(wl.acc.shape, dtype=torch.int32).pin_memory()
    hn = torch.empty(wl.nxt.shape, dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hx, hl, hb, hd))
    d2h = sum(t.numel() * t.element_size() for t in (ho, ha, hn))
    # two input sets on the device: set 0 is the workload's own tensors
    sets = [(wl.x, wl.logits, wl.block, wl.draft),
            (torch.empty_like(wl.x), torch.empty_like(wl.logits), torch.empty_like(wl.block),
             torch.empty_like(wl.draft))]

    def copy_in(i):
        x, lg, blk, dr = sets[i]
        x.view(torch.int16).copy_(hx, non_blocking=True)
        lg.copy_(hl, non_blocking=True)
        blk.copy_(hb, non_blocking=True)
        dr.copy_(hd, non_blocking=True)

    def step_out(i):
        wl.x, wl.logits, wl.block, wl.draft = sets[i]
        wl.step(variant)
        ho.copy_(wl.out, non_blocking=True)
        ha.copy_(wl.acc, non_blocking=True)
        hn.copy_(wl.nxt, non_blocking=True)

    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream()
    for i in (0, 1):
        copy_in(i)
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
    wl.x, wl.logits, wl.block, wl.draft = sets[0]
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_done = [torch.cuda.Event(), torch.cuda.Event()]

    def run(n):
        copy.wait_stream(compute)
        with torch.cuda.stream(copy):
            copy_in(0)
            ev_in[0].record(copy)
        for i in range(n):
            cur, nxt = i % 2, 1 - i % 2
            if i + 1 < n:
                if i >= 1:
                    copy.wait_event(ev_done[nxt])     # step i-1 has read set nxt
                with torch.cuda.stream(copy):
                    copy_in(nxt)
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
    return a.elapsed_time(b) / steps, h2d, d2h, "CUDA graph per step, copy-in of the next step overlapped"


# --------------------------------------------------------------- CPU oracle --

def oracle_step_seconds(sh, n_expert_sample=4, seed_shift=0):
    """Time the CPU oracle on one step of the workload, with the expert FFN
    on a sample of the active experts, scaled to all of them."""
    from threadpoolctl import threadpool_limits

    from oracle import accept as oacc
    from oracle import moe as omoe
    s = synth.Shape(**{**sh.__dict__, "seed": sh.seed + seed_shift})
    x64 = synth.bf16_bits_to_f32(synth.x_bf16_bits(s)).astype(np.float64)
    logits = synth.router_logits(s)
    block = synth.block_logits(s)
    draft = synth.greedy_drafts(s, block)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        idx, w, _ = omoe.route_topk(logits, s.k)
        off, sp, pr = omoe.permute(idx, s.E)
        t_route = time.perf_counter() - t0
        act = [e for e in range(s.E) if off[e + 1] > off[e]]
        sample = act[:: max(1, len(act) // n_expert_sample)][:n_expert_sample]
        y = np.zeros((s.P, s.H))
        t_ffn = 0.0
        for e in sample:
            r0, r1 = off[e], off[e + 1]
            wts = (synth.weight_codes_np(s, "w13", e), synth.weight_scales_np(s, "w13", e),
                   synth.weight_codes_np(s, "w2", e), synth.weight_scales_np(s, "w2", e))
            t0 = time.perf_counter()            # weights are inputs: drawn before timing
            _, y[r0:r1] = omoe.expert_ffn(x64[sp[r0:r1] // s.k], *wts, s.I)
            t_ffn += time.perf_counter() - t0
        t_ffn *= len(act) / len(sample)
        t0 = time.perf_counter()
        omoe.combine(y, pr, w)
        oacc.greedy(block, draft)
        t_rest = time.perf_counter() - t0
    total = t_route + t_ffn + t_rest
    return total, {"experts_active": len(act), "experts_sampled": len(sample)}


class OracleStep:
    """The reference arm's step: the oracle (one thread) on the step's inputs,
    drawn once.  Routing, permutation, combine and greedy acceptance run in
    full; the expert FFN runs for one active expert on the first `i_s` of
    its I intermediate units (the SwiGLU of an I-slice is the same oracle
    code on fewer gate/up/down rows), and its time is scaled by
    (active experts) x I / i_s.  `i_s` is chosen so that the whole run of
    steps fits the time budget."""

    def __init__(self, sh):
        from oracle import moe as omoe
        self.sh = sh
        self.x64 = synth.bf16_bits_to_f32(synth.x_bf16_bits(sh)).astype(np.float64)
        self.logits = synth.router_logits(sh)
        self.block = synth.block_logits(sh)
        self.draft = synth.greedy_drafts(sh, self.block)
        idx, _, _ = omoe.route_topk(self.logits, sh.k)
        off, _, _ = omoe.permute(idx, sh.E)
        self.active = [e for e in range(sh.E) if off[e + 1] > off[e]]
        e = self.active[len(self.active) // 2]
        self.expert = e
        self.w13c = synth.weight_codes_np(sh, "w13", e)
        self.w13s = synth.weight_scales_np(sh, "w13", e)
        self.w2c = synth.weight_codes_np(sh, "w2", e)
        self.w2s = synth.weight_scales_np(sh, "w2", e)
        self.i_s = sh.I

    def _slice(self, i_s):
        I = self.sh.I
        rows = np.r_[0:i_s, I:I + i_s]
        return (self.w13c[rows], self.w13s[rows], self.w2c[:, :i_s // 2],
                self.w2s[:, :i_s // 32])

    def run(self):
        from threadpoolctl import threadpool_limits

        from oracle import accept as oacc
        from oracle import moe as omoe
        sh, i_s = self.sh, self.i_s
        wts = self._slice(i_s)
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            idx, w, _ = omoe.route_topk(self.logits, sh.k)
            off, sp, pr = omoe.permute(idx, sh.E)
            t_route = time.perf_counter() - t0
            e = self.expert
            r0, r1 = off[e], off[e + 1]
            y = np.zeros((sh.P, sh.H))
            t0 = time.perf_counter()
            _, y[r0:r1] = omoe.expert_ffn(self.x64[sp[r0:r1] // sh.k], *wts, i_s)
            t_ffn = (time.perf_counter() - t0) * len(self.active) * sh.I / i_s
            t0 = time.perf_counter()
            omoe.combine(y, pr, w)
            oacc.greedy(self.block, self.draft)
            t_rest = time.perf_counter() - t0
        return t_route + t_ffn + t_rest

    def fit(self, steps, budget_s):
        """Shrink the I-slice until steps x (one step's wall time) fits."""
        while True:
            t0 = time.perf_counter()
            self.run()
            wall = time.perf_counter() - t0
            if wall * steps <= budget_s or self.i_s <= 64:
                return
            self.i_s = max(64, (int(self.i_s * budget_s / (wall * steps)) // 32) * 32)

    def sample_text(self):
        return (f"route+permute+combine+greedy in full; expert FFN on 1 of "
                f"{len(self.active)} active experts and {self.i_s} of its {self.sh.I} "
                f"intermediate units, time scaled to all")


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
        if rank != 0:
            return
        ostep = OracleStep(sh)
        ostep.fit(args.warmup + args.steps, budget_s=150.0)   # the whole run: a few minutes
        times = []
        for i in range(args.warmup + args.steps):
            t = ostep.run()
            if i >= args.warmup:
                times.append(t)
        ms = 1e3 * statistics.mean(times)
        value = sh.T / (ms / 1e3)
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded counter-based generator)",
            "config": workload_config(sh, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": ostep.sample_text()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return

    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import mxfp4_moe_block_b200 as mm
    mm.lib()
    wl = Workload(sh, dev, rank)
    variant = args.variant

    for _ in range(max(3, args.warmup)):
        wl.step(variant)
    torch.cuda.synchronize()
    act_bytes, n_act = wl.activated_bytes()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # CUDA graph of one step (launch gaps removed); eager launches otherwise
    graph = None
    if not args.no_graph:
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

    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            wl.step(variant)
    t_end.record()
    torch.cuda.synchronize()
    barrier()
    ms = t_start.elapsed_time(t_end) / args.steps
    # per-call breakdown on eager launches, events on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        wl.step(variant, evs[i])
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    eager_ms = e0.elapsed_time(e1) / args.steps
    ffn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    route_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    tail_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    ms = max_over_ranks(ms, world, dev)
    # draft tokens the step accepted (sum of accept_len over the sequences)
    accepted = sum_over_ranks(int(wl.acc.sum().item()), world, dev)

    if args.no_e2e:
        e2e_ms, h2d, d2h, e2e_mode = float("nan"), 0, 0, None
    else:
        e2e_ms, h2d, d2h, e2e_mode = e2e_time(wl, variant, args.steps, 3)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    peak, peak_kind = load_peaks()
    achieved = act_bytes / (ffn_ms * 1e-3) / 1e9
    vname = {0: "auto", 1: "fma", 2: "tensor"}[variant]
    traffic = load_traffic(sh.name, vname)
    tokens = sh.T * world
    launches_per_step, kernel_names = count_launches(wl, variant)
    line = {
        "metric": METRIC, "value": tokens / (ms * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "mxfp4 weights, bf16 activations, f32 accumulate",
        "data": "synthetic (seeded counter-based generator; random MXFP4 weights)",
        "config": workload_config(sh, world),
        "ffn_variant": vname, "timing": "CUDA graph replay" if graph is not None else "eager",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "mxfp4_moe_ffn (GEMM-1+SwiGLU and GEMM-2 launches)",
                     "algorithmic_bytes": act_bytes, "active_experts": n_act,
                     "peak_source": f"{peak_kind} hbm_gbs"},
        "breakdown_ms": {"route+permute": route_ms, "ffn": ffn_ms, "combine+greedy": tail_ms,
                         "eager_step": eager_ms, "graph_step": ms if graph is not None else None},
        "ffn_tflops": wl.ffn_flops() / (ffn_ms * 1e-3) / 1e12,
        "accepted_tokens_per_s": accepted / (ms * 1e-3),
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "timing": e2e_mode},
        "gpu_launches": launches_per_step * args.steps,
        "launches_per_step": launches_per_step,
        "kernels": [n.split("(")[0].split("<")[0].replace("void ", "") for n in kernel_names],
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t, info = oracle_step_seconds(sh)
        line["cpu_baseline"] = {
            "value": sh.T / t, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"one step; expert FFN on {info['experts_sampled']} of "
                      f"{info['experts_active']} active experts, time scaled to all"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
