"""Time one expert-FFN call (mxfp4_moe_ffn) on a seeded workload.

    python -m mxfp4_moe_block_b200.time_ffn [--workload batch1] [--variant 0] [--calls 20]

Draws the workload's layer-0 inputs and weights on the device, routes and
permutes once, then times `--calls` back-to-back FFN calls between CUDA
events (the activated weights exceed L2 for every shape but tiny).  Prints
the mean time per call, the active experts' MXFP4 bytes and the bandwidth
they imply.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

import mxfp4_moe_block_b200 as mm
from mxfp4_moe_block_b200 import synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="batch1", choices=list(synth.SHAPES))
    ap.add_argument("--variant", type=int, default=mm.FFN_AUTO,
                    help="0 auto, 1 FMA, 2 tensor, 3 kind::mxf8f6f4, 4 kind::mxf4")
    ap.add_argument("--calls", type=int, default=20)
    args = ap.parse_args()
    sh = synth.SHAPES[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    x = torch.from_numpy(synth.x_bf16_bits(sh).view(np.int16)).to(dev).view(torch.bfloat16)
    logits = torch.from_numpy(synth.router_logits(sh)).to(dev)
    w = synth.weights_torch(sh, 0, dev)
    _, _, off, sp, _ = mm.moe_route_permute(logits, sh.k)
    y = torch.empty((sh.P, sh.H), dtype=torch.float32, device=dev)
    ws = mm.alloc_workspace(sh.T, sh.k, sh.H, sh.I, dev)
    for _ in range(3):
        mm.mxfp4_moe_ffn(x, sh.k, *w, off, sp, y=y, workspace=ws, variant=args.variant)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.calls):
        mm.mxfp4_moe_ffn(x, sh.k, *w, off, sp, y=y, workspace=ws, variant=args.variant)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.calls
    active = int((np.diff(off.cpu().numpy()) > 0).sum())
    gb = active * sh.expert_bytes() / 1e9
    st = mm.moe_get_device_status()
    print(f"{sh.name} variant {args.variant}: {ms * 1e3:.1f} us per call, {active} active experts, "
          f"{gb:.3f} GB -> {gb / ms * 1e3:.0f} GB/s, device status {st}")


if __name__ == "__main__":
    main()
