"""Failure detection on the GPU, without a fault, and host-side robustness.

The tensor-core FFN bounds every wait it makes.  Here the limit is lowered
far below a kernel's run time (moe_set_wait_limit_ns), so a wait runs out:
the kernel must report MOE_DEV_TIMEOUT through the device status word, drain
the copies and MMAs it issued, free its tensor memory and return, leaving the
context usable -- the next call, at the normal limit, matches the oracle.  The
CTA-pair launch also tells the partner CTA, which holds operands and barriers
of the same MMAs, and the two leave together.

The library's per-device set-up (kernel attributes, the tensor-map encoder)
must also survive two host threads making their first calls at once.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import mxfp4_moe_block_b200 as mm
from mxfp4_moe_block_b200 import synth
from oracle import moe as omoe

from gpu_helpers import Layer, assert_ffn_close, bf16_to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _problem():
    sh = synth.Shape("waits", H=512, I=256, E=8, k=2, S=1, K=16, V=64, seed=41)
    L = Layer(sh, 0, DEV)
    idx, w = mm.moe_route_topk(L.logits, sh.k)
    off, sp, pr = mm.moe_permute(idx, sh.E)
    ridx, _, _ = omoe.route_topk(L.logits_np, sh.k)
    roff, rsp, _ = omoe.permute(ridx, sh.E)
    h_ref, y_ref = omoe.moe_ffn(L.x_f64(), sh.k, sh.I, L.oracle_weights, roff, rsp)
    return sh, L, off, sp, h_ref, y_ref


@pytest.mark.parametrize("variant", [mm.FFN_TENSOR_F8, mm.FFN_TENSOR_F4, mm.FFN_TENSOR_FUSED,
                                     mm.FFN_TENSOR_F8_PAIR],
                         ids=["mxf8f6f4", "mxf4", "fused", "pair"])
def test_wait_timeout_reports_and_context_recovers(variant):
    sh, L, off, sp, h_ref, y_ref = _problem()
    timed_out = False
    try:
        for _ in range(5):
            mm.moe_clear_device_status()
            mm.moe_set_wait_limit_ns(1)
            y, ws = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp, variant=variant)
            st = mm.moe_get_device_status()          # synchronises the stream
            mm.moe_set_wait_limit_ns(0)
            if st == (mm._lib.MOE_OK + 5, 4):        # MOE_ERR_DEVICE, MOE_DEV_TIMEOUT
                timed_out = True
                break
            # a call whose waits all finished in time is an ordinary call
            assert st == (0, 0), st
            assert_ffn_close(y.cpu().numpy(), y_ref, "call within the limit")
    finally:
        mm.moe_set_wait_limit_ns(0)
        mm.moe_clear_device_status()
    assert timed_out, "no wait ran out at a 1 ns limit"
    # the context is usable and the next call is correct
    y, ws = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp, variant=variant)
    assert_ffn_close(bf16_to_f64(mm.workspace_h(ws, sh.P, sh.I)), h_ref, "h after recovery")
    assert_ffn_close(y.cpu().numpy(), y_ref, "y after recovery")
    assert mm.moe_get_device_status() == (0, 0)


def test_first_calls_from_two_host_threads():
    """A fresh process whose first FFN calls come from two host threads at
    once (each with its own stream and workspace): both succeed and agree."""
    script = textwrap.dedent(f"""
        import sys, threading
        sys.path.insert(0, {ROOT!r})
        sys.path.insert(0, {os.path.join(ROOT, 'tests')!r})
        import numpy as np, torch
        import mxfp4_moe_block_b200 as mm
        from mxfp4_moe_block_b200 import synth
        from gpu_helpers import Layer
        torch.cuda.set_device(0)
        sh = synth.Shape("threads", H=512, I=256, E=8, k=2, S=1, K=16, V=64, seed=43)
        L = Layer(sh, 0, "cuda")
        idx, w = mm.moe_route_topk(L.logits, sh.k)
        off, sp, pr = mm.moe_permute(idx, sh.E)
        torch.cuda.synchronize()
        out, errs = {{}}, []
        go = threading.Barrier(2)
        def run(i):
            try:
                torch.cuda.set_device(0)
                s = torch.cuda.Stream()
                go.wait()
                with torch.cuda.stream(s):
                    y, _ = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp, variant=2 + i % 2 * 2)
                s.synchronize()
                out[i] = y.cpu().numpy()
            except Exception as e:
                errs.append(repr(e))
        th = [threading.Thread(target=run, args=(i,)) for i in range(2)]
        [t.start() for t in th]
        [t.join() for t in th]
        assert not errs, errs
        r = np.linalg.norm(out[0] - out[1]) / np.linalg.norm(out[0])
        assert r < 2e-3, r
        assert mm.moe_get_device_status() == (0, 0)
        print("ok", r)
    """)
    res = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-2000:]
    assert res.stdout.strip().startswith("ok")
