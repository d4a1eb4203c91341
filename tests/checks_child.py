"""Run by tests/test_gpu_checks.py in a child process with MXFP4_MOE_CHECKS=1,
so that the package loads the checked build (libmxfp4_moe_checks.so).

1. On good inputs the checked build agrees with the oracle (FFN through the
   FMA path, both tensor-core kinds and the CTA-pair launch; combine).
2. A pair id past the end of sorted_pair's range, expert offsets that go
   down, and a pair_row entry past the end each set MOE_DEV_BAD_INDEX; the
   checked kernels never address memory with them.
3. After the status is cleared the next call is green again.
Prints "checks ok" last.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import mxfp4_moe_block_b200 as mm  # noqa: E402
from mxfp4_moe_block_b200 import _lib, synth  # noqa: E402
from oracle import moe as omoe  # noqa: E402

from gpu_helpers import Layer, assert_ffn_close  # noqa: E402

assert _lib.LIB_PATH.endswith("libmxfp4_moe_checks.so"), _lib.LIB_PATH
DEV = torch.device("cuda", 0)
BAD = (_lib.MOE_OK + 5, _lib.DEV_BAD_INDEX)          # MOE_ERR_DEVICE, MOE_DEV_BAD_INDEX

sh = synth.Shape("checked", H=1024, I=512, E=8, k=2, S=2, K=8, V=64, seed=2301)
L = Layer(sh, 0, DEV)
mm.moe_clear_device_status()
idx, tw = mm.moe_route_topk(L.logits, sh.k)
off, sp, pr = mm.moe_permute(idx, sh.E)
ridx, rw, _ = omoe.route_topk(L.logits_np, sh.k)
roff, rsp, rpr = omoe.permute(ridx, sh.E)
assert np.array_equal(off.cpu().numpy(), roff) and np.array_equal(sp.cpu().numpy(), rsp)
h_ref, y_ref = omoe.moe_ffn(L.x_f64(), sh.k, sh.I, L.oracle_weights, roff, rsp)

variants = (mm.FFN_FMA, mm.FFN_TENSOR_F8, mm.FFN_TENSOR_F4, mm.FFN_TENSOR_F8_PAIR)
for v in variants:
    y, ws = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp, variant=v)
    assert_ffn_close(y.cpu().numpy(), y_ref, f"checked build, variant {v}")
    assert mm.moe_get_device_status() == (0, 0), v
y, ws = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp, variant=mm.FFN_TENSOR_F8)
out = mm.moe_combine(y, pr, tw)
ref_out, _ = omoe.combine(y.cpu().numpy().astype(np.float64), pr.cpu().numpy(), tw.cpu().numpy())
assert_ffn_close(out.float().cpu().numpy(), ref_out, "checked build, combine")
assert mm.moe_get_device_status() == (0, 0)

# a pair id past the end: the activation gathers of every path
for v in variants:
    bad_sp = sp.clone()
    bad_sp[3] = sh.P + 7
    mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, bad_sp, variant=v)
    assert mm.moe_get_device_status() == BAD, v
    mm.moe_clear_device_status()

# expert offsets that go down: the GEMMs' tile tables and the FMA path
bad_off = off.clone()
o = off.cpu().numpy()
e = int(np.argmax(np.diff(o) > 0))                 # an expert with rows
bad_off[e + 1] = o[e] - 1
for v in variants:
    mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, bad_off, sp, variant=v)
    assert mm.moe_get_device_status() == BAD, v
    mm.moe_clear_device_status()
bad_off = off.clone()
bad_off[sh.E] = sh.P + 64                           # past the pairs
mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, bad_off, sp, variant=mm.FFN_TENSOR_F8)
assert mm.moe_get_device_status() == BAD
mm.moe_clear_device_status()

# a pair_row entry past the end: combine
bad_pr = pr.clone()
bad_pr[5] = sh.P + 3
mm.moe_combine(y, bad_pr, tw)
assert mm.moe_get_device_status() == BAD
mm.moe_clear_device_status()

# green again
y, ws = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp, variant=mm.FFN_TENSOR_F8)
assert_ffn_close(y.cpu().numpy(), y_ref, "checked build after the bad inputs")
assert mm.moe_get_device_status() == (0, 0)
print("checks ok")
