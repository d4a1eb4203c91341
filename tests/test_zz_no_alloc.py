"""mxfp4_moe_ffn_noalloc: the FFN for callers that may not allocate device
memory (plugins whose host engine owns all device memory, latency-critical
loops that cannot afford cudaMalloc/cudaFree).  It must give the results of
mxfp4_moe_ffn, call after call, from its built-in scratch array.

Collected last on purpose, so that a run stopping at the first failure has
run every other test before this one."""
import numpy as np
import pytest
import torch

import mxfp4_moe_block_b200 as mm
from mxfp4_moe_block_b200 import synth
from oracle import moe as omoe

from gpu_helpers import Layer, assert_ffn_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc(L, sh, off, sp):
    """One call through the C ABI; y starts as NaN so unwritten rows show."""
    y = torch.full((sh.P, sh.H), float("nan"), dtype=torch.float32, device=DEV)
    st = mm.lib().mxfp4_moe_ffn_noalloc(
        L.x.data_ptr(), sh.T, sh.H, sh.I, sh.E, sh.k,
        L.w[0].data_ptr(), L.w[1].data_ptr(), L.w[2].data_ptr(), L.w[3].data_ptr(),
        off.data_ptr(), sp.data_ptr(), y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, f"status {st}"
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _problem(sh):
    L = Layer(sh, 0, DEV)
    idx, w = mm.moe_route_topk(L.logits, sh.k)
    off, sp, pr = mm.moe_permute(idx, sh.E)
    y_ref, _ = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp)
    return L, off, sp, y_ref.cpu().numpy()


def _oracle_rows(L, sh, off, sp, y, n_experts=2):
    """Every row of a few active experts against the oracle."""
    offn, spn = off.cpu().numpy(), sp.cpu().numpy()
    act = np.nonzero(np.diff(offn))[0]
    for e in act[:: max(1, len(act) // n_experts)][:n_experts]:
        r0, r1 = int(offn[e]), int(offn[e + 1])
        _, ye = omoe.expert_ffn(L.x_f64()[spn[r0:r1] // sh.k], *L.oracle_weights(int(e)), sh.I)
        assert_ffn_close(y[r0:r1], ye, f"no-alloc expert {e} vs oracle")


def test_noalloc_matches_ffn_on_two_calls_in_a_row():
    """Two calls on the batch-1 problem with a call on a different problem
    between them: each result equals mxfp4_moe_ffn's on the same inputs (so
    nothing the previous call left in the shared scratch is read), and
    sampled experts match the oracle."""
    sh = synth.SHAPES["batch1"]          # 8-token block, top-8: fits the built-in scratch
    assert mm.mxfp4_moe_ffn_workspace_bytes(sh.T, sh.k, sh.H, sh.I) <= mm._lib.NOALLOC_SCRATCH_BYTES
    other = synth.Shape("noalloc-other", H=1024, I=512, E=16, k=4, S=2, K=8, V=64, seed=77)
    L, off, sp, y_ref = _problem(sh)
    L2, off2, sp2, y2_ref = _problem(other)
    y_first = _noalloc(L, sh, off, sp)
    assert_ffn_close(y_first, y_ref, "no-alloc call 1")
    y_other = _noalloc(L2, other, off2, sp2)
    assert_ffn_close(y_other, y2_ref, "no-alloc call on another problem")
    y_second = _noalloc(L, sh, off, sp)
    assert_ffn_close(y_second, y_ref, "no-alloc call 2")
    _oracle_rows(L, sh, off, sp, y_second)
    _oracle_rows(L2, other, off2, sp2, y_other)
    assert mm.moe_get_device_status() == (0, 0)


def test_noalloc_rejects_problems_beyond_its_scratch():
    sh = synth.SHAPES["serving"]         # 128 tokens x top-8: needs more than 8 MiB
    assert mm.mxfp4_moe_ffn_workspace_bytes(sh.T, sh.k, sh.H, sh.I) > mm._lib.NOALLOC_SCRATCH_BYTES
    st = mm.lib().mxfp4_moe_ffn_noalloc(None, sh.T, sh.H, sh.I, sh.E, sh.k, *([None] * 7),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 4
    # a bad argument is reported as such, whatever the problem's size
    st = mm.lib().mxfp4_moe_ffn_noalloc(None, sh.T, sh.H, sh.I, sh.E, 33, *([None] * 7),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 1
