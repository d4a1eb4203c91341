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

from gpu_helpers import Layer, assert_ffn_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_noalloc_matches_ffn_on_two_calls_in_a_row():
    sh = synth.SHAPES["batch1"]          # 8-token block, top-8: fits the built-in scratch
    assert mm.mxfp4_moe_ffn_workspace_bytes(sh.T, sh.k, sh.H, sh.I) <= mm._lib.NOALLOC_SCRATCH_BYTES
    L = Layer(sh, 0, DEV)
    idx, w = mm.moe_route_topk(L.logits, sh.k)
    off, sp, pr = mm.moe_permute(idx, sh.E)
    y_ref, _ = mm.mxfp4_moe_ffn(L.x, sh.k, *L.w, off, sp)
    L2 = mm.lib()
    outs = []
    for call in range(2):
        y = torch.full((sh.P, sh.H), float("nan"), dtype=torch.float32, device=DEV)
        st = L2.mxfp4_moe_ffn_noalloc(
            L.x.data_ptr(), sh.T, sh.H, sh.I, sh.E, sh.k,
            L.w[0].data_ptr(), L.w[1].data_ptr(), L.w[2].data_ptr(), L.w[3].data_ptr(),
            off.data_ptr(), sp.data_ptr(), y.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        outs.append(y.cpu().numpy())
        assert_ffn_close(outs[-1], y_ref.cpu().numpy(), f"no-alloc call {call}")
    assert mm.moe_get_device_status() == (0, 0)


def test_noalloc_rejects_problems_beyond_its_scratch():
    sh = synth.SHAPES["serving"]         # 128 tokens x top-8: needs more than 8 MiB
    assert mm.mxfp4_moe_ffn_workspace_bytes(sh.T, sh.k, sh.H, sh.I) > mm._lib.NOALLOC_SCRATCH_BYTES
    st = mm.lib().mxfp4_moe_ffn_noalloc(None, sh.T, sh.H, sh.I, sh.E, sh.k, *([None] * 7),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 4
