"""ctypes binding of libmxfp4_moe.so (declared in include/mxfp4_moe.h).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  Torch supplies device memory and the current stream.  There
is no fallback: if the shared library is missing, or a tensor is not on a
CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
# MXFP4_MOE_CHECKS=1: the checked build (every caller-supplied index tested
# on the device before use; see build.py)
LIB_PATH = os.path.join(HERE, "libmxfp4_moe_checks.so" if os.environ.get("MXFP4_MOE_CHECKS") == "1"
                        else "libmxfp4_moe.so")

MOE_OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error",
                4: "workspace", 5: "device status"}
# device status details (second value of moe_get_device_status)
DEV_OK, DEV_BAD_EXPERT, DEV_NO_MASS, DEV_BAD_TOKEN, DEV_TIMEOUT, DEV_BAD_INDEX = 0, 1, 2, 3, 4, 5
(FFN_AUTO, FFN_FMA, FFN_TENSOR, FFN_TENSOR_F8, FFN_TENSOR_F4, FFN_TENSOR_FUSED,
 FFN_TENSOR_F8_PAIR) = 0, 1, 2, 3, 4, 5, 6

_c_int, _c_float, _c_size, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

# name -> (restype, argtypes)
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_c_int]),
    "moe_version": (_c_int, []),
    "moe_route_topk": (_c_int, [_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "moe_permute": (_c_int, [_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp]),
    "moe_route_permute": (_c_int, [_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxfp4_moe_ffn_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "mxfp4_moe_ffn": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                               _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_size, _vp]),
    "mxfp4_moe_ffn_variant": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                       _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_size,
                                       _c_int, _vp]),
    "mxfp4_moe_ffn_workspace_h": (_vp, [_vp]),
    "mxfp4_moe_ffn_noalloc": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                       _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_combine": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "moe_rms_norm": (_c_int, [_vp, _c_int, _c_int, _c_float, _vp, _vp]),
    "block_accept_greedy": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "block_accept_rejection": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                        _vp, _vp, _vp]),
    "block_accept_greedy_bonus": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "block_accept_rejection_bonus": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                              _vp, _vp, _vp]),
    "mxfp4_quantize": (_c_int, [_vp, ctypes.c_int64, _c_int, _vp, _vp, _vp]),
    "moe_get_device_status": (_c_int, [_vp, ctypes.POINTER(_c_int)]),
    "moe_clear_device_status": (_c_int, [_vp]),
    "moe_set_wait_limit_ns": (_c_int, [ctypes.c_uint64, _vp]),
}

_LIB = None


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: status {status} ({STATUS_NAMES.get(status, '?')})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load the CUDA library once; raise if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m mxfp4_moe_block_b200.build`"
                + (" --checks" if LIB_PATH.endswith("_checks.so") else ""))
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def moe_route_topk(logits, k, topk_idx=None, topk_w=None, stream=None):
    T, E = logits.shape
    dev = logits.device
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    _check(lib().moe_route_topk(_ptr(logits, torch.float32, "logits"), T, E, k,
                                _ptr(topk_idx, torch.int32), _ptr(topk_w, torch.float32),
                                _stream(stream)), "moe_route_topk")
    return topk_idx, topk_w


def moe_permute(topk_idx, E, expert_offsets=None, sorted_pair=None, pair_row=None, stream=None):
    T, k = topk_idx.shape
    dev = topk_idx.device
    P = T * k
    if expert_offsets is None:
        expert_offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    if sorted_pair is None:
        sorted_pair = torch.empty(P, dtype=torch.int32, device=dev)
    if pair_row is None:
        pair_row = torch.empty(P, dtype=torch.int32, device=dev)
    _check(lib().moe_permute(_ptr(topk_idx, torch.int32, "topk_idx"), T, k, E,
                             _ptr(expert_offsets, torch.int32), _ptr(sorted_pair, torch.int32),
                             _ptr(pair_row, torch.int32), _stream(stream)), "moe_permute")
    return expert_offsets, sorted_pair, pair_row


def moe_route_permute(logits, k, E=None, topk_idx=None, topk_w=None, expert_offsets=None,
                      sorted_pair=None, pair_row=None, stream=None):
    """moe_route_topk + moe_permute in one call (one kernel for T <= 128)."""
    T, E_ = logits.shape
    E = E_ if E is None else E
    dev = logits.device
    P = T * k
    i32 = dict(dtype=torch.int32, device=dev)
    topk_idx = torch.empty((T, k), **i32) if topk_idx is None else topk_idx
    topk_w = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_w is None else topk_w
    expert_offsets = torch.empty(E + 1, **i32) if expert_offsets is None else expert_offsets
    sorted_pair = torch.empty(P, **i32) if sorted_pair is None else sorted_pair
    pair_row = torch.empty(P, **i32) if pair_row is None else pair_row
    _check(lib().moe_route_permute(
        _ptr(logits, torch.float32, "logits"), T, E, k, _ptr(topk_idx, torch.int32),
        _ptr(topk_w, torch.float32), _ptr(expert_offsets, torch.int32),
        _ptr(sorted_pair, torch.int32), _ptr(pair_row, torch.int32), _stream(stream)),
        "moe_route_permute")
    return topk_idx, topk_w, expert_offsets, sorted_pair, pair_row


def mxfp4_moe_ffn_workspace_bytes(T, k, H, I):
    return int(lib().mxfp4_moe_ffn_workspace_bytes(T, k, H, I))


def alloc_workspace(T, k, H, I, device):
    n = mxfp4_moe_ffn_workspace_bytes(T, k, H, I)
    return torch.empty(n, dtype=torch.uint8, device=device)   # torch blocks are 256B-aligned


def mxfp4_moe_ffn(x, k, w13_codes, w13_scales, w2_codes, w2_scales, expert_offsets,
                  sorted_pair, y=None, workspace=None, variant=FFN_AUTO, stream=None):
    """x [T,H] bf16; weights uint8 as in the header; returns (y [T*k,H] f32, workspace)."""
    T, H = x.shape
    E, twoI, _ = w13_codes.shape
    I = twoI // 2
    dev = x.device
    if y is None:
        y = torch.empty((T * k, H), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = alloc_workspace(T, k, H, I, dev)
    _check(lib().mxfp4_moe_ffn_variant(
        _ptr(x, torch.bfloat16, "x"), T, H, I, E, k,
        _ptr(w13_codes, torch.uint8, "w13_codes"), _ptr(w13_scales, torch.uint8, "w13_scales"),
        _ptr(w2_codes, torch.uint8, "w2_codes"), _ptr(w2_scales, torch.uint8, "w2_scales"),
        _ptr(expert_offsets, torch.int32), _ptr(sorted_pair, torch.int32),
        _ptr(y, torch.float32, "y"), _ptr(workspace), workspace.numel(), variant,
        _stream(stream)), "mxfp4_moe_ffn")
    return y, workspace


NOALLOC_SCRATCH_BYTES = 8 << 20


def mxfp4_moe_ffn_noalloc(x, k, w13_codes, w13_scales, w2_codes, w2_scales, expert_offsets,
                          sorted_pair, y=None, stream=None):
    """mxfp4_moe_ffn without a caller-supplied workspace: the library uses its
    own fixed device scratch (NOALLOC_SCRATCH_BYTES), so the call allocates
    nothing when ``y`` is given.  For callers that may not allocate device
    memory; calls that overlap on the GPU share that scratch and race."""
    T, H = x.shape
    E, twoI, _ = w13_codes.shape
    I = twoI // 2
    if y is None:
        y = torch.empty((T * k, H), dtype=torch.float32, device=x.device)
    _check(lib().mxfp4_moe_ffn_noalloc(
        _ptr(x, torch.bfloat16, "x"), T, H, I, E, k,
        _ptr(w13_codes, torch.uint8, "w13_codes"), _ptr(w13_scales, torch.uint8, "w13_scales"),
        _ptr(w2_codes, torch.uint8, "w2_codes"), _ptr(w2_scales, torch.uint8, "w2_scales"),
        _ptr(expert_offsets, torch.int32), _ptr(sorted_pair, torch.int32),
        _ptr(y, torch.float32, "y"), _stream(stream)), "mxfp4_moe_ffn_noalloc")
    return y


def workspace_h(workspace, P, I):
    """View of the bf16 SwiGLU outputs h [P, I] kept in the FFN workspace."""
    return workspace[:P * I * 2].view(torch.bfloat16).view(P, I)


def moe_combine(y, pair_row, topk_w, residual=None, out=None, stream=None):
    T, k = topk_w.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
    _check(lib().moe_combine(_ptr(y, torch.float32, "y"), _ptr(pair_row, torch.int32),
                             _ptr(topk_w, torch.float32), T, k, H,
                             _ptr(residual, torch.bfloat16, "residual"),
                             _ptr(out, torch.bfloat16, "out"), _stream(stream)), "moe_combine")
    return out


def moe_rms_norm(x, eps=1e-6, out=None, stream=None):
    T, H = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(lib().moe_rms_norm(_ptr(x, torch.bfloat16, "x"), T, H, float(eps),
                              _ptr(out, torch.bfloat16, "out"), _stream(stream)), "moe_rms_norm")
    return out


def block_accept_greedy(logits, draft, accept_len=None, next_token=None, stream=None):
    S, K, V = logits.shape
    dev = logits.device
    if accept_len is None:
        accept_len = torch.empty(S, dtype=torch.int32, device=dev)
    if next_token is None:
        next_token = torch.empty(S, dtype=torch.int32, device=dev)
    _check(lib().block_accept_greedy(_ptr(logits, torch.float32, "logits"),
                                     _ptr(draft, torch.int32, "draft"), S, K, V,
                                     _ptr(accept_len, torch.int32), _ptr(next_token, torch.int32),
                                     _stream(stream)), "block_accept_greedy")
    return accept_len, next_token


def block_accept_rejection(p, q, draft, u_accept, u_resample, accept_len=None,
                           next_token=None, stream=None):
    S, K, V = p.shape
    dev = p.device
    if accept_len is None:
        accept_len = torch.empty(S, dtype=torch.int32, device=dev)
    if next_token is None:
        next_token = torch.empty(S, dtype=torch.int32, device=dev)
    _check(lib().block_accept_rejection(
        _ptr(p, torch.float32, "p"), _ptr(q, torch.float32, "q"), _ptr(draft, torch.int32, "draft"),
        _ptr(u_accept, torch.float32, "u_accept"), _ptr(u_resample, torch.float32, "u_resample"),
        S, K, V, _ptr(accept_len, torch.int32), _ptr(next_token, torch.int32), _stream(stream)),
        "block_accept_rejection")
    return accept_len, next_token


def block_accept_greedy_bonus(logits, draft, accept_len=None, next_token=None, stream=None):
    """logits [S, K+1, V] (row K: the target after the block), draft [S, K]."""
    S, K1, V = logits.shape
    K = K1 - 1
    if tuple(draft.shape) != (S, K):
        raise ValueError("draft must be [S, K] for logits [S, K+1, V]")
    dev = logits.device
    if accept_len is None:
        accept_len = torch.empty(S, dtype=torch.int32, device=dev)
    if next_token is None:
        next_token = torch.empty(S, dtype=torch.int32, device=dev)
    _check(lib().block_accept_greedy_bonus(_ptr(logits, torch.float32, "logits"),
                                           _ptr(draft, torch.int32, "draft"), S, K, V,
                                           _ptr(accept_len, torch.int32),
                                           _ptr(next_token, torch.int32), _stream(stream)),
           "block_accept_greedy_bonus")
    return accept_len, next_token


def block_accept_rejection_bonus(p, q, draft, u_accept, u_resample, accept_len=None,
                                 next_token=None, stream=None):
    """p [S, K+1, V] (row K: the target after the block), q [S, K, V]."""
    S, K1, V = p.shape
    K = K1 - 1
    if tuple(q.shape) != (S, K, V) or tuple(draft.shape) != (S, K):
        raise ValueError("q [S, K, V] and draft [S, K] for p [S, K+1, V]")
    dev = p.device
    if accept_len is None:
        accept_len = torch.empty(S, dtype=torch.int32, device=dev)
    if next_token is None:
        next_token = torch.empty(S, dtype=torch.int32, device=dev)
    _check(lib().block_accept_rejection_bonus(
        _ptr(p, torch.float32, "p"), _ptr(q, torch.float32, "q"), _ptr(draft, torch.int32, "draft"),
        _ptr(u_accept, torch.float32, "u_accept"), _ptr(u_resample, torch.float32, "u_resample"),
        S, K, V, _ptr(accept_len, torch.int32), _ptr(next_token, torch.int32), _stream(stream)),
        "block_accept_rejection_bonus")
    return accept_len, next_token


def mxfp4_quantize(w, codes=None, scales=None, stream=None):
    """w [R, K] bf16 -> (codes [R, K/2] uint8, scales [R, K/32] uint8), OCP MXFP4."""
    R, K = w.shape
    dev = w.device
    if codes is None:
        codes = torch.empty((R, K // 2), dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty((R, K // 32), dtype=torch.uint8, device=dev)
    _check(lib().mxfp4_quantize(_ptr(w, torch.bfloat16, "w"), R, K, _ptr(codes, torch.uint8),
                                _ptr(scales, torch.uint8), _stream(stream)), "mxfp4_quantize")
    return codes, scales


def moe_get_device_status(stream=None):
    """(status, detail): synchronises the stream and reads the status word."""
    d = ctypes.c_int(0)
    st = lib().moe_get_device_status(_stream(stream), ctypes.byref(d))
    return st, d.value


def moe_clear_device_status(stream=None):
    _check(lib().moe_clear_device_status(_stream(stream)), "moe_clear_device_status")


def moe_set_wait_limit_ns(ns=0, stream=None):
    """Limit of the FFN kernels' bounded waits (0 = the 2 s default)."""
    _check(lib().moe_set_wait_limit_ns(int(ns), _stream(stream)), "moe_set_wait_limit_ns")
