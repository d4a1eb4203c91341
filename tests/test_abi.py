"""The C-ABI library loads on a machine without a GPU and exports every
function include/*.h declares; the binding declares the same set."""
import glob
import os
import re

import pytest

from mxfp4_moe_block_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            if m.group(1) not in ("if", "while", "for", "return"):
                names.append(m.group(1))
    return sorted(set(names))


@pytest.fixture(scope="module")
def library():
    build.build()
    return _lib.lib()


def test_header_declares_the_six_calls():
    d = declared_functions()
    for n in ("moe_route_topk", "moe_permute", "mxfp4_moe_ffn", "moe_combine",
              "block_accept_greedy", "block_accept_rejection"):
        assert n in d


def test_every_declared_symbol_is_exported(library):
    for n in declared_functions():
        assert hasattr(library, n), n


def test_binding_covers_the_header():
    assert set(declared_functions()) == set(_lib.SIGNATURES)


def test_host_only_calls(library):
    assert library.moe_version() == 10000
    assert library.moe_status_string(4) == b"workspace too small or misaligned"
    assert library.mxfp4_moe_ffn_workspace_bytes(8, 8, 7168, 2048) >= 64 * 2048 * 2
    # argument checks return before any CUDA call
    assert library.moe_route_topk(None, 4, 8, 9, None, None, None) == 1
    assert library.block_accept_greedy(None, None, 1, 0, 10, None, None, None) == 1
    # a vocabulary beyond the greedy key's 26 token bits is refused up front
    # (non-null dummy addresses: the size check comes before any device use)
    assert library.block_accept_greedy(16, 16, 1, 8, (1 << 26) + 1, 16, 16, None) == 2


def header_enum_values(prefix):
    """Name -> value of the header's enumerators that start with `prefix`."""
    vals = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h, encoding="utf-8").read(), flags=re.S)
        for m in re.finditer(r"\b(" + prefix + r"\w*)\s*=\s*(-?\d+)", text):
            vals[m.group(1)] = int(m.group(2))
    return vals


def test_ffn_variant_constants_match_the_header():
    v = header_enum_values("MOE_FFN_")
    assert v == {"MOE_FFN_AUTO": 0, "MOE_FFN_FMA": 1, "MOE_FFN_TENSOR": 2, "MOE_FFN_TENSOR_F8": 3,
                 "MOE_FFN_TENSOR_F4": 4, "MOE_FFN_TENSOR_FUSED": 5, "MOE_FFN_TENSOR_F8_PAIR": 6}
    for name, val in v.items():
        assert getattr(_lib, name[len("MOE_"):]) == val, name


def test_variant_range_is_checked(library):
    # a variant past the last enumerator is refused before any device use
    last = max(header_enum_values("MOE_FFN_").values())
    assert library.mxfp4_moe_ffn_variant(None, 1, 512, 256, 8, 2, None, None, None, None,
                                         None, None, None, None, 0, last + 1, None) == 1


def test_device_detail_constants_match_the_header():
    v = header_enum_values("MOE_DEV_")
    assert v == {"MOE_DEV_OK": 0, "MOE_DEV_BAD_EXPERT": 1, "MOE_DEV_NO_MASS": 2,
                 "MOE_DEV_BAD_TOKEN": 3, "MOE_DEV_TIMEOUT": 4, "MOE_DEV_BAD_INDEX": 5}
    for name, val in v.items():
        assert getattr(_lib, name[len("MOE_"):]) == val, name


def test_checked_build_exports_every_declared_symbol():
    """The MOE_CHECKS build (libmxfp4_moe_checks.so) is the same ABI."""
    import ctypes
    path = build.build(checks=True)
    assert path.endswith("libmxfp4_moe_checks.so")
    L = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(L, n), n
    assert L.moe_version() == 10000
