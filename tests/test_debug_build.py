"""The bounds-checked debug variant of the library (libsvdq_debug.so, built with
-DSVDQ_DEBUG_BOUNDS): it builds for sm_100a without a GPU, exports the same C
ABI as the release library, and reports itself through svdq_debug_build()."""
import ctypes
import re

import pytest

from diffusion_transformer_w4a4_b200 import build

HEADER = __import__("os").path.join(__import__("os").path.dirname(__file__), "..", "include", "svdq.h")


@pytest.fixture(scope="module")
def libs():
    rel = ctypes.CDLL(build.build())
    dbg = ctypes.CDLL(build.build(debug=True))
    return rel, dbg


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", text)) - {"svdq_status", "svdq_format"})


def test_debug_variant_exports_the_same_abi(libs):
    rel, dbg = libs
    for name in _declared():
        assert hasattr(rel, name), name
        assert hasattr(dbg, name), name


def test_debug_variant_reports_itself(libs):
    rel, dbg = libs
    assert rel.svdq_debug_build() == 0
    assert dbg.svdq_debug_build() == 1
    dbg.svdq_status_string.restype = ctypes.c_char_p
    assert b"BOUNDS" in dbg.svdq_status_string(7)
