"""The tracing build of the library (csrc/timeline.cuh, -DSA_TIMELINE) compiles
as a library of its own, exports the setters of its three traced units, and
leaves the library proper without them."""
import ctypes

import cross_layer_shared_b200 as sa
from cross_layer_shared_b200 import build


def test_timeline_build_exports_its_setters_and_the_proper_library_does_not():
    lt = ctypes.CDLL(build.build_timeline())
    for unit in ("indexer", "topk", "attn"):
        assert hasattr(lt, f"sa_timeline_set_{unit}")
    build.build()
    proper = ctypes.CDLL(sa.LIB_PATH)
    for unit in ("indexer", "topk", "attn"):
        assert not hasattr(proper, f"sa_timeline_set_{unit}")
