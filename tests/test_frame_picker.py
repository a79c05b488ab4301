"""The library's frame picker against the page's printed list and the oracle."""
import ctypes
import json
import os

import pytest

import kv_cached_segment_b200 as nm
import oracle
from kv_cached_segment_b200 import _build


@pytest.fixture(scope="module", autouse=True)
def _lib():
    _build.build()
    nm.load_library()


def test_printed_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "frame_picker_T360.json")))
    assert nm.temporal_context_frames(g["n_past"], g["budget"], g["gamma"]) == g["kept_frames"]


def test_matches_oracle_on_a_grid():
    for gamma in (1.0, 2.0, 3.0, 0.5):
        for budget in (1, 2, 5, 18, 40):
            for t in list(range(0, 80)) + [119, 240, 360, 361, 1000, 1999, 7200]:
                want = oracle.temporal_context_frame_indices(t, budget, gamma).tolist()
                assert nm.temporal_context_frames(t, budget, gamma) == want, (t, budget, gamma)


def test_errors():
    lib = nm.load_library()
    n = ctypes.c_int32(0)
    out = (ctypes.c_int32 * 4)()
    assert lib.nomas_temporal_context_frames(-1, 18, 2.0, out, 4, ctypes.byref(n)) == nm.NOMAS_ERR_INVALID_ARG
    assert lib.nomas_temporal_context_frames(10, 18, float("nan"), out, 4, ctypes.byref(n)) == nm.NOMAS_ERR_INVALID_ARG
    assert lib.nomas_temporal_context_frames(100, 18, 2.0, out, 4, ctypes.byref(n)) == nm.NOMAS_ERR_CAPACITY
    assert lib.nomas_temporal_context_frames(100, 18, 2.0, out, 4, None) == nm.NOMAS_ERR_INVALID_ARG
    assert lib.nomas_temporal_context_frames(0, 18, 2.0, None, 0, ctypes.byref(n)) == nm.NOMAS_OK and n.value == 0
