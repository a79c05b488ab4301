"""The sweep's layer structure under the oracle.

The 54-layer sweep keeps each layer's text keys and values with that layer's
cache (one buffer: cached rows, then the text rows) and rotates the segment's
keys into a separate buffer each layer, so its spans differ from the
single-layer step's.  Two layers of that structure, at full 720p size, are
compared with the fp64 oracle on sampled query rows, among them the first and
last segment rows and the first and last text rows.
"""
import pytest

import bench

pytestmark = pytest.mark.gpu


def test_sweep_layers_match_the_oracle():
    step = bench.SweepStep(seed=1, layers=2)
    for layer in (0, 1):
        par = bench.sweep_parity(step, layer, n_rows=12)
        assert par["pass"], par
        assert par["rows"] >= 14
    assert int(step.err.item()) == 0
