"""The oracle reproduces hand-derived neighbor lists (tests/golden/*.json).

Each fixture states its citation and the derivation of every value."""
import glob
import json
import os

import numpy as np
import pytest

GOLDEN = sorted(glob.glob(os.path.join(os.path.dirname(__file__), "golden", "tiny_*.json")))


@pytest.mark.parametrize("path", GOLDEN, ids=[os.path.basename(p) for p in GOLDEN])
def test_oracle_reproduces_golden(oracle, path):
    g = json.load(open(path))
    pos = np.array(g["positions"], np.float32)
    for fn in (oracle.build, oracle.bruteforce):
        nbr, cnt, ov = fn(pos, g["box"], g["cutoff"], g["skin"], g["capacity"])
        np.testing.assert_array_equal(nbr, np.array(g["rows"], np.int32))
        np.testing.assert_array_equal(cnt, np.array(g["counts"], np.int32))
        assert ov == g.get("overflow", False)
