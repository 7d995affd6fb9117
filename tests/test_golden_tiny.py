"""The oracle still produces the frozen tiny-workload record (see golden/make_golden.py)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_golden  # noqa: E402


def test_tiny_oracle_record_unchanged():
    ref = json.load(open(os.path.join(HERE, "golden", "tiny_oracle.json")))
    now = make_golden.tiny_record()
    assert now["initial_free"] == ref["initial_free"]
    for a, b in zip(now["frames"], ref["frames"]):
        for key in ("page_row", "slot_map", "free_list", "traj_pages", "traj_len"):
            assert a[key] == b[key], (a["t"], key)
        np.testing.assert_allclose(a["out_sum"], b["out_sum"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(a["out_abs_sum"], b["out_abs_sum"], rtol=1e-12)
        np.testing.assert_allclose(a["out_sample"], b["out_sample"], rtol=1e-12, atol=1e-14)
