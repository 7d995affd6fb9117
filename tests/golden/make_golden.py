"""Writes tests/golden/tiny_oracle.json from the CPU oracle alone.

The file freezes the oracle's integer bookkeeping (page rows, slot maps, free list,
trajectory pages) and a digest of its fp64 attention outputs on the tiny workload, so that a
later change to the oracle shows up as a diff. Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import gca_inputs as gi  # noqa: E402
import oracle as orc  # noqa: E402


def tiny_record():
    w = gi.workload("tiny")
    o = orc.GcaOracle(num_heads=w.num_heads, head_dim=w.head_dim, page_size=w.page_size,
                      grid_h=w.grid_h, grid_w=w.grid_w, num_special=w.num_special,
                      anchor_frames=w.anchor_frames, window_frames=w.window_frames,
                      keep_tokens=w.keep_tokens, rope_base=w.rope_base,
                      initial_free=gi.initial_free_list(w).tolist(),
                      frame_source=lambda t: gi.draw_frame(w, t))
    frames = []
    for t in range(w.frames):
        o.append(t)
        out = o.attend(t)
        frames.append({
            "t": t,
            "page_row": o.book.frame_pages[t],
            "slot_map": o.book.slot_map,
            "free_list": list(o.book.alloc.free),
            "traj_pages": list(o.book.traj_pages),
            "traj_len": o.book.traj_len,
            "out_sum": float(out.sum()),
            "out_abs_sum": float(np.abs(out).sum()),
            "out_sample": [float(x) for x in out[::17, :, ::13].ravel()],
        })
    return {"workload": "tiny", "initial_free": gi.initial_free_list(w).tolist(),
            "frames": frames}


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(tiny_record(), f, indent=1)
    print("wrote", path)
