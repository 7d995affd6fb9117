"""Positions one cache at frame t of a workload and runs gca_attend there once.

For profilers: the appends of frames 0..t run first (cheap kernels), then exactly `--repeat`
attention calls at frame t, so a capture can select them with few launches before them.

    python -m paged_kv_cache_gca_b200.profile_frame --workload w16_320 --frame 319 --repeat 1
"""
import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gca_inputs as gi  # noqa: E402
import paged_kv_cache_gca_b200 as gca  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="w16_320")
    ap.add_argument("--frame", type=int, default=-1)
    ap.add_argument("--repeat", type=int, default=1)
    args = ap.parse_args()
    w = gi.workload(args.workload)
    t_last = w.frames - 1 if args.frame < 0 else args.frame
    T, H, D = w.tokens_per_frame, w.num_heads, w.head_dim
    ring = gi.draw_ring(w).cuda()
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    q_rot = torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)
    for t in range(t_last + 1):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
    for _ in range(args.repeat):
        cache.attend(t_last, q_rot, out)
    torch.cuda.synchronize()
    status = cache.check()
    inf = cache.attend_info()
    print(f"{w.name} t={t_last}: Nk={inf.visible_keys} grid={inf.grid} split={inf.split} "
          f"status={status}")
    sys.exit(0 if status == 0 else 1)


if __name__ == "__main__":
    main()
