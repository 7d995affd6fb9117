"""Profiling helper of the benchmark: positions one cache at frame t of a workload and runs
gca_attend there.

For profilers: the appends of frames 0..t run first (cheap kernels), then exactly `--repeat`
attention calls at frame t, so a capture can select them with few launches before them.

    python profile_frame.py --workload w16_320 --frame 319 --repeat 1

With --batch N it instead creates N caches of the workload and runs --frame + 1 batched appends
(gca_append_frames over all N caches; frame of cache c at step t: ring slot (N t + c) mod R):

    python profile_frame.py --workload stack24x4 --batch 16 --frame 15

With --prefill it appends the workload's anchor (scale) frames and runs --repeat joint
attentions over them (gca_attend_prefill):

    python profile_frame.py --workload scale8 --prefill --repeat 1
"""
import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gca_inputs as gi  # noqa: E402
import paged_kv_cache_gca_b200 as gca  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="w16_320")
    ap.add_argument("--frame", type=int, default=-1)
    ap.add_argument("--repeat", type=int, default=1)
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--prefill", action="store_true")
    args = ap.parse_args()
    if args.batch > 0:
        return batched(args)
    if args.prefill:
        return prefill(args)
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


def prefill(args):
    w = gi.workload(args.workload)
    n = w.anchor_frames
    T, H, D = w.tokens_per_frame, w.num_heads, w.head_dim
    ring = gi.draw_ring(w, slots=n).cuda()
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    q_all = torch.empty((n * T, H, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_all)
    for t in range(n):
        q, k, v = ring[t]
        cache.append_frame(t, q, k, v, q_all[t * T:(t + 1) * T])
    for _ in range(args.repeat):
        cache.attend_prefill(n, q_all, out)
    torch.cuda.synchronize()
    status = cache.check()
    inf = cache.attend_info()
    print(f"{w.name} prefill of {n} frames: grid={inf.grid} split={inf.split} status={status}")
    sys.exit(0 if status == 0 else 1)


def batched(args):
    w = gi.workload(args.workload)
    n = args.batch
    T, H, D = w.tokens_per_frame, w.num_heads, w.head_dim
    ring = gi.draw_ring(w).cuda()
    R = ring.shape[0]
    caches = [gca.GcaCache(gca.config_for(w, gi.rope_base_for_layer(w, c % w.num_layers)))
              for c in range(n)]
    q_rot = [torch.empty((T, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    stream = torch.cuda.current_stream().cuda_stream
    for t in range(args.frame + 1):
        f = [ring[(n * t + c) % R] for c in range(n)]
        gca.gca_append_frames([c.handle for c in caches], [t] * n, [x[0].data_ptr() for x in f],
                              [x[1].data_ptr() for x in f], [x[2].data_ptr() for x in f],
                              [x.data_ptr() for x in q_rot], stream)
    torch.cuda.synchronize()
    status = max(c.check() for c in caches)
    print(f"{w.name} x{n}: {args.frame + 1} batched appends, status={status}")
    sys.exit(0 if status == 0 else 1)


if __name__ == "__main__":
    main()
