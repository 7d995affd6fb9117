"""Full-size streams that drive the online softmax through its data-dependent branches, checked
against the CPU oracle element by element (the frame's queries attend over anchor, window and
trajectory pools: "LingBot-Map runs 10,000 frames on monocular video", section "How GCT's
Anchor-Pose-Trajectory Pools Make Monocular 3D Tractable"; GCT page, FlashInferBlock
compute_attention).

On the benchmark's inputs (q, k ~ N(0,1)/8) the bound |q| max|k| keeps every row's scores within
the lazy-rescale threshold after a piece's first key tile, so the exact row max, the O rescale and
merges of pieces with far-apart maxima never run. Here:
  * unit-variance q and k: the bound no longer rules out a rescale, so the exact row max runs on
    every tile;
  * needles: every query shares a direction with a few keys planted late in the key order (the
    last page of some window frames, and camera tokens that eviction keeps in the trajectory
    pool), so rows rescale O when they reach those tiles and the split-KV combine merges pieces
    whose maxima lie more than 2^8 apart.
The cache's branch counters show that each of these paths ran.
"""
import numpy as np
import pytest
import torch

import gca_inputs as gi
import paged_kv_cache_gca_b200 as gca
from gca_testutil import MAX_ABS, MEAN_ABS, REL_FRO, check_book, device_ring, make_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_gca_b200 import build

    build.build()
    torch.cuda.init()


def _np(x):
    return x.double().cpu().numpy()


# The stated bar (max abs 2e-2, mean abs 2e-3) is for the workloads' values ~N(0,1)/8. These
# streams draw q, k, v at unit scale, 8 times larger, and the bf16 rounding of P and of the
# output grows with the values: the absolute bars scale by the same factor. The relative
# Frobenius bound does not depend on the scale and stays as it is.
def check_scaled(gpu, ref, scale, what):
    f = scale / 0.125
    d = np.abs(gpu - ref)
    assert d.max() <= MAX_ABS * f, f"{what}: max abs {d.max():.3e}"
    assert d.mean() <= MEAN_ABS * f, f"{what}: mean abs {d.mean():.3e}"
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= REL_FRO, f"{what}: relative error {rel:.3e}"


def _stream(w, samples, rows=None, seed=0):
    cache = gca.GcaCache(gca.config_for(w), initial_free=gi.initial_free_list(w))
    o = make_oracle(w)
    ring = device_ring(w)
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    q_rot = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q_rot)
    rng = np.random.default_rng(seed)
    splits = 0
    for t in range(w.frames):
        q, k, v = ring[t % w.ring]
        cache.append_frame(t, q, k, v, q_rot)
        cache.attend(t, q_rot, out)
        o.append(t)
        if t in samples:
            torch.cuda.synchronize()
            splits += cache.attend_info().split
            check_book(cache, o.book, t)
            r = None if rows is None else np.sort(rng.choice(w.tokens_per_frame, rows, False))
            gpu = _np(out) if r is None else _np(out[torch.as_tensor(r, device="cuda")])
            check_scaled(gpu, o.attend(t, r), w.value_scale, f"{w.name} t={t}")
    assert cache.check() == 0
    assert splits == len(samples)  # every checked frame went through the combine
    return cache.counters()


NEEDLES = dict(needle_every=11, needle_slot=5, needle_q_gain=8.0, needle_k_gain=16.0)


def test_w16_320_unit_variance_exact_max_on_every_tile():
    w = gi.workload("w16_320").replace(value_scale=1.0)
    samples = {0, 16, 17, 18, 97, 200, 319}
    cnt = _stream(w, samples)
    # the Cauchy-Schwarz skip is off past the first tile of every piece
    assert cnt.exact_max_rows > 0


def test_w16_320_needles_rescale_and_wide_merges():
    w = gi.workload("w16_320").replace(value_scale=1.0, **NEEDLES)
    samples = {5, 16, 17, 60, 137, 250, 318, 319}
    cnt = _stream(w, samples)
    assert cnt.exact_max_rows > 0
    assert cnt.rescaled_rows > 0      # O was rescaled in tensor memory
    assert cnt.wide_merge_rows > 0    # the combine merged pieces with maxima > 2^8 apart


def test_long_trajectory_needles_multi_cta_split():
    # the 10,000-frame layer shape on a 1,500-frame stream: a trajectory pool of ~17.6k tokens
    # whose pages are spread over several CTAs of every work unit
    w = gi.workload("w32_10k").replace(frames=1500, value_scale=1.0, **NEEDLES)
    samples = {33, 34, 700, 1498, 1499}
    cnt = _stream(w, samples, rows=64, seed=3)
    assert cnt.rescaled_rows > 0 and cnt.wide_merge_rows > 0
