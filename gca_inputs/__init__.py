"""Seeded synthetic inputs and workload shapes for the GCA paged KV cache.

This module is shared by the CUDA path's tests/bench and by the CPU oracle. It holds
shapes, seeds and random draws only: no RoPE, no paging, no attention arithmetic.

Workload shapes follow the pages' streaming setup:
  * LingBot-Map at 518x378 with patch 14: the size is read as width x height, as image
    sizes are usually quoted, so a frame is 27 patch rows x 37 patch columns (999 patches),
    plus a camera token and register tokens ("How GCT's Anchor-Pose-Trajectory Pools Make
    Monocular 3D Tractable", first paragraph; GCT deep-dive page, "Practical Usage
    Example": img_size 518, patch_size 14, embed_dim 1024 = 16 heads x 64).
  * Sliding windows of 16-64 frames (same news page, pool list), the 320-view RoPE
    training range and 10k-frame streams (news page, "Cloning and Installing").
  * A 12-frame local window with no anchor and no trajectory pool (ABot-Recon page,
    "The Local Context Architecture").

Per-frame draws: q, k, v ~ N(0, 1) * scale in fp32, rounded to bf16. Frame t of a
stream takes its data from ring slot t mod ring, so a long stream reuses a bounded set
of distinct frames (RoPE positions still differ per frame).

Needles (optional, for tests of the online softmax's rescale path): every query gets a
common component q_gain * u_h along a fixed unit direction u_h per head, and in ring slots
with slot % needle_every == needle_slot the keys of token 0 (the camera token, which an
evicted frame keeps in the trajectory pool) and of the frame's last token (its last page)
are set to k_gain * u_h. Those keys then score far above all others, late in the key order.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "frame_seed",
    "draw_frame",
    "draw_ring",
    "initial_free_list",
    "rope_base_for_layer",
    "needle_directions",
]


@dataclass(frozen=True)
class Workload:
    name: str
    num_heads: int
    head_dim: int
    page_size: int
    grid_h: int
    grid_w: int
    num_special: int  # camera token + register tokens
    anchor_frames: int  # A
    window_frames: int  # W (includes the current frame)
    keep_tokens: int  # K kept per evicted frame (0 = no trajectory pool)
    frames: int  # frames per stream
    seed: int
    value_scale: float  # q,k,v ~ N(0,1) * value_scale
    permuted_free_list: bool
    ring: int  # distinct frames drawn; frame t uses slot t % ring
    num_pages: int  # physical page capacity of one cache
    max_frames: int  # RoPE table length (frame index must stay below it)
    rope_base: float = 10000.0
    num_layers: int = 1  # independent caches per stream (stack stress)
    num_streams: int = 1  # concurrent streams
    rope_base_varies_by_layer: bool = False
    needle_every: int = 0  # 0: no needles; else slots with slot % needle_every == needle_slot
    needle_slot: int = 0
    needle_q_gain: float = 0.0
    needle_k_gain: float = 0.0

    @property
    def tokens_per_frame(self) -> int:
        return self.num_special + self.grid_h * self.grid_w

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def rope_base_for_layer(w: Workload, layer: int) -> float:
    """Per-layer RoPE base for the stack workload: 10000 * 2**(layer/4) (the pages only say
    the bases vary; this spread is an input choice, not part of the method)."""
    if not w.rope_base_varies_by_layer:
        return w.rope_base
    return w.rope_base * (2.0 ** (layer / 4.0))


# The five stream workloads, then the scale-frame workload (8 scale frames processed jointly,
# which become the anchors, then a causal window of 16) and the causal camera head's cache (one
# camera token per frame, 32 heads x 64 = its 2048-wide input, the aggregator's window policy,
# one cache per layer of its 4-layer trunk). num_pages leaves a little headroom above the peak
# a stream needs.
WORKLOADS = {
    "tiny": Workload(
        name="tiny", num_heads=2, head_dim=64, page_size=16, grid_h=8, grid_w=8,
        num_special=4, anchor_frames=1, window_frames=2, keep_tokens=4, frames=6,
        seed=0, value_scale=1.0, permuted_free_list=True, ring=6, num_pages=24,
        max_frames=64),
    "w16_320": Workload(
        name="w16_320", num_heads=16, head_dim=64, page_size=16, grid_h=27, grid_w=37,
        num_special=5, anchor_frames=1, window_frames=16, keep_tokens=12, frames=320,
        seed=1, value_scale=0.125, permuted_free_list=False, ring=64, num_pages=1400,
        max_frames=320),
    "w64_1000": Workload(
        name="w64_1000", num_heads=16, head_dim=64, page_size=16, grid_h=27, grid_w=37,
        num_special=5, anchor_frames=1, window_frames=64, keep_tokens=12, frames=1000,
        seed=2, value_scale=0.125, permuted_free_list=True, ring=64, num_pages=4900,
        max_frames=1000),
    "w32_10k": Workload(
        name="w32_10k", num_heads=16, head_dim=64, page_size=16, grid_h=27, grid_w=37,
        num_special=5, anchor_frames=1, window_frames=32, keep_tokens=12, frames=10000,
        seed=3, value_scale=0.125, permuted_free_list=False, ring=64, num_pages=9650,
        max_frames=10000),
    "stack24x4": Workload(
        name="stack24x4", num_heads=16, head_dim=64, page_size=16, grid_h=27, grid_w=37,
        num_special=5, anchor_frames=0, window_frames=12, keep_tokens=0, frames=500,
        seed=4, value_scale=0.125, permuted_free_list=False, ring=64, num_pages=832,
        max_frames=500, num_layers=24, num_streams=4, rope_base_varies_by_layer=True),
    "scale8": Workload(
        name="scale8", num_heads=16, head_dim=64, page_size=16, grid_h=27, grid_w=37,
        num_special=5, anchor_frames=8, window_frames=16, keep_tokens=12, frames=48,
        seed=5, value_scale=0.125, permuted_free_list=True, ring=64, num_pages=1650,
        max_frames=48),
    "camera4": Workload(
        name="camera4", num_heads=32, head_dim=64, page_size=16, grid_h=0, grid_w=0,
        num_special=1, anchor_frames=1, window_frames=16, keep_tokens=1, frames=1024,
        seed=6, value_scale=0.125, permuted_free_list=False, ring=64, num_pages=96,
        max_frames=1024, num_layers=4),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def frame_seed(seed: int, slot: int) -> int:
    return seed * 1_000_003 + slot


def needle_directions(w: Workload) -> torch.Tensor:
    """fp32 [H, D]: one seeded unit direction per head (the needles' common direction)."""
    g = torch.Generator().manual_seed(frame_seed(w.seed, 999_983))
    u = torch.randn((w.num_heads, w.head_dim), generator=g, dtype=torch.float32)
    return u / u.norm(dim=1, keepdim=True)


def draw_frame(w: Workload, t: int):
    """bf16 (q, k, v), each [T, H, D], for frame t of workload w (CPU tensors)."""
    slot = t % w.ring
    g = torch.Generator().manual_seed(frame_seed(w.seed, slot))
    shape = (w.tokens_per_frame, w.num_heads, w.head_dim)
    out = []
    for _ in range(3):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        out.append(x * w.value_scale)
    if w.needle_every > 0:
        u = needle_directions(w)
        out[0] = out[0] + w.needle_q_gain * u[None]
        if slot % w.needle_every == w.needle_slot:
            out[1][0] = w.needle_k_gain * u
            out[1][-1] = w.needle_k_gain * u
    return tuple(x.to(torch.bfloat16) for x in out)


def draw_ring(w: Workload, slots: int | None = None):
    """Stacked bf16 ring [R, 3, T, H, D] of the distinct frames (slot r = frame r)."""
    r = w.ring if slots is None else slots
    frames = [torch.stack(draw_frame(w, s)) for s in range(r)]
    return torch.stack(frames)


def initial_free_list(w: Workload, seed: int | None = None) -> torch.Tensor:
    """Initial free-page order (int32). Identity, or a seeded permutation for the
    fragmented-pool workloads."""
    if not w.permuted_free_list and seed is None:
        return torch.arange(w.num_pages, dtype=torch.int32)
    s = w.seed if seed is None else seed
    g = torch.Generator().manual_seed(s)
    return torch.randperm(w.num_pages, generator=g).to(torch.int32)
