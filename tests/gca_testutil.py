"""Helpers shared by the GPU parity tests: run a workload through the C ABI, build the oracle
of the same stream, and compare."""
from __future__ import annotations

import numpy as np
import torch

import gca_inputs as gi
import oracle as orc
import paged_kv_cache_gca_b200 as gca

# Attention tolerance on bf16 inputs with fp32 accumulation (the stated bar).
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Relative Frobenius error bound: P is rounded to bf16 (relative error <= 2^-9 per weight) and
# the output is rounded to bf16 (<= 2^-9); with fp32 sums the combined relative error stays a
# few times 2^-9 ~ 2e-3. 1e-2 leaves margin and still fails an all-zero or half-missing output.
REL_FRO = 1e-2


def make_oracle(w: gi.Workload, rope_base=None, initial_free=None, source=None):
    free = gi.initial_free_list(w) if initial_free is None else initial_free
    src = source if source is not None else (lambda t: gi.draw_frame(w, t))
    return orc.GcaOracle(num_heads=w.num_heads, head_dim=w.head_dim, page_size=w.page_size,
                         grid_h=w.grid_h, grid_w=w.grid_w, num_special=w.num_special,
                         anchor_frames=w.anchor_frames, window_frames=w.window_frames,
                         keep_tokens=w.keep_tokens,
                         rope_base=w.rope_base if rope_base is None else rope_base,
                         initial_free=[int(x) for x in free], frame_source=src,
                         slot_of=lambda t: t % w.ring)


def device_ring(w: gi.Workload, device="cuda"):
    """[R, 3, T, H, D] bf16 on the device; frame t uses slot t % R."""
    return gi.draw_ring(w).to(device)


def check_attention(gpu_out: np.ndarray, ref: np.ndarray, what=""):
    d = np.abs(gpu_out.astype(np.float64) - ref)
    assert d.max() <= MAX_ABS, f"{what}: max abs {d.max():.3e}"
    assert d.mean() <= MEAN_ABS, f"{what}: mean abs {d.mean():.3e}"
    rel = np.linalg.norm(gpu_out - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= REL_FRO, f"{what}: relative error {rel:.3e}"
    return d.max(), d.mean(), rel


def check_book(cache: gca.GcaCache, book: orc.CacheBook, t: int):
    """Page table row, slot map, free list and trajectory pages: bit-exact."""
    v = cache.views()
    st = cache.state()
    assert st.frames_appended == book.frames
    assert st.traj_len == book.traj_len
    assert st.traj_pages == len(book.traj_pages)
    assert st.pages_in_use == book.pages_in_use()
    assert v["frame_pages"][t].cpu().tolist() == book.frame_pages[t]
    assert v["slot_map"].cpu().tolist() == book.slot_map
    assert cache.free_list() == list(book.alloc.free)
    assert v["traj_pages"].cpu().tolist() == book.traj_pages


def bf16_close(gpu: np.ndarray, ref: np.ndarray):
    """Rotated values: the GPU rotates in fp32 and rounds to bf16 once."""
    bound = np.abs(ref) * 2.0 ** -8 + 1e-6
    return np.all(np.abs(gpu - ref) <= bound)
