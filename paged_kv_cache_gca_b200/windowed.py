"""Windowed inference over one GCA cache: restarts with overlap past the RoPE training range.

The pages give the mode only as a command line ("--mode windowed --window_size 128
--overlap_keyframes 8": a fixed-size memory window that slides when a sequence exceeds the
~320 views the video RoPE was trained on; LingBot-Map 10,000-frame page, "Cloning and
Installing"; summary page, "Main features"). Reading used here: the video is cut into windows
of `window_size` frames, each starting `window_size - overlap` frames after the previous one,
so consecutive windows share `overlap` frames. At the start of every window the cache is reset
(gca_reset, the pages' clean_kv_cache) and the window's frames -- the overlap frames of the
previous window first -- are streamed as a fresh causal stream: frame g of window w is cache
frame (and RoPE time position) g - start(w), always below window_size.

This module is host scheduling only: every step of the path runs in the library's kernels.
"""
from __future__ import annotations

__all__ = ["window_starts", "windowed_schedule", "WindowedStream"]


def window_starts(total_frames: int, window_size: int, overlap: int) -> list[int]:
    """First video frame of every window; the last window ends at the last frame."""
    if window_size < 1 or not 0 <= overlap < window_size:
        raise ValueError("need 0 <= overlap < window_size")
    if total_frames <= 0:
        return []
    step = window_size - overlap
    starts = [0]
    while starts[-1] + window_size < total_frames:
        starts.append(starts[-1] + step)
    return starts


def windowed_schedule(total_frames: int, window_size: int, overlap: int):
    """Yields (window index, video frame g, local frame index) in processing order."""
    for w, s in enumerate(window_starts(total_frames, window_size, overlap)):
        for g in range(s, min(s + window_size, total_frames)):
            yield w, g, g - s


class WindowedStream:
    """Drives one GcaCache through a windowed schedule: resets it at every window start and
    appends / attends each frame at its local index."""

    def __init__(self, cache, window_size: int, overlap: int):
        self.cache = cache
        self.window_size = window_size
        self.overlap = overlap

    def step(self, local_t: int, q, k, v, q_rot, out, stream=None):
        """Appends frame local_t of the current window (local_t == 0 restarts the cache), then
        attends it. The caller supplies the frame's q, k, v: the network recomputes the overlap
        frames' tokens in the new window."""
        if local_t == 0:
            self.cache.reset(stream=stream)
        self.cache.append_frame(local_t, q, k, v, q_rot, stream=stream)
        self.cache.attend(local_t, q_rot, out, stream=stream)
