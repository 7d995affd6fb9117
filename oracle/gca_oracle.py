"""CPU oracle for the GCA paged KV cache: fp64 NumPy and plain Python.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module: only the tests,
the smoke check and the benchmark's CPU-baseline / reference arm do. It shares no code with
the CUDA library (no kernels, headers, tables or helpers); the only common dependency is the
seeded input module `gca_inputs`, which holds no method arithmetic.

Sources (web pages, cited by title and section):
  [GCT]   "How the Geometric Context Transformer Enables Streaming 3D Reconstruction in
          LingBot-Map" -- sections "Causal Aggregation with KV-Cache Management"
          (KV-Cache Initialization, 3D Rotary Positional Embeddings), "Attention Blocks:
          FlashInfer vs. SDPA" (FlashInferBlock), and the FAQ on scale frames / causality.
  [POOLS] "LingBot-Map runs 10,000 frames on monocular video" -- section "How GCT's
          Anchor-Pose-Trajectory Pools Make Monocular 3D Tractable".
  [ABOT]  "Stop hoarding memory: how ABot-Recon reconstructs infinite 3D streams with a fixed
          12-frame window" -- section "The Local Context Architecture".

What the pages fix: a frame's tokens get 3D (t,y,x) RoPE with t the global frame index
[GCT, 3D RoPE]; the frame's K/V are appended to a paged cache, frames that left the window are
evicted, then the frame's queries attend over the cache [GCT, FlashInferBlock]; the cache holds
three pools -- anchor frame(s), a window of recent frames, and a trajectory pool that keeps a
few tokens of each evicted frame [POOLS]; attention across frames is causal [GCT, FAQ "Why are
scale frames processed differently"]; a 12-frame window means 11 cached frames plus the current
one [ABOT].

Parity unpinned (by the pages): the conventions R1, R2 and R6 below are readings. The pins in
the tests check that this code implements them as written (closed forms, invariants, hand-derived
sequences), but no page fixes the conventions themselves.

Readings where the pages are silent (each is listed in the design notes):
  R1 token order in a frame: [camera, registers, patches row-major over (grid_h, grid_w)].
  R2 RoPE band split d_y = d_x = 2*floor(D/6), d_t = D - d_y - d_x, order (t, y, x);
     interleaved pairs (2j, 2j+1); pair j of a band of width d turns by pos * base**(-2j/d);
     a patch at (row r, col c) sits at (t, r+1, c+1), special tokens at (t, 0, 0); q and k
     rotate, v does not; k is cached rotated.
  R3 pools at step t, in order append -> evict -> attend: anchor = frames 0..A-1;
     window = frames max(A, t-W+1)..t (W counts the current frame); trajectory = kept tokens
     of frames A..t-W. Before frame A the frame sees frames 0..t. No mask inside a frame.
  R4 kept tokens: K <= S -> tokens 0..K-1; else all S special tokens plus patches
     S + j*floor(P/(K-S)), j = 0..K-S-1. Trajectory order: by evicted frame, then kept index.
  R5 softmax scale 1/sqrt(D).
  R6 allocator: FIFO free list. Append pops ceil(T/ps) pages for the frame (frames start
     page-aligned); eviction then copies the kept tokens to the trajectory tail, popping a
     page whenever the tail page is full (trajectory pages are dense and never freed), and
     finally pushes the evicted frame's pages to the tail in row order. Anchor pages are
     never freed. Reset restores the initial order.
  R11 keyframe-only caching [GCT, FlashInferBlock `skip_append`; Streaming Inference API
     `keyframe_interval`]: video frame g is a keyframe when g % N == 0. Cache frames ("slots")
     count the kept frames; a keyframe takes the next slot with the normal append -> evict ->
     attend. A non-keyframe takes the next slot transiently: append (pages popped, nothing
     evicted) -> attend -> roll back (its pages return to the free-list head in reverse order,
     which restores the allocator exactly). With no eviction before its attention, a transient
     frame at slot s sees the anchors, window slots max(A, s-W)..s (up to W+1 frames, itself
     included) and the kept tokens of slots A..s-W-1. The RoPE time position of a slot is the
     global index g of the video frame it holds [GCT, 3D RoPE]; without keyframes g = slot.
  R12 scale-frame prefill [GCT, Streaming Inference API step 2 and the FAQ on scale frames]:
     the first n scale frames (n <= A: they become the anchor pool) are processed jointly
     with bidirectional attention: after their appends, the queries of all n frames (frame
     by frame, n*T rows) attend over every token of frames 0..n-1, with no mask across them.
     Streaming then continues causally (R3).
  R14 windowed restart [LingBot-Map 10,000-frame page, "Cloning and Installing"; summary page,
     "Main features": --mode windowed --window_size N --overlap_keyframes V]: windows of N
     video frames, each starting N - V frames after the previous one (the last one ends at the
     last frame); at each window start the cache restarts empty and the window's frames (the
     previous window's last V first) stream causally with local indices g - start.
"""
from __future__ import annotations

import math
from collections import deque

import numpy as np

__all__ = [
    "OutOfPages",
    "rope_band_widths",
    "token_positions",
    "rope_angles",
    "rotate_pairs",
    "kept_token_indices",
    "pool_frames",
    "visible_keys",
    "visible_key_count",
    "keyframe_stream",
    "windowed_frames",
    "softmax_attention",
    "FifoPages",
    "CacheBook",
    "GcaOracle",
]


class OutOfPages(RuntimeError):
    pass


# --------------------------------------------------------------------------------------
# 3D RoPE [GCT, "3D Rotary Positional Embeddings"; reading R2]
# --------------------------------------------------------------------------------------

def rope_band_widths(head_dim: int):
    """(d_t, d_y, d_x): two spatial bands of 2*floor(D/6) dims each, the rest for time."""
    d_sp = 2 * (head_dim // 6)
    return head_dim - 2 * d_sp, d_sp, d_sp


def token_positions(t: int, num_special: int, grid_h: int, grid_w: int) -> np.ndarray:
    """int64 [T, 3] positions (t, y, x) of frame t's tokens, token order R1."""
    T = num_special + grid_h * grid_w
    pos = np.zeros((T, 3), dtype=np.int64)
    pos[:, 0] = t
    for p in range(grid_h * grid_w):
        r, c = divmod(p, grid_w)
        pos[num_special + p, 1] = r + 1
        pos[num_special + p, 2] = c + 1
    return pos


def rope_angles(pos: np.ndarray, head_dim: int, base: float) -> np.ndarray:
    """fp64 [N, D/2] rotation angle of every pair: band b of width d gives pair j the
    angle pos_b * base**(-2j/d)."""
    widths = rope_band_widths(head_dim)
    cols = []
    for b, d in enumerate(widths):
        j = np.arange(d // 2, dtype=np.float64)
        inv_freq = np.power(float(base), -2.0 * j / d)
        cols.append(pos[:, b : b + 1].astype(np.float64) * inv_freq[None, :])
    return np.concatenate(cols, axis=1)


def rotate_pairs(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate interleaved pairs (x[2j], x[2j+1]) by angles[..., j].

    x: fp64 [N, H, D]; angles: [N, D/2]. Returns fp64 [N, H, D].
    """
    a = x[..., 0::2]
    b = x[..., 1::2]
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


# --------------------------------------------------------------------------------------
# Pools [POOLS; GCT FlashInferBlock order append -> evict -> attend; readings R3, R4]
# --------------------------------------------------------------------------------------

def kept_token_indices(num_special: int, num_patches: int, keep: int):
    """Token indices an evicted frame keeps in the trajectory pool (reading R4)."""
    if keep <= 0:
        return []
    if keep <= num_special:
        return list(range(keep))
    extra = keep - num_special
    stride = num_patches // extra
    if stride < 1:
        raise ValueError("more kept patches than patches")
    return list(range(num_special)) + [num_special + j * stride for j in range(extra)]


def pool_frames(t: int, A: int, W: int, transient: bool = False):
    """(anchor frames, window frames, evicted frames) visible at step t (reading R3); for a
    transient (non-keyframe) frame at slot t, nothing was evicted before its attention (R11)."""
    if t < A:
        return list(range(t + 1)), [], []
    anchor = list(range(A))
    w0 = max(A, t - W + (0 if transient else 1))
    window = list(range(w0, t + 1))
    evicted = list(range(A, w0))
    return anchor, window, evicted


def visible_keys(t: int, A: int, W: int, T: int, kept, transient: bool = False):
    """Pool-ordered list of (frame, token) keys that frame t's queries see."""
    anchor, window, evicted = pool_frames(t, A, W, transient)
    keys = [(f, i) for f in anchor for i in range(T)]
    keys += [(f, i) for f in window for i in range(T)]
    keys += [(f, i) for f in evicted for i in kept]
    return keys


def visible_key_count(t: int, A: int, W: int, T: int, K: int, transient: bool = False) -> int:
    anchor, window, evicted = pool_frames(t, A, W, transient)
    return (len(anchor) + len(window)) * T + len(evicted) * K


# --------------------------------------------------------------------------------------
# Attention: softmax(q k^T / sqrt(D)) v over the visible keys [GCT compute_attention; R5]
# --------------------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """fp64 attention of one head. q [Nq, D], k [Nk, D], v [Nk, D] -> [Nq, D]."""
    d = q.shape[-1]
    s = (q @ k.T) / math.sqrt(d)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ v) / p.sum(axis=1, keepdims=True)


# --------------------------------------------------------------------------------------
# Page bookkeeping [GCT "paged KV cache", KV-Cache Initialization; reading R6]
# --------------------------------------------------------------------------------------

class FifoPages:
    """FIFO free list of physical page ids."""

    def __init__(self, initial_order):
        self.initial = [int(p) for p in initial_order]
        self.free = deque(self.initial)

    def pop(self) -> int:
        if not self.free:
            raise OutOfPages("free list empty")
        return self.free.popleft()

    def push(self, page: int) -> None:
        self.free.append(page)

    def reset(self) -> None:
        self.free = deque(self.initial)

    def unpop(self, page: int) -> None:
        """Return a page to the head (undo of the last pop)."""
        self.free.appendleft(page)


class CacheBook:
    """Integer state of one cache: page rows per frame, slot map, trajectory pages.

    Spells out the allocator reading R6 step by step; every GPU page id is compared with it.
    """

    def __init__(self, *, T, page_size, anchor_frames, window_frames, kept, initial_free):
        self.T = T
        self.ps = page_size
        self.A = anchor_frames
        self.W = window_frames
        self.kept = list(kept)
        self.ppf = -(-T // page_size)
        self.alloc = FifoPages(initial_free)
        self.reset()

    def reset(self):
        self.alloc.reset()
        self.frame_pages = {}  # frame -> list of page ids (live frames)
        self.all_rows = {}  # frame -> page row (also kept after eviction, for inspection)
        self.traj_pages = []
        self.traj_tokens = []  # (frame, token) per trajectory slot, in order
        self.frames = 0
        self.slot_map = []
        self.transient = False  # the last append was a non-keyframe awaiting rollback (R11)

    @property
    def traj_len(self):
        return len(self.traj_tokens)

    def pages_in_use(self):
        return sum(len(r) for r in self.frame_pages.values()) + len(self.traj_pages)

    def append(self, t: int, transient: bool = False):
        if t != self.frames or self.transient:
            raise ValueError("frames must be appended in order (a transient frame first rolls back)")
        # 1. the new frame's pages, popped in order
        row = [self.alloc.pop() for _ in range(self.ppf)]
        self.frame_pages[t] = row
        self.all_rows[t] = row
        self.slot_map = [row[i // self.ps] * self.ps + i % self.ps for i in range(self.T)]
        self.transient = transient
        # 2. eviction of the frame that left the window (none for a transient frame, R11)
        e = t - self.W
        if e >= self.A and not transient:
            for i in self.kept:
                if self.traj_len % self.ps == 0:
                    self.traj_pages.append(self.alloc.pop())
                self.traj_tokens.append((e, i))
            for p in self.frame_pages.pop(e):
                self.alloc.push(p)
        self.frames += 1

    def rollback(self, t: int):
        """Undo the transient append of frame t: its pages go back to the free-list head in
        reverse order, so the free list is exactly what it was before the append (R11)."""
        if not self.transient or t != self.frames - 1:
            raise ValueError("only a transient last frame rolls back")
        row = self.frame_pages.pop(t)
        self.all_rows.pop(t)
        for p in reversed(row):
            self.alloc.unpop(p)
        self.frames -= 1
        self.transient = False

    def location_of(self, frame: int, token: int):
        """(page, slot) that holds a live frame's token."""
        row = self.frame_pages[frame]
        return row[token // self.ps], token % self.ps

    def traj_location(self, n: int):
        return self.traj_pages[n // self.ps], n % self.ps


# --------------------------------------------------------------------------------------
# Whole stream
# --------------------------------------------------------------------------------------

class GcaOracle:
    """fp64 oracle of one GCA cache fed by a seeded synthetic stream.

    `frame_source(g)` returns the bf16 (q, k, v) tensors [T, H, D] of video frame g (torch or
    numpy); they are widened exactly. `slot_of(g)` names the distinct input frame that frame g
    reuses (identity by default), so long streams keep a bounded set of raw frames in memory.
    Cache frame (slot) t holds video frame gidx[t]: t itself unless `append` was given another
    global index (keyframe streams, R11); its RoPE time position and its inputs are those of
    gidx[t].
    """

    def __init__(self, *, num_heads, head_dim, page_size, grid_h, grid_w, num_special,
                 anchor_frames, window_frames, keep_tokens, rope_base, initial_free,
                 frame_source, slot_of=None):
        self.H = num_heads
        self.D = head_dim
        self.ps = page_size
        self.gh = grid_h
        self.gw = grid_w
        self.S = num_special
        self.P = grid_h * grid_w
        self.T = self.S + self.P
        self.A = anchor_frames
        self.W = window_frames
        self.K = keep_tokens
        self.base = rope_base
        self.kept = kept_token_indices(self.S, self.P, self.K)
        self.source = frame_source
        self.slot_of = slot_of if slot_of is not None else (lambda t: t)
        self.book = CacheBook(T=self.T, page_size=page_size, anchor_frames=anchor_frames,
                              window_frames=window_frames, kept=self.kept,
                              initial_free=initial_free)
        self._raw = {}  # slot -> (q, k, v) as float32 arrays (exact copies of bf16)
        self._pos = token_positions(0, self.S, self.gh, self.gw)
        self.gidx = {}  # cache frame -> global (video) frame index, when not the identity
        self.rpos = {}  # cache frame -> RoPE time position, when not its global index (R14)

    def global_index(self, t):
        return self.gidx.get(int(t), int(t))

    def rope_index(self, t):
        return self.rpos.get(int(t), self.global_index(t))

    # inputs ---------------------------------------------------------------------------
    def raw32(self, t):
        g = self.global_index(t)
        slot = self.slot_of(g)
        if slot not in self._raw:
            q, k, v = self.source(g)
            self._raw[slot] = tuple(_to_f32(x) for x in (q, k, v))
        return self._raw[slot]

    def raw(self, t):
        return tuple(x.astype(np.float64) for x in self.raw32(t))

    def positions(self, frames, tokens):
        """int64 [N, 3] positions of the (frame, token) pairs."""
        frames = np.asarray(frames, dtype=np.int64)
        tokens = np.asarray(tokens, dtype=np.int64)
        pos = self._pos[tokens].copy()
        pos[:, 0] = ([self.rope_index(f) for f in frames] if (self.gidx or self.rpos)
                     else frames)
        return pos

    def q_rot(self, t, rows=None):
        toks = np.arange(self.T) if rows is None else np.asarray(rows)
        q = self.raw32(t)[0][toks].astype(np.float64)
        ang = rope_angles(self.positions(np.full(len(toks), t), toks), self.D, self.base)
        return rotate_pairs(q, ang)

    def k_rot(self, t, tokens=None):
        toks = np.arange(self.T) if tokens is None else np.asarray(tokens)
        k = self.raw32(t)[1][toks].astype(np.float64)
        ang = rope_angles(self.positions(np.full(len(toks), t), toks), self.D, self.base)
        return rotate_pairs(k, ang)

    # bookkeeping ----------------------------------------------------------------------
    def append(self, t, g=None, transient=False, rope_pos=None):
        """Append cache frame t holding video frame g (default t), rotated at time rope_pos
        (default g); transient: a non-keyframe that will roll back (R11)."""
        self.book.append(t, transient)
        if g is None or g == t:
            self.gidx.pop(t, None)
        else:
            self.gidx[t] = int(g)
        if rope_pos is None or rope_pos == self.global_index(t):
            self.rpos.pop(t, None)
        else:
            self.rpos[t] = int(rope_pos)

    def rollback(self, t):
        self.book.rollback(t)
        self.gidx.pop(t, None)
        self.rpos.pop(t, None)

    def restart(self):
        """Empty cache (reset, R14)."""
        self.book.reset()
        self.gidx.clear()
        self.rpos.clear()

    def _transient(self, t):
        return self.book.transient and t == self.book.frames - 1

    def visible(self, t):
        return visible_keys(t, self.A, self.W, self.T, self.kept, self._transient(t))

    def key_index(self, t):
        """(frames, tokens) int arrays of the keys frame t sees, in pool order."""
        anchor, window, evicted = pool_frames(t, self.A, self.W, self._transient(t))
        full = np.asarray(anchor + window, dtype=np.int64)
        fr = [np.repeat(full, self.T)]
        tk = [np.tile(np.arange(self.T, dtype=np.int64), len(full))]
        if evicted and self.kept:
            ev = np.asarray(evicted, dtype=np.int64)
            fr.append(np.repeat(ev, len(self.kept)))
            tk.append(np.tile(np.asarray(self.kept, dtype=np.int64), len(ev)))
        return np.concatenate(fr), np.concatenate(tk)

    def gather_head(self, t, h, frames=None, tokens=None, angles=None):
        """fp64 (K_rot, V) [Nk, D] of head h over the keys frame t sees, in pool order."""
        if frames is None:
            frames, tokens = self.key_index(t)
        if angles is None:
            angles = rope_angles(self.positions(frames, tokens), self.D, self.base)
        k = np.empty((len(frames), self.D), dtype=np.float64)
        v = np.empty((len(frames), self.D), dtype=np.float64)
        slots = np.asarray([self.slot_of(self.global_index(f)) for f in frames])
        for s in np.unique(slots):
            sel = np.nonzero(slots == s)[0]
            f0 = int(frames[sel[0]])
            _, kr, vr = self.raw32(f0)
            k[sel] = kr[tokens[sel], h, :]
            v[sel] = vr[tokens[sel], h, :]
        k = rotate_pairs(k[:, None, :], angles)[:, 0, :]
        return k, v

    def attend_prefill(self, n, rows=None):
        """fp64 output [len(rows), H, D] of the joint (bidirectional) attention of scale frames
        0..n-1 (R12); rows index the n*T concatenated query rows (frame-major)."""
        if not (1 <= n <= max(self.A, 1)) or self.book.frames != n:
            raise ValueError("prefill needs exactly the first n <= A frames appended")
        r = np.arange(n * self.T) if rows is None else np.asarray(rows)
        frame_of, tok_of = r // self.T, r % self.T
        qr = np.empty((len(r), self.H, self.D), dtype=np.float64)
        for f in np.unique(frame_of):
            sel = np.nonzero(frame_of == f)[0]
            qr[sel] = self.q_rot(int(f), tok_of[sel])
        frames = np.repeat(np.arange(n, dtype=np.int64), self.T)
        tokens = np.tile(np.arange(self.T, dtype=np.int64), n)
        angles = rope_angles(self.positions(frames, tokens), self.D, self.base)
        out = np.empty_like(qr)
        for h in range(self.H):
            k, v = self.gather_head(n - 1, h, frames, tokens, angles)
            out[:, h, :] = softmax_attention(qr[:, h, :], k, v)
        return out

    def attend(self, t, rows=None):
        """fp64 attention output [len(rows), H, D] of frame t's query rows."""
        qr = self.q_rot(t, rows)
        frames, tokens = self.key_index(t)
        angles = rope_angles(self.positions(frames, tokens), self.D, self.base)
        out = np.empty_like(qr)
        for h in range(self.H):
            k, v = self.gather_head(t, h, frames, tokens, angles)
            out[:, h, :] = softmax_attention(qr[:, h, :], k, v)
        return out


def keyframe_stream(oracle: GcaOracle, frames: int, interval: int, on_frame=None):
    """Streams video frames 0..frames-1 keeping every `interval`-th one (R11). After each
    frame's append, `on_frame(g, slot, keyframe)` runs (the frame's attention happens there);
    a non-keyframe then rolls back. Returns the slots of the keyframes."""
    kept = []
    for g in range(frames):
        slot = oracle.book.frames
        key = g % interval == 0
        oracle.append(slot, g, transient=not key)
        if on_frame is not None:
            on_frame(g, slot, key)
        if key:
            kept.append(slot)
        else:
            oracle.rollback(slot)
    return kept


def windowed_frames(total, window, overlap):
    """(window, video frame, local index) in processing order (R14)."""
    out = []
    start, w = 0, 0
    while True:
        end = min(start + window, total)
        out += [(w, g, g - start) for g in range(start, end)]
        if end >= total:
            return out
        start += window - overlap
        w += 1


def _to_f32(x):
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.to(torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float32)
