"""Python binding of libgca.so, the B200 paged KV cache for Geometric Context Attention.

The functions below carry the C ABI's names (include/gca.h) and only marshal arguments;
every step of the path runs in the library's CUDA kernels. PyTorch supplies device memory and
streams. There is no fallback: if the library is missing or fails to load, the first call
raises.

`GcaCache` is a convenience owner of one cache: it allocates the workspace with torch, keeps
the handle and exposes read-only tensor views of the device state for inspection.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "GcaError", "GcaConfig", "GcaState", "GcaAttendInfo", "lib", "library_path",
    "gca_validate_config", "gca_workspace_bytes", "gca_cache_create", "gca_append_frame",
    "gca_attend", "gca_reset", "gca_cache_destroy", "gca_check", "gca_get_state",
    "gca_last_attend_info", "gca_status_string", "gca_attend_noalloc", "gca_append_frames",
    "gca_append_frame_ex", "gca_rollback_last_frame", "gca_attend_prefill",
    "GCA_APPEND_TRANSIENT", "GcaCache", "config_for", "EXPORTED_SYMBOLS",
    "gca_set_wait_limit", "gca_test_withhold_copies", "gca_read_attend_counters",
    "GcaAttendCounters", "gca_set_split_event",
]

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    """The in-tree libgca.so built by paged_kv_cache_gca_b200.build, or the file GCA_LIBRARY
    names (another build of this library, e.g. one compiled with different kernel settings)."""
    return os.environ.get("GCA_LIBRARY", os.path.join(_HERE, "libgca.so"))


GCA_OK = 0
GCA_APPEND_TRANSIENT = 1
STATUS = {0: "GCA_OK", -1: "GCA_ERR_INVALID_ARG", -2: "GCA_ERR_OUT_OF_PAGES",
          -3: "GCA_ERR_FRAME_ORDER", -4: "GCA_ERR_CUDA", -5: "GCA_ERR_UNSUPPORTED",
          -6: "GCA_ERR_DEVICE"}


class GcaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class GcaConfig(ctypes.Structure):
    _fields_ = [
        ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
        ("num_special", ctypes.c_int32), ("anchor_frames", ctypes.c_int32),
        ("window_frames", ctypes.c_int32), ("keep_tokens", ctypes.c_int32),
        ("max_frames", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("rope_base", ctypes.c_float),
    ]


class GcaState(ctypes.Structure):
    _fields_ = [
        ("frames_appended", ctypes.c_int64), ("free_head", ctypes.c_int64),
        ("free_tail", ctypes.c_int64), ("traj_len", ctypes.c_int64),
        ("traj_pages", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
        ("pages_per_frame", ctypes.c_int32), ("pages_in_use", ctypes.c_int32),
        ("device_error", ctypes.c_uint32), ("transient", ctypes.c_int32),
        ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
        ("free_ring", ctypes.c_void_p), ("frame_pages", ctypes.c_void_p),
        ("traj_page_list", ctypes.c_void_p), ("slot_map", ctypes.c_void_p),
        ("kept_tokens", ctypes.c_void_p),
    ]


class GcaAttendInfo(ctypes.Structure):
    _fields_ = [
        ("frame_idx", ctypes.c_int64), ("visible_keys", ctypes.c_int64),
        ("logical_pages", ctypes.c_int32), ("kv_tiles", ctypes.c_int32),
        ("query_tiles", ctypes.c_int32), ("grid", ctypes.c_int32), ("split", ctypes.c_int32),
        ("launches", ctypes.c_int32),
    ]


class GcaAttendCounters(ctypes.Structure):
    _fields_ = [
        ("exact_max_rows", ctypes.c_uint64), ("rescaled_rows", ctypes.c_uint64),
        ("wide_merge_rows", ctypes.c_uint64), ("reserved", ctypes.c_uint64),
    ]


# Every symbol include/gca.h declares.
EXPORTED_SYMBOLS = (
    "gca_validate_config", "gca_workspace_bytes", "gca_cache_create", "gca_append_frame",
    "gca_attend", "gca_reset", "gca_cache_destroy", "gca_check", "gca_get_state",
    "gca_last_attend_info", "gca_status_string", "gca_attend_noalloc", "gca_append_frames",
    "gca_append_frame_ex", "gca_rollback_last_frame", "gca_attend_prefill",
    "gca_set_wait_limit", "gca_test_withhold_copies", "gca_read_attend_counters",
    "gca_set_split_event",
)

_lib = None


def lib():
    """Loads libgca.so once. Raises if it is missing: there is no fallback path."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"libgca.so not built ({path}); run "
                          "`python -m paged_kv_cache_gca_b200.build`")
    L = ctypes.CDLL(path)
    P, I32, I64, SZ, VP = (ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                           ctypes.c_void_p)
    sig = {
        "gca_validate_config": (I32, [P(GcaConfig)]),
        "gca_workspace_bytes": (SZ, [P(GcaConfig)]),
        "gca_cache_create": (I32, [P(GcaConfig), VP, SZ, VP, VP, P(VP)]),
        "gca_append_frame": (I32, [VP, I64, VP, VP, VP, VP, VP]),
        "gca_attend": (I32, [VP, I64, VP, VP, VP]),
        "gca_reset": (I32, [VP, VP]),
        "gca_cache_destroy": (I32, [VP]),
        "gca_check": (I32, [VP]),
        "gca_get_state": (I32, [VP, P(GcaState)]),
        "gca_last_attend_info": (I32, [VP, P(GcaAttendInfo)]),
        "gca_status_string": (ctypes.c_char_p, [I32]),
        "gca_attend_noalloc": (I32, [VP, I64, VP, VP, VP]),
        "gca_append_frames": (I32, [P(VP), I32, P(I64), P(VP), P(VP), P(VP), P(VP), VP]),
        "gca_append_frame_ex": (I32, [VP, I64, I64, ctypes.c_uint32, VP, VP, VP, VP, VP]),
        "gca_rollback_last_frame": (I32, [VP, I64, VP]),
        "gca_attend_prefill": (I32, [VP, I32, VP, VP, VP]),
        "gca_set_wait_limit": (I32, [VP, ctypes.c_uint64]),
        "gca_test_withhold_copies": (I32, [VP]),
        "gca_read_attend_counters": (I32, [VP, P(GcaAttendCounters)]),
        "gca_set_split_event": (I32, [VP, VP]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _ok(status: int, where: str) -> None:
    if status != GCA_OK:
        raise GcaError(status, where)


def gca_status_string(status: int) -> str:
    return lib().gca_status_string(status).decode()


def gca_validate_config(cfg: GcaConfig) -> int:
    return lib().gca_validate_config(ctypes.byref(cfg))


def gca_workspace_bytes(cfg: GcaConfig) -> int:
    return lib().gca_workspace_bytes(ctypes.byref(cfg))


def gca_cache_create(cfg: GcaConfig, workspace_ptr: int, workspace_bytes: int,
                     initial_free_ptr: int | None, stream: int | None) -> int:
    h = ctypes.c_void_p()
    _ok(lib().gca_cache_create(ctypes.byref(cfg), workspace_ptr, workspace_bytes,
                               initial_free_ptr, stream, ctypes.byref(h)), "gca_cache_create")
    return h.value


def gca_append_frame(handle, frame_idx, q_ptr, k_ptr, v_ptr, q_rot_ptr, stream) -> None:
    _ok(lib().gca_append_frame(handle, frame_idx, q_ptr, k_ptr, v_ptr, q_rot_ptr, stream),
        "gca_append_frame")


def gca_append_frame_ex(handle, frame_idx, rope_frame, flags, q_ptr, k_ptr, v_ptr, q_rot_ptr,
                        stream) -> None:
    _ok(lib().gca_append_frame_ex(handle, frame_idx, rope_frame, flags, q_ptr, k_ptr, v_ptr,
                                  q_rot_ptr, stream), "gca_append_frame_ex")


def gca_rollback_last_frame(handle, frame_idx, stream=None) -> None:
    _ok(lib().gca_rollback_last_frame(handle, frame_idx, stream), "gca_rollback_last_frame")


def gca_attend_prefill(handle, n, q_rot_ptr, out_ptr, stream) -> None:
    _ok(lib().gca_attend_prefill(handle, n, q_rot_ptr, out_ptr, stream), "gca_attend_prefill")


def gca_attend(handle, frame_idx, q_rot_ptr, out_ptr, stream) -> None:
    _ok(lib().gca_attend(handle, frame_idx, q_rot_ptr, out_ptr, stream), "gca_attend")


def gca_attend_noalloc(handle, frame_idx, q_rot_ptr, out_ptr, stream) -> None:
    """gca_attend with its scratch in the library's fixed device array (no allocation)."""
    _ok(lib().gca_attend_noalloc(handle, frame_idx, q_rot_ptr, out_ptr, stream),
        "gca_attend_noalloc")


def gca_append_frames(handles, frame_idx, q_ptrs, k_ptrs, v_ptrs, q_rot_ptrs, stream) -> None:
    """One launch appending frame_idx[i] to cache handles[i] (sequences of equal length)."""
    n = len(handles)
    arr = lambda t, xs: (t * n)(*xs)
    VP, I64 = ctypes.c_void_p, ctypes.c_int64
    _ok(lib().gca_append_frames(arr(VP, handles), n, arr(I64, frame_idx), arr(VP, q_ptrs),
                                arr(VP, k_ptrs), arr(VP, v_ptrs), arr(VP, q_rot_ptrs), stream),
        "gca_append_frames")


def gca_set_wait_limit(handle, wait_ns: int) -> None:
    _ok(lib().gca_set_wait_limit(handle, wait_ns), "gca_set_wait_limit")


def gca_test_withhold_copies(handle) -> None:
    """Test hook: the next attention launch's CTA 0 never issues its first tile's copies."""
    _ok(lib().gca_test_withhold_copies(handle), "gca_test_withhold_copies")


def gca_read_attend_counters(handle) -> GcaAttendCounters:
    out = GcaAttendCounters()
    _ok(lib().gca_read_attend_counters(handle, ctypes.byref(out)), "gca_read_attend_counters")
    return out


def gca_set_split_event(handle, cuda_event) -> None:
    """cuda_event: a cudaEvent_t handle (int, e.g. torch.cuda.Event().cuda_event) or None."""
    _ok(lib().gca_set_split_event(handle, cuda_event), "gca_set_split_event")


def gca_reset(handle, stream) -> None:
    _ok(lib().gca_reset(handle, stream), "gca_reset")


def gca_cache_destroy(handle) -> None:
    _ok(lib().gca_cache_destroy(handle), "gca_cache_destroy")


def gca_check(handle) -> int:
    return lib().gca_check(handle)


def gca_get_state(handle) -> GcaState:
    st = GcaState()
    _ok(lib().gca_get_state(handle, ctypes.byref(st)), "gca_get_state")
    return st


def gca_last_attend_info(handle) -> GcaAttendInfo:
    inf = GcaAttendInfo()
    _ok(lib().gca_last_attend_info(handle, ctypes.byref(inf)), "gca_last_attend_info")
    return inf


def config_for(w, rope_base: float | None = None) -> GcaConfig:
    """C config of a workload description (gca_inputs.Workload or anything with its fields)."""
    return GcaConfig(num_heads=w.num_heads, head_dim=w.head_dim, page_size=w.page_size,
                     grid_h=w.grid_h, grid_w=w.grid_w, num_special=w.num_special,
                     anchor_frames=w.anchor_frames, window_frames=w.window_frames,
                     keep_tokens=w.keep_tokens, max_frames=w.max_frames,
                     num_pages=w.num_pages,
                     rope_base=w.rope_base if rope_base is None else rope_base)


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


class GcaCache:
    """One GCA cache on the current CUDA device, its workspace allocated by torch."""

    def __init__(self, cfg: GcaConfig, initial_free=None, stream=None, device=None):
        import torch

        self.cfg = cfg
        st = gca_validate_config(cfg)
        _ok(st, "gca_validate_config")
        self.nbytes = gca_workspace_bytes(cfg)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.workspace = torch.empty(self.nbytes + 1024, dtype=torch.uint8, device=dev)
        base = self.workspace.data_ptr()
        self._off = (-base) % 1024
        self._free = None
        if initial_free is not None:
            self._free = torch.as_tensor(initial_free, dtype=torch.int32).to(dev).contiguous()
        self.handle = gca_cache_create(
            cfg, base + self._off, self.nbytes,
            None if self._free is None else self._free.data_ptr(), _stream_handle(stream))

    def close(self):
        if getattr(self, "handle", None):
            gca_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ hot path
    def append_frame(self, t, q, k, v, q_rot, stream=None, rope_frame=None, transient=False):
        """Appends cache frame t; rope_frame (default t) is its RoPE time position; transient:
        a non-keyframe that is rolled back after its attention."""
        if rope_frame is None and not transient:
            gca_append_frame(self.handle, t, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                             q_rot.data_ptr(), _stream_handle(stream))
        else:
            gca_append_frame_ex(self.handle, t, t if rope_frame is None else rope_frame,
                                GCA_APPEND_TRANSIENT if transient else 0, q.data_ptr(),
                                k.data_ptr(), v.data_ptr(), q_rot.data_ptr(),
                                _stream_handle(stream))

    def rollback(self, t):
        gca_rollback_last_frame(self.handle, t)

    def attend(self, t, q_rot, out, stream=None):
        gca_attend(self.handle, t, q_rot.data_ptr(), out.data_ptr(), _stream_handle(stream))

    def attend_prefill(self, n, q_rot, out, stream=None):
        """Joint bidirectional attention of the first n frames (q_rot, out: [n*T, H, D])."""
        gca_attend_prefill(self.handle, n, q_rot.data_ptr(), out.data_ptr(),
                           _stream_handle(stream))

    def reset(self, stream=None):
        gca_reset(self.handle, _stream_handle(stream))

    # ------------------------------------------------------------------ inspection
    def check(self) -> int:
        return gca_check(self.handle)

    def state(self) -> GcaState:
        return gca_get_state(self.handle)

    def attend_info(self) -> GcaAttendInfo:
        return gca_last_attend_info(self.handle)

    def counters(self) -> GcaAttendCounters:
        """Attention branch counters since create / reset (synchronises)."""
        return gca_read_attend_counters(self.handle)

    def _view(self, ptr, count, dtype):
        import torch

        start = ptr - self.workspace.data_ptr()
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        return self.workspace[start:start + nbytes].view(dtype)

    def views(self):
        """Device tensors over the cache state (no copies)."""
        import torch

        c, s = self.cfg, self.state()
        ppf = s.pages_per_frame
        page_shape = (c.num_pages, c.num_heads, c.page_size, c.head_dim)
        n_page = c.num_pages * c.num_heads * c.page_size * c.head_dim
        return {
            "k_pool": self._view(s.k_pool, n_page, torch.bfloat16).view(page_shape),
            "v_pool": self._view(s.v_pool, n_page, torch.bfloat16).view(page_shape),
            "free_ring": self._view(s.free_ring, c.num_pages, torch.int32),
            "frame_pages": self._view(s.frame_pages, c.max_frames * ppf,
                                      torch.int32).view(c.max_frames, ppf),
            "traj_pages": self._view(s.traj_page_list, max(s.traj_pages, 0), torch.int32),
            "slot_map": self._view(s.slot_map, s.tokens_per_frame, torch.int32),
            "kept_tokens": self._view(s.kept_tokens, c.keep_tokens, torch.int32),
        }

    def free_list(self):
        """Free page ids in FIFO order (host list; synchronises)."""
        s = self.state()
        ring = self.views()["free_ring"].cpu().tolist()
        n = self.cfg.num_pages
        return [ring[i % n] for i in range(s.free_head, s.free_tail)]
