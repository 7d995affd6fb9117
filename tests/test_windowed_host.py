"""Host scheduling of the windowed mode (paged_kv_cache_gca_b200.windowed) against the oracle's
own statement of the schedule (reading R14). CPU only."""
import pytest

import oracle as orc
from paged_kv_cache_gca_b200 import windowed


@pytest.mark.parametrize("total,N,V", [(1000, 128, 8), (320, 128, 8), (128, 128, 8), (129, 128, 8),
                                       (17, 4, 1), (9, 9, 0), (1, 3, 2), (0, 3, 1), (40, 6, 5)])
def test_schedule_matches_the_oracle(total, N, V):
    assert list(windowed.windowed_schedule(total, N, V)) == orc.windowed_frames(total, N, V) \
        if total > 0 else list(windowed.windowed_schedule(total, N, V)) == []


def test_schedule_rejects_bad_overlap():
    for N, V in ((4, 4), (4, -1), (0, 0)):
        with pytest.raises(ValueError):
            windowed.window_starts(10, N, V)


class _RecordingCache:
    """Stands in for GcaCache: records the calls the driver makes."""

    def __init__(self):
        self.calls = []

    def reset(self, stream=None):
        self.calls.append(("reset",))

    def append_frame(self, t, q, k, v, q_rot, stream=None):
        self.calls.append(("append", t, q))

    def attend(self, t, q_rot, out, stream=None):
        self.calls.append(("attend", t))


def test_driver_resets_at_every_window_start_and_uses_local_indices():
    N, V, total = 5, 2, 12
    cache = _RecordingCache()
    drv = windowed.WindowedStream(cache, N, V)
    for w, g, loc in windowed.windowed_schedule(total, N, V):
        drv.step(loc, g, None, None, None, None)  # q stands for the video frame here
    calls = cache.calls
    starts = windowed.window_starts(total, N, V)
    assert [c for c in calls if c[0] == "reset"] == [("reset",)] * len(starts)
    # every append is followed by the attend of the same local frame
    for i, c in enumerate(calls):
        if c[0] == "append":
            assert calls[i + 1] == ("attend", c[1])
    # after each reset the local indices restart at 0 and the video frames follow the windows
    seq, cur = [], None
    for c in calls:
        if c[0] == "reset":
            cur = []
            seq.append(cur)
        elif c[0] == "append":
            cur.append((c[1], c[2]))
    for s0, win in zip(starts, seq):
        assert [loc for loc, _ in win] == list(range(len(win)))
        assert [g for _, g in win] == list(range(s0, min(s0 + N, total)))
