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
