"""Host-side planning of mxattn_forward_host (CPU only): the default group
schedule covers every (batch, head) slice exactly once, in order, starts and
ends with a one-slice group when there are at least three groups, and keeps
the middle groups within one slice of each other; the library's workspace size
for the call is the workspace of its largest group."""
import ctypes

import pytest

from mxfp4_microscaled_quantization_b200 import mxattn as mx
from mxfp4_microscaled_quantization_b200.mxattn import host_groups


@pytest.mark.parametrize("BH", [0, 1, 2, 3, 5, 16, 40, 41, 97, 960])
@pytest.mark.parametrize("chunks", [1, 2, 3, 4, 16, 40, 1000])
def test_default_group_schedule(BH, chunks):
    g = host_groups(BH, chunks)
    assert sum(g) == BH and all(x >= 1 for x in g)
    if BH == 0:
        assert g == []
    elif BH >= 3 and chunks >= 3:
        assert len(g) == min(chunks, BH)
        assert g[0] == 1 and g[-1] == 1
        mid = g[1:-1]
        assert max(mid) - min(mid) <= 1
    else:  # one or two groups: equal sizes, the last possibly smaller
        assert len(g) <= max(1, min(chunks, BH))
        assert all(x == g[0] for x in g[:-1]) and g[-1] <= g[0]


@pytest.mark.parametrize("BH", [1, 2, 3, 5, 16, 40, 41, 97, 960])
@pytest.mark.parametrize("chunks", [0, 1, 2, 3, 4, 16, 40, 1000])
def test_library_schedule_matches_host_groups(BH, chunks):
    """The library sizes its workspace for its largest group, which must be the
    largest group of the schedule restated in Python (chunks 0 means 16)."""
    N, d = 300, 128
    want = mx.mxattn_workspace_size(1, max(host_groups(BH, chunks or 16)), N, d)
    assert mx.forward_host_workspace_size(1, BH, N, d, chunks) == want


def test_host_workspace_size_with_explicit_groups():
    assert mx.forward_host_workspace_size(2, 5, 300, 64, groups=[4, 1, 5]) == mx.mxattn_workspace_size(1, 5, 300, 64)
    assert mx.forward_host_workspace_size(2, 5, 300, 64, groups=[4, 1, 4]) == 0   # does not sum to B*H
    assert mx.forward_host_workspace_size(2, 5, 300, 64, groups=[10, 0]) == 0    # empty group
    assert mx.lib().mxattn_forward_host_workspace_size(1, 3, 300, 64, None, -1) == 0  # negative group count
