"""Host-side planning of attention_from_host (CPU only): the default group
schedule covers every (batch, head) slice exactly once, in order, starts and
ends with a one-slice group when there are at least three groups, and keeps
the middle groups within one slice of each other."""
import pytest

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
