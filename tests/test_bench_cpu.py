"""Host-side rules of bench.py that the timing contract rests on (no GPU)."""
import pytest

import bench


@pytest.mark.parametrize("K,R", [(2000, 4), (1000, 8), (3, 1), (7, 4), (2000, 8), (40, 4), (1, 1), (97, 1)])
def test_steps_per_graph_divides_and_cycles(K, R):
    """G divides K (exactly K steps are timed as K / G replays), is a multiple
    of R (each replay cycles every replica equally) or 1, and is at most 32."""
    G = bench.steps_per_graph(K, R)
    assert 1 <= G <= 32 and K % G == 0
    assert G % R == 0 or G == 1
    # no larger admissible G was skipped
    assert not any(K % g == 0 and g % R == 0 for g in range(G + 1, min(K, 32) + 1))


def test_peaks_reads_measured_file():
    hbm, src = bench.peaks()
    assert hbm > 1000 and src in ("measured", "fallback")
