"""The causal launch order (the `band_unit` mapping of the forward and
gradient kernels' 1-D grids), evaluated by the library's own code on the host
(attn_schedule_band_unit) and checked against a Python statement of it:
every (pair, tile) unit is launched exactly once, bands never exceed their
size, and inside a band the costliest tile rank of every pair comes before
the next rank.  A greedy
list-scheduling model of 148 SMs then shows why the order matters for causal
row tiles (tile t costs about t + 1 key tiles): the head-major order reaches
about 86% of the ideal makespan, the banded costliest-first order 95-100%."""
import heapq

import pytest

from io_aware_exact_29_b200 import attn


def _band_unit(u, band, n_pairs, n_tiles):
    per_band = band * n_tiles
    bi = u // per_band
    r = u - bi * per_band
    hb = min(band, n_pairs - bi * band)
    rank = r // hb
    return bi * band + (r - rank * hb), rank


@pytest.mark.parametrize("n_pairs", [1, 5, 16, 64, 100])
@pytest.mark.parametrize("n_tiles", [1, 3, 16])
@pytest.mark.parametrize("band", [1, 8, 24, 96])
def test_every_unit_once_in_band_order(n_pairs, n_tiles, band):
    band = min(band, n_pairs)
    units = [attn.schedule_band_unit(u, band, n_pairs, n_tiles) for u in range(n_pairs * n_tiles)]
    # the library's mapping is the one stated in Python here
    assert units == [_band_unit(u, band, n_pairs, n_tiles) for u in range(n_pairs * n_tiles)]
    assert sorted(units) == [(p, t) for p in range(n_pairs) for t in range(n_tiles)]
    # within a band, ranks are non-decreasing in launch order
    for u in range(1, len(units)):
        same_band = units[u][0] // band == units[u - 1][0] // band
        if same_band:
            assert units[u][1] >= units[u - 1][1]


def _makespan(costs, n_sm=148, overhead=1.0):
    free = [0.0] * n_sm
    heapq.heapify(free)
    for c in costs:
        heapq.heappush(free, heapq.heappop(free) + c + overhead)
    return max(free)


@pytest.mark.parametrize("N", [4096, 16384])
def test_costliest_first_balances_causal_tiles(N):
    B, H, nt = 16384 // N, 16, N // 256
    cost = lambda ct: 2 * ct + 2  # key-tile periods of a causal 256-row CTA
    ideal = sum(cost(ct) + 1.0 for ct in range(nt)) * B * H / 148
    head_major = [cost(nt - 1 - x) for _ in range(B * H) for x in range(nt)]
    band = 8
    banded = [cost(nt - 1 - attn.schedule_band_unit(u, band, B * H, nt)[1])
              for u in range(B * H * nt)]
    eff_head = ideal / _makespan(head_major)
    eff_band = ideal / _makespan(banded)
    assert eff_head < 0.9 and eff_band > 0.95


def test_band_unit_rejects_bad_arguments():
    for args in ((0, 0, 4, 4), (0, 5, 4, 4), (16, 4, 4, 4), (0, 1, 0, 1)):
        with pytest.raises(attn.AttnError):
            attn.schedule_band_unit(*args)
