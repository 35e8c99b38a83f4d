"""Host-side tiling of the neighborhood kernel (dit_na3d_plan, no GPU): the step count and
the choice of Q brick are checked against a brute force written from the definitions: a
query's window along an axis is the K positions starting at clamp(i - K/2, 0, L - K); a Q
brick visits the 4 x 4 x 8 (t, y, x) KV bricks laid from the first position of the union of
its rows' windows; a unit is two Q bricks side by side along one axis and takes as many
steps as the longer of their two lists; the choice minimises steps + 2 * units per head."""

import itertools

import pytest

KV_BRICK = (4, 4, 8)


def _window(i, K, L):
    s = min(max(i - K // 2, 0), L - K)
    return range(s, s + K)


def _bricks_along(a, ext, K, L, b):
    """KV bricks of extent b along one axis for the queries [a, a + ext) (0 if none)."""
    rows = [i for i in range(a, a + ext) if i < L]
    if not rows:
        return 0
    covered = set()
    for i in rows:
        covered.update(_window(i, K, L))
    lo, hi = min(covered), max(covered)
    assert covered == set(range(lo, hi + 1))            # windows of neighbours overlap
    return -(-(hi - lo + 1) // b)


def _brute(grid, window, qb, pax):
    ext = [qb[d] * (2 if d == pax else 1) for d in range(3)]
    nu = [-(-grid[d] // ext[d]) for d in range(3)]
    steps = 0
    for o in itertools.product(*[range(0, nu[d] * ext[d], ext[d]) for d in range(3)]):
        n = []
        for t in range(2):
            oo = list(o)
            oo[pax] += t * qb[pax]
            c = 1
            for d in range(3):
                c *= _bricks_along(oo[d], qb[d], window[d], grid[d], KV_BRICK[d])
            n.append(c)
        steps += max(n)
    return steps, nu[0] * nu[1] * nu[2]


CASES = [((21, 30, 52), (7, 7, 7)), ((21, 30, 52), (7, 15, 15)), ((1, 12, 16), (1, 5, 5)), ((5, 6, 9), (5, 5, 9)),
         ((8, 4, 16), (7, 3, 15)), ((3, 10, 20), (3, 5, 7)), ((4, 8, 8), (1, 1, 1))]


@pytest.mark.parametrize("grid,window", CASES)
def test_plan_matches_brute_force(cuda_lib_host, grid, window):
    plan = cuda_lib_host.dit_na3d_plan(*grid, *window)
    qb, pax = plan["q_brick"], plan["pair_axis"]
    assert qb[0] * qb[1] * qb[2] == 128 and 0 <= pax <= 2
    steps, units = _brute(grid, window, qb, pax)
    assert plan["steps_per_head"] == steps
    assert plan["units_per_head"] == units
    best = min(s + 2 * u for s, u in (
        _brute(grid, window, (1 << a, 1 << b, 1 << (7 - a - b)), p)
        for a in range(8) for b in range(8 - a) for p in range(3)))
    assert steps + 2 * units == best


@pytest.mark.parametrize("grid,window", [((3, 4, 5), (2, 3, 3)), ((3, 4, 5), (5, 3, 3)), ((0, 4, 5), (1, 1, 1)),
                                         ((3, 4, 5), (1, 0, 1))])
def test_plan_rejects_bad_windows(cuda_lib_host, grid, window):
    with pytest.raises(cuda_lib_host.DitError) as e:
        cuda_lib_host.dit_na3d_plan(*grid, *window)
    assert e.value.status == cuda_lib_host.DIT_ERR_INVALID_ARG
