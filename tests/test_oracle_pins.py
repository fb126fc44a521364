"""Pins for the CPU oracle: closed forms, brute force, library routines and invariants.

Each test checks the oracle against something other than itself, chosen so that a
plausible slip (a dropped term, a wrong index, a transposed operand, a wrong divisor) fails.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import bsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


GRIDS = [(4, 8, 8), (6, 10, 9), (5, 7, 3), (8, 16, 16), (1, 1, 1), (9, 4, 5)]


# ------------------------------------------------------------------------------ reorder
@pytest.mark.parametrize("grid", GRIDS)
def test_reorder_forward_formula(grid):
    """Every token lands at the tile/slot given by the forward formula; padding is zero."""
    T, Hs, Ws = grid
    B, H, d = 2, 3, 5
    x = _rand((B, T * Hs * Ws, H, d), 1) + 10.0
    xt = O.reorder(x, T, Hs, Ws)
    nT, nY, nX = -(-T // 4), -(-Hs // 4), -(-Ws // 4)
    assert xt.shape == (B, H, nT * nY * nX, 64, d)
    seen = np.zeros(xt.shape[2:4], dtype=bool)
    for t in range(T):
        for y in range(Hs):
            for xx in range(Ws):
                n = (t * Hs + y) * Ws + xx
                j = ((t // 4) * nY + y // 4) * nX + xx // 4
                r = ((t % 4) * 4 + y % 4) * 4 + xx % 4
                assert np.array_equal(xt[:, :, j, r, :], x[:, n, :, :])
                seen[j, r] = True
    assert np.all(xt[:, :, ~seen, :] == 0.0)
    assert seen.sum() == T * Hs * Ws


@pytest.mark.parametrize("grid", GRIDS)
def test_reorder_round_trip_bitwise(grid):
    T, Hs, Ws = grid
    x = torch.randn(1, T * Hs * Ws, 2, 8, generator=torch.Generator().manual_seed(3))
    xb = x.to(torch.bfloat16).view(torch.int16).numpy()
    back = O.unreorder(O.reorder(xb, T, Hs, Ws), T, Hs, Ws)
    assert back.dtype == xb.dtype and np.array_equal(back, xb)


# ------------------------------------------------------------------------------ pooling
@pytest.mark.parametrize("grid", [(6, 10, 9), (8, 16, 16), (5, 7, 3)])
def test_pool_matches_raster_block_mean(grid):
    """Mean over the raster block of each tile, computed by slicing the raster grid."""
    T, Hs, Ws = grid
    B, H, d = 1, 2, 4
    x = _rand((B, T * Hs * Ws, H, d), 5)
    xb = O.pool(O.reorder(x, T, Hs, Ws), T, Hs, Ws)
    g = x.reshape(B, T, Hs, Ws, H, d)
    nT, nY, nX = O.tile_grid(T, Hs, Ws)
    for tt in range(nT):
        for ty in range(nY):
            for tx in range(nX):
                blk = g[:, 4 * tt:4 * tt + 4, 4 * ty:4 * ty + 4, 4 * tx:4 * tx + 4]
                ref = blk.reshape(B, -1, H, d).mean(axis=1)             # [B, H, d]
                j = (tt * nY + ty) * nX + tx
                np.testing.assert_allclose(xb[:, :, j, :], ref, rtol=1e-13, atol=1e-13)


def test_pool_constant_tiles_exact():
    T, Hs, Ws = 6, 10, 9                       # ragged: partial tiles everywhere at edges
    NT = np.prod(O.tile_grid(T, Hs, Ws))
    vals = np.arange(NT, dtype=np.float64) * 0.375 - 3.0
    src = O.slot_tokens(T, Hs, Ws)
    x = np.zeros((1, T * Hs * Ws, 1, 3))
    for j in range(NT):
        for r in range(64):
            if src[j, r] >= 0:
                x[0, src[j, r], 0, :] = vals[j]
    xb = O.pool(O.reorder(x, T, Hs, Ws), T, Hs, Ws)
    assert np.array_equal(xb[0, 0, :, 0], vals)


# ------------------------------------------------------------------------------ windows
def _golden_windows():
    rows = []
    with open(os.path.join(GOLDEN, "window_sizes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kind, r, size = line.split()
            rows.append((0 if kind == "cube" else 1, int(r), int(size)))
    return rows


@pytest.mark.parametrize("kind,r,size", _golden_windows())
def test_window_interior_size(kind, r, size):
    T = Hs = Ws = 4 * (2 * r + 3)              # big enough that the centre tile is interior
    nT, nY, nX = O.tile_grid(T, Hs, Ws)
    c = ((nT // 2) * nY + nY // 2) * nX + nX // 2
    assert int(O.window_row(kind, r, c, T, Hs, Ws).sum()) == size
    assert int(O.window(kind, r, T, Hs, Ws)[c].sum()) == size


@pytest.mark.parametrize("kind", [0, 1])
@pytest.mark.parametrize("r", [0, 1, 2, 3])
@pytest.mark.parametrize("grid", [(8, 16, 16), (6, 10, 9), (21, 30, 52)])
def test_window_brute_force_and_clipped_counts(kind, r, grid):
    """Brute-force loops (small grids) and per-axis clipped counts (all grids)."""
    T, Hs, Ws = grid
    nT, nY, nX = O.tile_grid(T, Hs, Ws)
    W = O.window(kind, r, T, Hs, Ws)

    def clip_count(c, s, n):
        return max(0, min(c + s, n - 1) - max(c - s, 0) + 1) if s >= 0 else 0

    for i in range(W.shape[0]):
        tt, rem = divmod(i, nY * nX)
        ty, tx = divmod(rem, nX)
        if kind == 0:
            expect = clip_count(tt, r, nT) * clip_count(ty, r, nY) * clip_count(tx, r, nX)
        else:
            expect = sum(clip_count(ty, r - abs(dt), nY) * clip_count(tx, r - abs(dt), nX)
                         for dt in range(-r, r + 1) if 0 <= tt + dt < nT)
        assert int(W[i].sum()) == expect
    if W.shape[0] <= 64:
        for i in range(W.shape[0]):
            ti, rem = divmod(i, nY * nX)
            yi, xi = divmod(rem, nX)
            for j in range(W.shape[1]):
                tj, rem = divmod(j, nY * nX)
                yj, xj = divmod(rem, nX)
                dt, dy, dx = abs(ti - tj), abs(yi - yj), abs(xi - xj)
                inside = max(dt, dy, dx) <= r if kind == 0 else (dt <= r and max(dy, dx) <= r - dt)
                assert W[i, j] == inside


# ------------------------------------------------------------------------------ routing
@pytest.mark.parametrize("rho", [0.0, 0.1, 0.2, 0.25, 0.5, 1.0])
def test_route_count_and_order(rho):
    rng = np.random.default_rng(7)
    d = rng.random((3, 37)).astype(np.float32)
    d[1, 5] = d[1, 9] = d[1, 30] = 0.999     # planted ties: lower index wins
    dense = O.route_dense(d, rho)
    nd = int(math.floor(float(np.float32(rho)) * 37 + 0.5))
    assert np.all(dense.sum(axis=1) == nd)
    for b in range(3):
        order = sorted(range(37), key=lambda i: (-float(d[b, i]), i))
        assert set(np.nonzero(dense[b])[0]) == set(order[:nd])
    if rho == 0.0:
        assert not dense.any()
    if rho == 1.0:
        assert dense.all()


# ------------------------------------------------------------------------------ selection
def _planted(T, Hs, Ws, H, d, kvals, qvec):
    """Tiled Q/K whose every valid slot of tile j holds qvec (Q) and kvals[j] (K)."""
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    valid = O.slot_valid(T, Hs, Ws)
    qt = np.zeros((1, H, NT, 64, d))
    kt = np.zeros((1, H, NT, 64, d))
    for j in range(NT):
        qt[0, :, j, valid[j]] = qvec
        kt[0, :, j, valid[j]] = kvals[j]
    return qt, kt


@pytest.mark.parametrize("kind", [0, 1])
def test_topk_planted_increasing_scores(kind):
    """kbar_j = c*j*e1, qbar = e1: the extra tiles are the highest-indexed outside the window."""
    T, Hs, Ws, d, k = 8, 16, 16, 8, 3
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    qt, kt = _planted(T, Hs, Ws, 2, d, [0.25 * (j + 1) * e1 for j in range(NT)], e1)
    diff = np.zeros((1, NT), np.float32)
    res = O.build_mask(qt, kt, diff, T=T, Hs=Hs, Ws=Ws, window_kind=kind, radius=1, topk=k,
                       dense_fraction=0.0)
    W = O.window(kind, 1, T, Hs, Ws)
    for i in range(NT):
        outside = [j for j in range(NT) if not W[i, j]]
        expect = set(np.nonzero(W[i])[0]) | set(outside[-k:])
        assert set(np.nonzero(res["mask"][0, 0, i])[0]) == expect
        assert res["count"][0, 0, i] == W[i].sum() + min(k, len(outside))


def test_topk_ties_go_to_lower_index():
    T, Hs, Ws, d, k = 8, 16, 16, 4, 2
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    qt, kt = _planted(T, Hs, Ws, 1, d, [e1 for _ in range(NT)], e1)   # all scores equal
    res = O.build_mask(qt, kt, np.zeros((1, NT), np.float32), T=T, Hs=Hs, Ws=Ws,
                       window_kind=0, radius=0, topk=k, dense_fraction=0.0)
    for i in range(NT):
        outside = [j for j in range(NT) if j != i]
        assert set(np.nonzero(res["mask"][0, 0, i])[0]) == {i, *outside[:k]}
        assert res["near_tie"][0, 0, i]                   # equal scores are flagged


def test_dense_rows_and_mask_invariants():
    from bsa_synth import WORKLOADS, generate_qkv, generate_difficulty
    w = WORKLOADS["tiny_ragged"]
    q, k, v = generate_qkv(w)
    diff = generate_difficulty(w).numpy()
    qt, kt = O.reorder(O.to_f64(q), w.T, w.Hs, w.Ws), O.reorder(O.to_f64(k), w.T, w.Hs, w.Ws)
    res = O.build_mask(qt, kt, diff, T=w.T, Hs=w.Hs, Ws=w.Ws, window_kind=0, radius=1,
                       topk=2, dense_fraction=0.25)
    NT = w.NT
    W = O.window(0, 1, w.T, w.Hs, w.Ws)
    assert res["dense"].sum() == O.n_dense(0.25, NT)
    for i in range(NT):
        for h in range(w.H):
            row = res["mask"][0, h, i]
            if res["dense"][0, i]:
                assert row.all()
            else:
                assert np.all(row[W[i]])
                assert row.sum() == W[i].sum() + min(2, NT - W[i].sum())
    # dense routing is shared by every head
    assert np.all(res["mask"][0, 0][res["dense"][0]] == res["mask"][0, 1][res["dense"][0]])


def test_pooled_scores_against_direct_sum():
    qbar = _rand((1, 2, 5, 16), 11)
    kbar = _rand((1, 2, 7, 16), 12)
    S = O.pooled_scores(qbar, kbar)
    for h in range(2):
        for i in range(5):
            for j in range(7):
                ref = sum(qbar[0, h, i, c] * kbar[0, h, j, c] for c in range(16)) / 4.0
                assert abs(S[0, h, i, j] - ref) < 1e-12


# ------------------------------------------------------------------------------ entropy budget
def test_entropy_matches_scipy():
    from scipy.special import softmax
    from scipy.stats import entropy
    s = _rand((3, 50), 13) * 3
    ref = np.array([entropy(softmax(row)) for row in s])
    np.testing.assert_allclose(O.row_entropy(s), ref, rtol=1e-12)


def test_entropy_budget_uniform_scores():
    """Identical kbar: every row's entropy is ln NKT and every budget is round(tau*NKT)."""
    T, Hs, Ws, d = 8, 16, 16, 4
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    qt, kt = _planted(T, Hs, Ws, 1, d, [e1] * NT, 0.3 * e1)
    for tau in (0.09, 0.14, 0.19, 0.5):
        res = O.build_mask(qt, kt, np.zeros((1, NT), np.float32), T=T, Hs=Hs, Ws=Ws,
                           window_kind=1, radius=0, topk=0, dense_fraction=0.0,
                           budget_mode=1, budget_target=tau)
        H = O.row_entropy(res["scores"][0, 0])
        np.testing.assert_allclose(H, math.log(NT), rtol=1e-12)
        expect = min(max(int(math.floor(float(np.float32(tau)) * NT + 0.5)), 1), NT)
        assert np.all(res["budget"][0, 0] == expect)
        assert np.all(res["count"][0, 0] == expect)


def test_entropy_one_hot_dominant():
    s = np.zeros((1, 20)); s[0, 3] = 60.0
    assert O.row_entropy(s)[0] < 1e-20
    b, x = O.entropy_budgets(np.array([0.0, math.log(20.0)]), 0.5, 20)
    # budgets proportional to exp(H): 1 : 20, total tau*NKT*NQT = 20
    np.testing.assert_allclose(x, [20.0 / 21.0, 400.0 / 21.0], rtol=1e-12)
    assert list(b) == [1, 19]


@pytest.mark.parametrize("grid", [(8, 16, 16), (33, 45, 80)])
def test_radius_for_budget_brute(grid):
    T, Hs, Ws = grid
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    rng = np.random.default_rng(4)
    for _ in range(12):
        i = int(rng.integers(NT))
        b = int(rng.integers(1, NT + 1))
        r = O.radius_for_budget(b, i, T, Hs, Ws)
        sizes = [int(O.window_row(1, rr, i, T, Hs, Ws).sum()) for rr in range(r + 2)]
        assert sizes[r] <= b
        assert sizes[r + 1] > b or sizes[r] == NT


def _decayed_window_by_loops(i, r, T, Hs, Ws):
    """Decayed window of query tile i (|dt| <= r, max(|dy|, |dx|) <= r - |dt|, clipped at the
    grid edges), written out with loops over tile coordinates."""
    nT, nY, nX = O.tile_grid(T, Hs, Ws)
    ti, yi, xi = i // (nY * nX), (i // nX) % nY, i % nX
    out = set()
    for tt in range(nT):
        for ty in range(nY):
            for tx in range(nX):
                dt = abs(tt - ti)
                if dt <= r and max(abs(ty - yi), abs(tx - xi)) <= r - dt:
                    out.add((tt * nY + ty) * nX + tx)
    return out


def _budget_row_by_definition(b, i, T, Hs, Ws, order_key):
    """The budget-mode row of query tile i written from the definition (Token Radius
    Attention, "Radius construction" and "Entropy-guided budgeting"): the radius grows from
    0 while the next decayed window still fits the budget b (stopping once the window covers
    the grid); the window is then topped up to b tiles with the best tiles outside it, in
    the order given by order_key (best first)."""
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    r = 0
    while len(_decayed_window_by_loops(i, r, T, Hs, Ws)) < NT and \
            len(_decayed_window_by_loops(i, r + 1, T, Hs, Ws)) <= b:
        r += 1
    win = _decayed_window_by_loops(i, r, T, Hs, Ws)
    outside = sorted((j for j in range(NT) if j not in win), key=order_key)
    return win | set(outside[:b - len(win)]), r


def test_budget_rows_planted_composition():
    """Entropy-budget rows under planted scores: which tiles a row holds, not only how many.

    qbar_i = a_i * e1 with a_i spread over a decade, kbar_j = c * (j + 1) * e1: every row ranks
    the key tiles by index (highest first), while its entropy, hence its budget b_i, varies
    with a_i. Each row must equal the decayed window of the largest radius that fits b_i,
    topped up with the highest-indexed tiles outside that window."""
    T, Hs, Ws, d = 12, 16, 20, 4
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    valid = O.slot_valid(T, Hs, Ws)
    alphas = np.geomspace(0.2, 4.0, NT)[np.random.default_rng(31).permutation(NT)]
    qt = np.zeros((1, 1, NT, 64, d))
    kt = np.zeros((1, 1, NT, 64, d))
    for j in range(NT):
        qt[0, 0, j, valid[j]] = alphas[j] * e1
        kt[0, 0, j, valid[j]] = 0.05 * (j + 1) * e1
    res = O.build_mask(qt, kt, np.zeros((1, NT), np.float32), T=T, Hs=Hs, Ws=Ws,
                       window_kind=1, radius=0, topk=0, dense_fraction=0.0,
                       budget_mode=1, budget_target=0.19)
    budgets = res["budget"][0, 0]
    radii, extras = set(), 0
    for i in range(NT):
        expect, r = _budget_row_by_definition(int(budgets[i]), i, T, Hs, Ws, lambda j: -j)
        assert set(np.nonzero(res["mask"][0, 0, i])[0]) == expect, i
        assert res["count"][0, 0, i] == budgets[i]
        radii.add(r)
        extras += int(budgets[i]) - len(_decayed_window_by_loops(i, r, T, Hs, Ws))
    # the case is not degenerate: several budgets and radii, and rows with top-up tiles
    assert len(set(budgets.tolist())) >= 5 and len(radii) >= 2 and extras > 0


def test_budget_rows_dominant_tile_outside_window():
    """Uniform kbar except one dominant key tile: every row holds its decayed window, that
    tile, and then the lowest-indexed tiles outside the window (ties to the lower index)."""
    T, Hs, Ws, d = 12, 16, 20, 4
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    star = 37
    kvals = [e1 * (6.0 if j == star else 1.0) for j in range(NT)]
    qt, kt = _planted(T, Hs, Ws, 1, d, kvals, e1)
    res = O.build_mask(qt, kt, np.zeros((1, NT), np.float32), T=T, Hs=Hs, Ws=Ws,
                       window_kind=1, radius=0, topk=0, dense_fraction=0.0,
                       budget_mode=1, budget_target=0.3)
    b = int(res["budget"][0, 0, 0])
    assert np.all(res["budget"][0, 0] == b) and b == 18        # equal entropies: round(0.3 * 60)
    n_star_outside = 0
    for i in range(NT):
        expect, r = _budget_row_by_definition(b, i, T, Hs, Ws, lambda j: (j != star, j))
        got = set(np.nonzero(res["mask"][0, 0, i])[0])
        assert got == expect, i
        n_star_outside += star not in _decayed_window_by_loops(i, r, T, Hs, Ws)
    assert n_star_outside > NT // 2


# ------------------------------------------------------------------------------ near-tie band
# Mask disagreements are allowed only where score gaps are below 1e-4 relative (the
# benchmark's tolerance statement); the pins use that number, not the oracle's constant.
BAND = 1e-4


def test_near_tie_flag_both_sides_of_band():
    """The boundary gap is judged against 1e-4 of the row's largest |score|: a gap of half
    that band is flagged, a gap of twice the band is not."""
    scale = 10.0
    base = np.array([scale, 9.0, 8.0, 0.0, 1.0, -3.0, 0.5, 2.0])
    excluded = np.zeros(base.size, dtype=bool)
    for frac, flagged in ((0.5, True), (0.99, True), (1.01, False), (2.0, False)):
        s = base.copy()
        s[3] = 8.0 - frac * BAND * scale        # the 4th best, just below the 3rd
        assert O.boundary_near_tie(s, excluded, 3) == flagged, frac
    # the band is relative to the row's scale, not to the scores at the boundary
    s = base.copy() * 1e3
    s[3] = s[2] - 0.5e-4 * np.abs(s).max()
    assert O.boundary_near_tie(s, excluded, 3)
    s[3] = s[2] - 2e-4 * np.abs(s).max()
    assert not O.boundary_near_tie(s, excluded, 3)
    # an excluded (window) tile never takes part in the boundary
    s = base.copy()
    s[3] = 8.0 - 0.5 * BAND * scale
    ex = excluded.copy(); ex[3] = True
    assert not O.boundary_near_tie(s, ex, 3)


@pytest.mark.parametrize("gap_in_bands,flagged", [(0.5, True), (2.0, False)])
def test_near_tie_flag_through_build_mask(gap_in_bands, flagged):
    """Fixed top-k rows under planted scores: the k-th and (k+1)-th best tiles outside the
    window differ by gap_in_bands times the band; rows are flagged exactly when that gap is
    inside the band."""
    T, Hs, Ws, d, k = 8, 16, 16, 4, 2
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    top, second, third = NT - 1, NT - 2, NT - 3       # the graded order puts these first
    vals = [0.01 * (j + 1) for j in range(NT)]
    smax = vals[top]
    vals[third] = vals[second] - gap_in_bands * BAND * smax
    qt, kt = _planted(T, Hs, Ws, 1, d, [v * e1 for v in vals], e1)
    res = O.build_mask(qt, kt, np.zeros((1, NT), np.float32), T=T, Hs=Hs, Ws=Ws,
                       window_kind=0, radius=0, topk=k, dense_fraction=0.0)
    for i in range(NT):
        if i in (top, second, third):
            continue                                   # the window removes one of the three
        assert set(np.nonzero(res["mask"][0, 0, i])[0]) == {i, top, second}
        assert res["near_tie"][0, 0, i] == flagged, i


@pytest.mark.parametrize("offset_in_bands,flagged", [(0.5, True), (2.0, False)])
def test_budget_half_integer_flag_both_sides(offset_in_bands, flagged):
    """Budget mode: a pre-rounding budget within 1e-4*max(x, 1) of a half-integer is flagged,
    one twice that band away is not. Equal rows (the same qbar for every query tile) make
    every pre-rounding budget tau*NKT; the graded kbar keeps the score gaps far from their
    own band."""
    T, Hs, Ws, d = 8, 16, 16, 4
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    qt, kt = _planted(T, Hs, Ws, 1, d, [0.02 * (j + 1) * e1 for j in range(NT)], e1)
    x0 = 6.5
    tau = (x0 + offset_in_bands * BAND * x0) / NT
    res = O.build_mask(qt, kt, np.zeros((1, NT), np.float32), T=T, Hs=Hs, Ws=Ws,
                       window_kind=1, radius=0, topk=0, dense_fraction=0.0,
                       budget_mode=1, budget_target=tau)
    np.testing.assert_allclose(res["budget_x"][0, 0], float(np.float32(tau)) * NT, rtol=1e-12)
    assert np.all(res["budget"][0, 0] == 7)
    assert np.all(res["near_tie"][0, 0] == flagged)


# ------------------------------------------------------------------------------ bitmask
def test_bitmask_layout():
    m = np.zeros((2, 70), dtype=bool)
    m[0, [0, 31, 32, 69]] = True
    m[1, 33] = True
    bits = O.pack_bitmask(m)
    assert bits.shape == (2, 3) and bits.dtype == np.uint32
    assert bits[0, 0] == (1 | (1 << 31)) and bits[0, 1] == 1 and bits[0, 2] == (1 << 5)
    assert bits[1, 1] == 2
    assert np.array_equal(O.unpack_bitmask(bits, 70), m)


# ------------------------------------------------------------------------------ attention
def _qkv(grid, B=1, H=2, d=8, seed=21):
    T, Hs, Ws = grid
    N = T * Hs * Ws
    return [_rand((B, N, H, d), seed + i) for i in range(3)]


@pytest.mark.parametrize("grid", [(4, 8, 8), (6, 10, 9)])
def test_all_retained_equals_dense_sdpa(grid):
    """All tiles retained == textbook dense softmax attention on the raster sequence."""
    T, Hs, Ws = grid
    q, k, v = _qkv(grid)
    qt, kt, vt = (O.reorder(a, T, Hs, Ws) for a in (q, k, v))
    NT = qt.shape[2]
    mask = np.ones((1, 2, NT, NT), dtype=bool)
    Ot, L = O.attention(qt, kt, vt, mask, T=T, Hs=Hs, Ws=Ws)
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3)
    np.testing.assert_allclose(Ot, ref.numpy(), rtol=1e-11, atol=1e-12)
    s = np.einsum("bnhd,bmhd->bhnm", q, k) / math.sqrt(8)
    lse_ref = np.log(np.exp(s).sum(-1))
    np.testing.assert_allclose(L, lse_ref, rtol=1e-12)


def test_sparse_equals_sdpa_with_token_mask():
    """A random tile mask expanded to tokens and fed to SDPA in raster order."""
    grid = (6, 10, 9)
    T, Hs, Ws = grid
    q, k, v = _qkv(grid, B=2, H=3, d=8, seed=31)
    qt, kt, vt = (O.reorder(a, T, Hs, Ws) for a in (q, k, v))
    NT = qt.shape[2]
    rng = np.random.default_rng(9)
    mask = rng.random((2, 3, NT, NT)) < 0.3
    mask[..., np.arange(NT), np.arange(NT)] = True
    Ot, L = O.attention(qt, kt, vt, mask, T=T, Hs=Hs, Ws=Ws)
    N = T * Hs * Ws
    tile_of = np.zeros(N, dtype=np.int64)
    src = O.slot_tokens(T, Hs, Ws)
    for j in range(NT):
        for r in range(64):
            if src[j, r] >= 0:
                tile_of[src[j, r]] = j
    tok_mask = mask[:, :, tile_of][:, :, :, tile_of]                     # [B,H,N,N]
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.from_numpy(tok_mask)).permute(0, 2, 1, 3)
    np.testing.assert_allclose(Ot, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_brute_force_per_query_softmax():
    """Plain loops over tokens, membership by tile lookup, on a tiny ragged grid."""
    T, Hs, Ws = 5, 6, 5
    q, k, v = _qkv((T, Hs, Ws), H=1, d=3, seed=41)
    qt, kt, vt = (O.reorder(a, T, Hs, Ws) for a in (q, k, v))
    nT, nY, nX = O.tile_grid(T, Hs, Ws)
    NT = nT * nY * nX
    mask = np.random.default_rng(2).random((1, 1, NT, NT)) < 0.5
    mask[..., np.arange(NT), np.arange(NT)] = True
    Ot, L = O.attention(qt, kt, vt, mask, T=T, Hs=Hs, Ws=Ws)

    def tile(n):
        t, rem = divmod(n, Hs * Ws)
        y, x = divmod(rem, Ws)
        return ((t // 4) * nY + y // 4) * nX + x // 4

    N = T * Hs * Ws
    for n in range(N):
        s = []
        for m in range(N):
            if mask[0, 0, tile(n), tile(m)]:
                s.append((sum(q[0, n, 0, c] * k[0, m, 0, c] for c in range(3)) / math.sqrt(3), m))
        mx = max(a for a, _ in s)
        z = sum(math.exp(a - mx) for a, _ in s)
        o = [sum(math.exp(a - mx) / z * v[0, m, 0, c] for a, m in s) for c in range(3)]
        assert np.allclose(Ot[0, n, 0], o, rtol=1e-12, atol=1e-13)
        assert abs(L[0, 0, n] - (mx + math.log(z))) < 1e-12


def test_weights_cover_exactly_retained_valid_keys():
    T, Hs, Ws = 6, 10, 9
    q, k, v = _qkv((T, Hs, Ws), H=1, d=4, seed=51)
    qt, kt, vt = (O.reorder(a, T, Hs, Ws) for a in (q, k, v))
    NT = qt.shape[2]
    mask = np.random.default_rng(3).random((1, 1, NT, NT)) < 0.4
    mask[..., np.arange(NT), np.arange(NT)] = True
    valid = O.slot_valid(T, Hs, Ws)
    rows = [(0, 0, i) for i in range(NT)]
    res = O.attention_tiles(qt, kt, vt, mask, rows, T=T, Hs=Hs, Ws=Ws, return_weights=True)
    for (b, h, i), e in res.items():
        ids = {tuple(x) for x in e["key_ids"]}
        expect = {(j, r) for j in np.nonzero(mask[0, 0, i])[0] for r in range(64) if valid[j, r]}
        assert ids == expect
        w = e["weights"][e["valid"]]
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-13)
        assert np.all(w > 0)


def test_zero_query_gives_mean_of_retained_values():
    T, Hs, Ws = 6, 10, 9
    q, k, v = _qkv((T, Hs, Ws), H=1, d=4, seed=61)
    q[:] = 0.0
    qt, kt, vt = (O.reorder(a, T, Hs, Ws) for a in (q, k, v))
    NT = qt.shape[2]
    mask = np.random.default_rng(5).random((1, 1, NT, NT)) < 0.4
    mask[..., np.arange(NT), np.arange(NT)] = True
    valid = O.slot_valid(T, Hs, Ws)
    res = O.attention_tiles(qt, kt, vt, mask, [(0, 0, i) for i in range(NT)], T=T, Hs=Hs, Ws=Ws)
    for (b, h, i), e in res.items():
        keep = np.nonzero(mask[0, 0, i])[0]
        vals = np.concatenate([vt[0, 0, j][valid[j]] for j in keep])
        np.testing.assert_allclose(e["o"][e["valid"]], np.broadcast_to(vals.mean(0), (e["valid"].sum(), 4)),
                                   rtol=1e-12)
        np.testing.assert_allclose(e["lse"][e["valid"]], math.log(len(vals)), rtol=1e-13)


def test_single_valid_key_returns_its_value():
    T, Hs, Ws = 5, 5, 5                        # tile (1,1,1) holds exactly one token
    q, k, v = _qkv((T, Hs, Ws), H=1, d=4, seed=71)
    qt, kt, vt = (O.reorder(a, T, Hs, Ws) for a in (q, k, v))
    NT = qt.shape[2]
    last = NT - 1
    assert O.slot_valid(T, Hs, Ws)[last].sum() == 1
    mask = np.zeros((1, 1, NT, NT), dtype=bool)
    mask[0, 0, :, last] = True
    Ot, _ = O.attention(qt, kt, vt, mask, T=T, Hs=Hs, Ws=Ws)
    n_last = T * Hs * Ws - 1
    np.testing.assert_allclose(Ot[0, :, 0, :], np.broadcast_to(v[0, n_last, 0], (T * Hs * Ws, 4)),
                               rtol=1e-14)


def test_full_forward_tiny_is_dense():
    """The 4x8x8 grid has 4 tiles, all inside a radius-1 cube: the path is dense attention."""
    from bsa_synth import WORKLOADS, generate_qkv, generate_difficulty
    w = WORKLOADS["tiny"]
    q, k, v = (O.to_f64(t) for t in generate_qkv(w))
    res = O.forward(q, k, v, generate_difficulty(w).numpy(), T=w.T, Hs=w.Hs, Ws=w.Ws,
                    window_kind=0, radius=1, topk=1, dense_fraction=0.25)
    assert res["mask"].all()
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3)
    np.testing.assert_allclose(res["O"], ref.numpy(), rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------------------------ cumulative mass
def _mass_mask(qt, kt, NT, T, Hs, Ws, theta, kind=1, radius=1):
    return O.build_mask(qt, kt, np.zeros((1, NT), np.float32), T=T, Hs=Hs, Ws=Ws,
                        window_kind=kind, radius=radius, topk=0, dense_fraction=0.0,
                        budget_mode=2, budget_target=theta)


def test_mass_uniform_scores_closed_form():
    """Identical kbar: every pooled probability is 1/NKT, so the rule adds
    ceil(theta * NKT - |window|) tiles (none when the window already holds theta), the
    lowest-indexed ones outside the window."""
    T, Hs, Ws, d = 8, 16, 16, 4
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    qt, kt = _planted(T, Hs, Ws, 1, d, [e1] * NT, 0.3 * e1)
    W = O.window(1, 1, T, Hs, Ws)
    for theta in (0.125, 0.5, 0.75, 1.0):
        th = float(np.float32(theta))
        res = _mass_mask(qt, kt, NT, T, Hs, Ws, theta)
        for i in range(NT):
            m = max(0, math.ceil(th * NT - W[i].sum() - 1e-9))
            outside = [j for j in range(NT) if not W[i, j]]
            assert set(np.nonzero(res["mask"][0, 0, i])[0]) == set(np.nonzero(W[i])[0]) | set(outside[:m])


def test_mass_limits():
    """theta = 1 keeps every tile; a target below the window's own mass keeps the window."""
    T, Hs, Ws, d = 8, 16, 16, 8
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    rng = np.random.default_rng(5)
    qt = rng.standard_normal((1, 2, NT, 64, d)); kt = rng.standard_normal((1, 2, NT, 64, d))
    full = _mass_mask(qt, kt, NT, T, Hs, Ws, 1.0)
    assert full["mask"].all()
    W = O.window(1, 1, T, Hs, Ws)
    tiny = _mass_mask(qt, kt, NT, T, Hs, Ws, 1e-12)
    assert np.array_equal(tiny["mask"][0, 0], W) and np.array_equal(tiny["mask"][0, 1], W)


def test_mass_planted_dominant_tile():
    """One key tile whose score dwarfs the rest carries almost all the pooled mass: a target
    of one half adds exactly that tile (or nothing when it lies in the window)."""
    T, Hs, Ws, d = 8, 16, 16, 4
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    e1 = np.zeros(d); e1[0] = 1.0
    star = 17
    kvals = [e1 * (40.0 if j == star else 0.0) for j in range(NT)]
    qt, kt = _planted(T, Hs, Ws, 1, d, kvals, e1)
    res = _mass_mask(qt, kt, NT, T, Hs, Ws, 0.5)
    W = O.window(1, 1, T, Hs, Ws)
    for i in range(NT):
        assert set(np.nonzero(res["mask"][0, 0, i])[0]) == set(np.nonzero(W[i])[0]) | {star}


def test_mass_monotone_and_brute_force():
    """Rows grow with theta, and each row equals a brute-force reading of the definition:
    the shortest prefix of the (score desc, index asc) order outside the window whose mass,
    with the window's, reaches theta."""
    T, Hs, Ws, d = 6, 10, 9, 8
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    rng = np.random.default_rng(9)
    qt = 2 * rng.standard_normal((1, 1, NT, 64, d)); kt = 2 * rng.standard_normal((1, 1, NT, 64, d))
    prev = None
    W = O.window(0, 1, T, Hs, Ws)
    for theta in (0.2, 0.4, 0.6, 0.8, 0.95):
        res = _mass_mask(qt, kt, NT, T, Hs, Ws, theta, kind=0, radius=1)
        cnt = res["count"][0, 0]
        if prev is not None:
            assert np.all(cnt >= prev)
        prev = cnt
        S = res["scores"][0, 0]
        th = float(np.float32(theta))
        for i in range(NT):
            e = [math.exp(x - max(S[i])) for x in S[i]]
            z = sum(e)
            p = [x / z for x in e]
            mass = sum(p[j] for j in range(NT) if W[i, j])
            keep = {j for j in range(NT) if W[i, j]}
            for j in sorted((j for j in range(NT) if not W[i, j]), key=lambda j: (-S[i, j], j)):
                if mass >= th:
                    break
                keep.add(j)
                mass += p[j]
            assert set(np.nonzero(res["mask"][0, 0, i])[0]) == keep


# ------------------------------------------------------------------------------ token-level circular support
def _golden_token_support():
    rows = []
    with open(os.path.join(os.path.dirname(__file__), "golden", "token_support_sizes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.mark.parametrize("rho,disc,size", _golden_token_support())
def test_token_support_interior_size(rho, disc, size):
    """Counted by brute force around an interior token: the lattice-point counts."""
    n = np.array([20, 20, 20])
    r = np.arange(-8, 9)
    box = np.stack(np.meshgrid(r, r, r, indexing="ij"), axis=-1).reshape(-1, 3) + n
    inside = O.in_token_support(n[None, :], box, rho)
    assert inside.sum() == size
    same_frame = inside & (box[:, 0] == n[0])
    assert same_frame.sum() == disc


@pytest.mark.parametrize("grid", [(8, 16, 16), (6, 10, 9), (13, 7, 11)])
def test_slot_coords_match_raster_tokens(grid):
    """Each valid slot's (t, y, x) gives back its raster token index (t Hs + y) Ws + x."""
    T, Hs, Ws = grid
    xy = O.slot_coords(T, Hs, Ws)
    tok = O.slot_tokens(T, Hs, Ws)
    valid = O.slot_valid(T, Hs, Ws)
    n = (xy[..., 0] * Hs + xy[..., 1]) * Ws + xy[..., 2]
    assert np.array_equal(n[valid], tok[valid])


def test_token_support_symmetric():
    rng = np.random.default_rng(3)
    a = rng.integers(0, 12, size=(500, 3))
    b = rng.integers(0, 12, size=(500, 3))
    for rho in (0, 1, 2, 4):
        assert np.array_equal(O.in_token_support(a, b, rho), O.in_token_support(b, a, rho))


def _valid_box(T, Hs, Ws):
    """Per tile, the [lo, hi] token range along t, y, x of its valid slots."""
    c = O.tile_coords(T, Hs, Ws) * 4
    hi = np.minimum(c + 3, np.array([T - 1, Hs - 1, Ws - 1]))
    return c, hi


@pytest.mark.parametrize("grid", [(8, 16, 16), (6, 10, 9), (13, 7, 11)])
@pytest.mark.parametrize("rho", [0, 1, 2, 3, 5])
def test_token_window_matches_interval_closed_form(grid, rho):
    """The valid tokens of a tile form a box, and a larger frame distance only shrinks the
    in-plane radius, so tile j is in tile i's window iff the smallest frame gap g_t and the
    smallest row/column gaps g_y, g_x between their boxes satisfy g_t <= rho and
    g_y^2 + g_x^2 <= (rho - g_t)^2."""
    T, Hs, Ws = grid
    lo, hi = _valid_box(T, Hs, Ws)
    gap = np.maximum(0, np.maximum(lo[None, :, :] - hi[:, None, :], lo[:, None, :] - hi[None, :, :]))
    gt, gy, gx = gap[..., 0], gap[..., 1], gap[..., 2]
    expect = (gt <= rho) & (gy ** 2 + gx ** 2 <= (rho - gt) ** 2)
    assert np.array_equal(O.token_window(rho, T, Hs, Ws), expect)


def test_token_window_attention_matches_brute_force():
    """Window kind 2 with top-k extras: the attention equals a softmax over the explicit
    token mask (support inside window tiles, whole extra tiles, every key for dense rows)."""
    T, Hs, Ws, d, H = 6, 10, 9, 8, 2
    rng = np.random.default_rng(31)
    NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
    qt = rng.standard_normal((1, H, NT, 64, d)); kt = rng.standard_normal((1, H, NT, 64, d))
    vt = rng.standard_normal((1, H, NT, 64, d))
    valid = O.slot_valid(T, Hs, Ws)
    for t in (qt, kt, vt):
        t[:, :, ~valid] = 0.0
    diff = rng.random((1, NT)).astype(np.float32)
    rho = 2
    m = O.build_mask(qt, kt, diff, T=T, Hs=Hs, Ws=Ws, window_kind=2, radius=rho, topk=2,
                     dense_fraction=0.25)
    rows = [(0, h, i) for h in range(H) for i in range(NT)]
    res = O.attention_tiles(qt, kt, vt, m["mask"], rows, T=T, Hs=Hs, Ws=Ws, token_rho=rho,
                            window=m["window"], dense=m["dense"])
    xy = O.slot_coords(T, Hs, Ws)
    keys = [(j, s_) for j in range(NT) for s_ in range(64) if valid[j, s_]]
    for (b, h, i) in rows:
        for r in range(64):
            if not valid[i, r]:
                continue
            logits, vals = [], []
            for (j, s_) in keys:
                if not m["mask"][b, h, i, j]:
                    continue
                local = m["window"][i, j] and not m["dense"][b, i]
                if local and not O.in_token_support(xy[i, r], xy[j, s_], rho):
                    continue
                logits.append(float(qt[b, h, i, r] @ kt[b, h, j, s_]) / math.sqrt(d))
                vals.append(vt[b, h, j, s_])
            lg = np.array(logits)
            w = np.exp(lg - lg.max())
            o = (w[:, None] * np.array(vals)).sum(0) / w.sum()
            np.testing.assert_allclose(res[(b, h, i)]["o"][r], o, rtol=1e-10, atol=1e-12)
            assert abs(res[(b, h, i)]["lse"][r] - (lg.max() + math.log(w.sum()))) < 1e-10


# ------------------------------------------------------------------------------ planted mistakes
def test_pins_catch_planted_pool_divisor(monkeypatch):
    """Dividing by 64 instead of the valid count must break the raster-mean pin."""
    def bad_pool(xt, T, Hs, Ws):
        valid = O.slot_valid(T, Hs, Ws).astype(np.float64)
        return np.einsum("bhjrd,jr->bhjd", np.asarray(xt, np.float64), valid) / 64.0
    monkeypatch.setattr(O, "pool", bad_pool)
    with pytest.raises(AssertionError):
        test_pool_matches_raster_block_mean((6, 10, 9))


def test_pins_catch_planted_transpose(monkeypatch):
    """Scoring K against Q (transposed operands) must break the top-k pin."""
    real = O.pooled_scores
    monkeypatch.setattr(O, "pooled_scores", lambda a, b: real(b, a))
    with pytest.raises(AssertionError):
        test_topk_planted_increasing_scores(0)


def test_pins_catch_planted_tie_break(monkeypatch):
    """Breaking ties toward the higher index must break the tie pin."""
    def bad_top(scores_row, excluded, m):
        cand = np.nonzero(~excluded)[0]
        order = np.lexsort((-cand, -scores_row[cand]))
        return cand[order[:m]]
    monkeypatch.setattr(O, "top_outside", bad_top)
    with pytest.raises(AssertionError):
        test_topk_ties_go_to_lower_index()


def test_pins_catch_planted_window_mass(monkeypatch):
    """Forgetting the window's own mass (counting only the added tiles toward the target)
    must break the closed-form mass pin."""
    real = O.mass_extra
    monkeypatch.setattr(O, "mass_extra", lambda p, s, w, t: real(p * np.where(w, 0.0, 1.0), s, w, t))
    with pytest.raises(AssertionError):
        test_mass_uniform_scores_closed_form()


def test_pins_catch_planted_square_support(monkeypatch):
    """A square (Chebyshev) support instead of the circular one must break the size pin."""
    def square(n, m, rho):
        dt = np.abs(m[..., 0] - n[..., 0])
        cheb = np.maximum(np.abs(m[..., 1] - n[..., 1]), np.abs(m[..., 2] - n[..., 2]))
        return (dt <= rho) & (cheb <= rho - dt)
    monkeypatch.setattr(O, "in_token_support", square)
    with pytest.raises(AssertionError):
        test_token_support_interior_size(2, 13, 25)


def test_pins_catch_planted_reversed_routing(monkeypatch):
    """Routing the least difficult query tiles to dense attention must break the route pin."""
    real = O.route_dense
    monkeypatch.setattr(O, "route_dense", lambda d, rho: real(-np.asarray(d), rho))
    with pytest.raises(AssertionError):
        test_route_count_and_order(0.25)


def test_pins_catch_planted_log2_entropy(monkeypatch):
    """Entropy in bits instead of nats must break the scipy pin."""
    real = O.row_entropy
    monkeypatch.setattr(O, "row_entropy", lambda s: real(s) / math.log(2.0))
    with pytest.raises(AssertionError):
        test_entropy_matches_scipy()


def test_pins_catch_planted_window_decay_off_by_one(monkeypatch):
    """A decayed window one tile too wide (max(|dy|,|dx|) <= r - |dt| + 1) must break the
    golden interior sizes."""
    real = O.window

    def bad_window(kind, r, T, Hs, Ws):
        if kind != 1:
            return real(kind, r, T, Hs, Ws)
        c = O.tile_coords(T, Hs, Ws)
        dt = np.abs(c[:, None, 0] - c[None, :, 0])
        dyx = np.maximum(np.abs(c[:, None, 1] - c[None, :, 1]), np.abs(c[:, None, 2] - c[None, :, 2]))
        return (dt <= r) & (dyx <= r - dt + 1)
    monkeypatch.setattr(O, "window", bad_window)
    with pytest.raises(AssertionError):
        test_window_interior_size(1, 2, 45)


def test_pins_catch_planted_topk_inside_window(monkeypatch):
    """Taking the top-k over every key tile (window tiles included) must break the row-size
    invariant |row| = |window| + min(k, outside)."""
    real = O.top_outside
    monkeypatch.setattr(O, "top_outside", lambda s, excluded, m: real(s, np.zeros_like(excluded), m))
    with pytest.raises(AssertionError):
        test_dense_rows_and_mask_invariants()


def test_pins_catch_planted_scale(monkeypatch):
    """Scaling scores by 1/d instead of 1/sqrt(d) must break the dense SDPA pin."""
    real = O.attention_tiles

    def bad(qt, kt, vt, mask, rows, **kw):
        if kw.get("scale") is None:
            kw["scale"] = 1.0 / qt.shape[-1]
        return real(qt, kt, vt, mask, rows, **kw)
    monkeypatch.setattr(O, "attention_tiles", bad)
    with pytest.raises(AssertionError):
        test_all_retained_equals_dense_sdpa((4, 8, 8))


def test_pins_catch_planted_budget_topk_over_whole_row(monkeypatch):
    """Budget mode taking the top b_i tiles over the whole row (window tiles competing with
    the rest) instead of topping the window up from outside it must break the composition
    pin."""
    real = O.top_outside
    monkeypatch.setattr(O, "top_outside",
                        lambda s, excluded, m: real(s, np.zeros_like(excluded), m + int(excluded.sum())))
    with pytest.raises(AssertionError):
        test_budget_rows_planted_composition()


def test_pins_catch_planted_budget_radius_one_short(monkeypatch):
    """A radius one below the largest that fits the budget (more tiles by score, fewer by
    distance) must break the composition pin."""
    real = O.radius_for_budget
    monkeypatch.setattr(O, "radius_for_budget", lambda b, i, T, Hs, Ws: max(real(b, i, T, Hs, Ws) - 1, 0))
    with pytest.raises(AssertionError):
        test_budget_rows_planted_composition()


@pytest.mark.parametrize("band,case", [(1e-3, (2.0, False)), (1e-5, (0.5, True))])
def test_pins_catch_planted_near_tie_band(monkeypatch, band, case):
    """A near-tie band ten times too wide (it would excuse real mask disagreements) or ten
    times too narrow (it would fail rows that float32 may decide either way) must break the
    two-sided band pins."""
    monkeypatch.setattr(O, "NEAR_TIE_REL", band)
    with pytest.raises(AssertionError):
        test_near_tie_flag_through_build_mask(*case)
    with pytest.raises(AssertionError):
        test_budget_half_integer_flag_both_sides(*case)
