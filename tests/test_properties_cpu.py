"""Property tests over random small grids (hypothesis), ragged T, Hs, Ws included, on the CPU.

They check what must hold for every grid, on the oracle and on the mask builder's window
predicate built for the host:
  - reorder / unreorder is a bitwise round trip and puts zeros in padding slots;
  - the host-built window predicate equals the oracle's windows, for every kind;
  - the token-level window is symmetric, holds the tile itself, and holds every tile
    that a valid token pair within the support reaches;
  - every mask row holds its window, has exactly |window| + min(k, outside) tiles in fixed
    mode (every tile for dense rows), and the dense rows are floor(rho NQT + 1/2) query
    tiles of highest difficulty;
  - attention weights sum to 1 over exactly the retained valid keys, each output lies in
    the range of the values it averages, and LSE is at least the largest score.
The examples are derandomised, so every run checks the same grids.
"""
import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from bsa_synth import Workload, generate_difficulty, generate_qkv
from oracle import bsa_oracle as O
from test_window_host import win  # noqa: F401  (the host build of the window predicate)

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)
axis = st.integers(min_value=1, max_value=14)


@SETTINGS
@given(T=axis, Hs=axis, Ws=axis, d=st.sampled_from([4, 8]), seed=st.integers(0, 2**16))
def test_reorder_round_trip(T, Hs, Ws, d, seed):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(1, T * Hs * Ws, 2, d))
    xt = O.reorder(x, T, Hs, Ws)
    valid = O.slot_valid(T, Hs, Ws)
    assert np.all(xt[:, :, ~valid] == 0.0)
    assert np.array_equal(O.unreorder(xt, T, Hs, Ws), x)


@SETTINGS
@given(T=axis, Hs=axis, Ws=axis, kind=st.sampled_from([0, 1, 2]), r=st.integers(0, 9))
def test_host_window_predicate_equals_oracle(win, T, Hs, Ws, kind, r):  # noqa: F811
    assert np.array_equal(win(kind, r, T, Hs, Ws), O.window(kind, r, T, Hs, Ws))


@SETTINGS
@given(T=axis, Hs=axis, Ws=axis, rho=st.integers(0, 12))
def test_token_window_properties(T, Hs, Ws, rho):
    W = O.token_window(rho, T, Hs, Ws)
    assert np.array_equal(W, W.T)                       # the support is symmetric
    assert np.all(np.diag(W))                           # a token supports itself
    # tiles whose closest valid tokens are within rho along one axis and equal on the
    # others are always reached
    c = O.tile_coords(T, Hs, Ws)
    for i in range(c.shape[0]):
        for j in range(c.shape[0]):
            dd = np.abs(c[i] - c[j])
            if np.count_nonzero(dd) == 1 and 4 * dd.max() - 3 <= rho:
                assert W[i, j], (i, j)


def _small_workload(T, Hs, Ws, kind, radius, topk, rho, seed):
    return Workload("prop", B=1, H=2, d=8, T=T, Hs=Hs, Ws=Ws, seed=seed, window_kind=kind,
                    radius=radius, topk=topk, dense_fraction=rho)


@SETTINGS
@given(T=axis, Hs=axis, Ws=axis, kind=st.sampled_from([0, 1, 2]), radius=st.integers(0, 6),
       topk=st.integers(0, 6), rho=st.sampled_from([0.0, 0.25, 0.5]), seed=st.integers(0, 2**16))
def test_mask_rows_hold_window_plus_topk(T, Hs, Ws, kind, radius, topk, rho, seed):
    w = _small_workload(T, Hs, Ws, kind, radius, topk, rho, seed)
    q, k, _ = generate_qkv(w)
    diff = generate_difficulty(w).numpy()
    qt, kt = (O.reorder(O.to_f64(x), T, Hs, Ws) for x in (q, k))
    m = O.build_mask(qt, kt, diff, T=T, Hs=Hs, Ws=Ws, window_kind=kind, radius=radius, topk=topk,
                     dense_fraction=rho)
    NT = qt.shape[2]
    W = O.window(kind, radius, T, Hs, Ws)
    assert m["dense"].sum() == O.n_dense(rho, NT)
    order = np.lexsort((np.arange(NT), -diff[0].astype(np.float64)))
    assert set(np.nonzero(m["dense"][0])[0]) == set(order[:O.n_dense(rho, NT)].tolist())
    for h in range(w.H):
        for i in range(NT):
            row = m["mask"][0, h, i]
            if m["dense"][0, i]:
                assert row.all()
                continue
            assert np.all(row[W[i]])
            assert row.sum() == W[i].sum() + min(topk, NT - W[i].sum())


@SETTINGS
@given(T=axis, Hs=axis, Ws=axis, seed=st.integers(0, 2**16), p=st.floats(0.05, 1.0))
def test_attention_weights_and_ranges(T, Hs, Ws, seed, p):
    w = _small_workload(T, Hs, Ws, 0, 0, 0, 0.0, seed)
    q, k, v = generate_qkv(w)
    qt, kt, vt = (O.reorder(O.to_f64(x), T, Hs, Ws) for x in (q, k, v))
    NT = qt.shape[2]
    rng = np.random.default_rng(seed)
    mask = rng.random((1, w.H, NT, NT)) < p
    mask |= np.eye(NT, dtype=bool)[None, None]
    valid = O.slot_valid(T, Hs, Ws)
    rows = [(0, h, i) for h in range(w.H) for i in range(NT)]
    res = O.attention_tiles(qt, kt, vt, mask, rows, T=T, Hs=Hs, Ws=Ws, return_weights=True)
    for (b, h, i), e in res.items():
        vq = e["valid"]
        wts = e["weights"][vq]
        assert np.allclose(wts.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        assert np.all(wts >= 0)
        ids = e["key_ids"]
        assert np.all(mask[b, h, i, ids[:, 0]]) and np.all(valid[ids[:, 0], ids[:, 1]])
        assert ids.shape[0] == sum(int(valid[j].sum()) for j in np.nonzero(mask[b, h, i])[0])
        V = np.concatenate([vt[b, h, j][valid[j]] for j in np.nonzero(mask[b, h, i])[0]])
        o = e["o"][vq]
        assert np.all(o <= V.max(axis=0) + 1e-9) and np.all(o >= V.min(axis=0) - 1e-9)
        K = np.concatenate([kt[b, h, j][valid[j]] for j in np.nonzero(mask[b, h, i])[0]])
        smax = (qt[b, h, i][vq] @ K.T / np.sqrt(w.d)).max(axis=1)
        assert np.all(e["lse"][vq] >= smax - 1e-9)
