"""The mask builder's window predicate (csrc/window.cuh), built for the host with g++ and
compared tile pair by tile pair with the oracle's windows: for the cube and decayed
windows the oracle's definitions, for the token-level circular support (kind 2) the
oracle's brute force over token pairs, which the predicate replaces by per-axis gap
arithmetic. The select kernel evaluates the same source on the device."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import bsa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_major_b200", "csrc")


@pytest.fixture(scope="module")
def win(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    so = str(tmp_path_factory.mktemp("win") / "libwin.so")
    subprocess.run([cxx, "-O1", "-std=c++17", "-shared", "-fPIC", "-I", CSRC,
                    os.path.join(ROOT, "tests", "window_host.cpp"), "-o", so], check=True)
    lib = ctypes.CDLL(so)
    lib.window_tiles.restype = ctypes.c_int
    lib.window_tiles.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p]
    lib.support_slots.restype = ctypes.c_ulonglong
    lib.support_slots.argtypes = [ctypes.c_int] * 7
    lib.all_inside.restype = ctypes.c_int
    lib.all_inside.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p]

    def run(kind, r, T, Hs, Ws):
        NT = int(np.prod(O.tile_grid(T, Hs, Ws)))
        out = np.zeros((NT, NT), dtype=np.uint8)
        assert lib.window_tiles(T, Hs, Ws, kind, r, out.ctypes.data) == NT
        return out.astype(bool)
    run.lib = lib
    return run


GRIDS = [(8, 16, 16), (6, 10, 9), (13, 7, 11), (5, 5, 5), (3, 3, 3), (1, 1, 1), (17, 2, 29)]


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("kind,radii", [(0, (0, 1, 2, 3)), (1, (0, 1, 2, 4))])
def test_tile_windows_match_oracle(win, grid, kind, radii):
    for r in radii:
        assert np.array_equal(win(kind, r, *grid), O.window(kind, r, *grid)), (kind, r)


@pytest.mark.parametrize("grid", GRIDS)
def test_token_support_window_matches_brute_force(win, grid):
    for rho in (0, 1, 2, 3, 4, 5, 6, 9, 10, 14):
        assert np.array_equal(win(2, rho, *grid), O.token_window(rho, *grid)), rho


def test_token_support_window_at_1p3b_grid(win):
    """The 21 x 30 x 52 latent grid (624 tiles, ragged along height and width), at the
    radius that maps the decayed tile window of radius 1 to tokens (4 r + 2)."""
    assert np.array_equal(win(2, 6, 21, 30, 52), O.token_window(6, 21, 30, 52))


def test_token_support_window_extremes(win):
    """The largest accepted radius covers every tile of the largest grid axis by axis; a
    radius of 0 keeps the tile itself only."""
    w = win(2, 32767, 4, 4, 4096)
    assert w.all()
    w0 = win(2, 0, 8, 8, 8)
    assert np.array_equal(w0, np.eye(w0.shape[0], dtype=bool))


@pytest.mark.parametrize("grid", [(8, 16, 16), (6, 10, 9), (13, 7, 11)])
def test_support_slots_match_oracle(win, grid):
    """The per-slot support mask the attention softmax uses inside window tiles, against
    the oracle's token support on the token coordinates of the slots."""
    T, Hs, Ws = grid
    xy = O.slot_coords(T, Hs, Ws)
    NT = xy.shape[0]
    rng = np.random.default_rng(sum(grid))
    for rho in (0, 1, 3, 6, 10):
        W = O.token_window(rho, T, Hs, Ws)
        for _ in range(60):
            i, j = int(rng.integers(NT)), int(rng.integers(NT))
            if rng.random() < 0.7:                          # mostly window pairs
                js = np.nonzero(W[i])[0]
                j = int(js[rng.integers(js.size)])
            r = int(rng.integers(64))
            got = win.lib.support_slots(T, Hs, Ws, i, r, j, rho)
            want = O.in_token_support(xy[i, r][None, :], xy[j], rho)
            bits = sum(1 << s_ for s_ in range(64) if want[s_])
            assert got == bits, (rho, i, r, j)


@pytest.mark.parametrize("grid", [(8, 16, 16), (6, 10, 9), (13, 7, 11), (5, 5, 5)])
def test_all_inside_matches_brute_force(win, grid):
    """Tile pairs that need no per-token mask: every valid token pair in the support."""
    T, Hs, Ws = grid
    xy = O.slot_coords(T, Hs, Ws)
    valid = O.slot_valid(T, Hs, Ws)
    NT = xy.shape[0]
    for rho in (0, 2, 5, 6, 9, 14):
        out = np.zeros((NT, NT), dtype=np.uint8)
        assert win.lib.all_inside(T, Hs, Ws, rho, out.ctypes.data) == NT
        for i in range(NT):
            q = xy[i][valid[i]]
            for j in range(NT):
                k = xy[j][valid[j]]
                want = bool(O.in_token_support(q[:, None, :], k[None, :, :], rho).all())
                assert bool(out[i, j]) == want, (rho, i, j)
