"""CPU checks of bench.py's accounting helpers and of its reference (oracle) arm."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


class _G:
    def __init__(self, B, H, d, T, Hs, Ws):
        self.B, self.H, self.d, self.T, self.Hs, self.Ws = B, H, d, T, Hs, Ws
        self.N = T * Hs * Ws
        self.NT = ((T + 3) // 4) * ((Hs + 3) // 4) * ((Ws + 3) // 4)
        self.NW = (self.NT + 31) // 32


@pytest.mark.parametrize("grid", [(8, 16, 16), (6, 10, 9), (21, 30, 52), (1, 1, 1)])
def test_tile_valid_counts(grid):
    g = _G(1, 1, 64, *grid)
    nv = bench._tile_valid_counts(g)
    assert nv.shape == (g.NT,) and nv.sum() == g.N and nv.max() <= 64 and nv.min() >= 1


def _bits(keep):
    """bool [B, H, NQT, NKT] -> int32 mask words."""
    B, H, NQ, NK = keep.shape
    nw = (NK + 31) // 32
    words = np.zeros((B, H, NQ, nw), np.uint32)
    for j in range(NK):
        words[..., j // 32] |= keep[..., j].astype(np.uint32) << np.uint32(j % 32)
    return torch.from_numpy(words.view(np.int32))


def test_valid_token_flops():
    g = _G(1, 2, 16, 6, 10, 9)
    nv = bench._tile_valid_counts(g).astype(np.float64)
    full = np.ones((1, 2, g.NT, g.NT), bool)
    assert bench._valid_token_flops(g, _bits(full)) == pytest.approx(4 * g.d * 2 * g.N * g.N)
    diag = np.zeros_like(full)
    diag[..., np.arange(g.NT), np.arange(g.NT)] = True
    assert bench._valid_token_flops(g, _bits(diag)) == pytest.approx(4 * g.d * 2 * float((nv * nv).sum()))


def test_mask_bytes():
    g = _G(1, 12, 128, 21, 30, 52)
    assert bench._mask_bytes(g) == 2 * 12 * 624 * 128 * 4 + 12 * 624 * (20 + 1) * 4


def test_reference_arm_prints_a_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
