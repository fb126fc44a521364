"""The pooled-score arithmetic of the tensor-core score kernel, replayed on the CPU.

The kernel splits each fp32 operand x into hi (x with its low 13 mantissa bits cleared,
exactly a tf32 value) and lo = x - hi, and accumulates hi*hi + hi*lo + lo*hi in fp32 with
tf32 products. Whether the tensor core reads its fp32 inputs by truncating them to tf32 or
by rounding them, hi passes unchanged and lo loses at most 2^-11 of itself (2^-21 of x).
This module replays both readings on the pooled means of seeded workloads and checks that
the scores stay within 2e-6 of the row's score scale of the fp64 values, far inside the
selection's near-tie band of 1e-4, while a single tf32 product does not. It pins the
arithmetic, not the kernel; the GPU mask parity tests pin the kernel.
"""
import numpy as np
import pytest

import _cases as C
from oracle import bsa_oracle as O


def tf32_trunc(x: np.ndarray) -> np.ndarray:
    return (x.astype(np.float32).view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


def tf32_round(x: np.ndarray) -> np.ndarray:
    """Round to nearest (ties to even) at 10 mantissa bits."""
    u = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(13)) & np.uint64(1)
    u = (u + np.uint64(0xFFF) + lsb) & np.uint64(0xFFFFE000)
    return u.astype(np.uint32).view(np.float32)


def scores_3xtf32(q: np.ndarray, k: np.ndarray, conv) -> np.ndarray:
    """[n, d] x [m, d] -> [n, m], fp32 accumulation over d in order, tf32 products."""
    qh = tf32_trunc(q)
    ql = (q.astype(np.float32) - qh).astype(np.float32)
    kh = tf32_trunc(k)
    kl = (k.astype(np.float32) - kh).astype(np.float32)
    a = [(conv(qh), conv(kh)), (conv(qh), conv(kl)), (conv(ql), conv(kh))]
    acc = np.zeros((q.shape[0], k.shape[0]), np.float32)
    for c in range(q.shape[1]):
        for x, y in a:
            acc = (acc + np.outer(x[:, c], y[:, c]).astype(np.float32)).astype(np.float32)
    return acc


def scores_1xtf32(q, k, conv):
    acc = np.zeros((q.shape[0], k.shape[0]), np.float32)
    x, y = conv(q), conv(k)
    for c in range(q.shape[1]):
        acc = (acc + np.outer(x[:, c], y[:, c]).astype(np.float32)).astype(np.float32)
    return acc


def _pooled(name):
    w, q, k, _, _ = C.inputs(name)
    qt, kt = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k))
    return O.pool(qt, w.T, w.Hs, w.Ws), O.pool(kt, w.T, w.Hs, w.Ws)


@pytest.mark.parametrize("name", ["small128", "ragged128", "tiny_ragged"])
@pytest.mark.parametrize("conv", [tf32_trunc, tf32_round])
def test_3xtf32_scores_within_near_tie_band(name, conv):
    qbar, kbar = _pooled(name)
    worst3 = worst1 = 0.0
    for b in range(qbar.shape[0]):
        for h in range(qbar.shape[1]):
            q = qbar[b, h].astype(np.float32)
            k = kbar[b, h].astype(np.float32)
            exact = q.astype(np.float64) @ k.astype(np.float64).T
            scale = np.abs(exact).max(axis=1, keepdims=True)
            worst3 = max(worst3, float((np.abs(scores_3xtf32(q, k, conv) - exact) / scale).max()))
            worst1 = max(worst1, float((np.abs(scores_1xtf32(q, k, conv) - exact) / scale).max()))
    assert worst3 < 2e-6, worst3
    assert worst1 > 1e-5, worst1        # one tf32 product alone is far coarser


def test_split_is_exact():
    rng = np.random.default_rng(3)
    x = (rng.normal(size=4096) * np.exp2(rng.integers(-20, 20, 4096))).astype(np.float32)
    hi = tf32_trunc(x)
    lo = (x - hi).astype(np.float32)
    assert np.array_equal((hi.astype(np.float64) + lo.astype(np.float64)), x.astype(np.float64))
    assert np.array_equal(tf32_trunc(hi), hi) and np.array_equal(tf32_round(hi), hi)
