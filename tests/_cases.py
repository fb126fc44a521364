"""Shared helpers of the parity tests: seeded inputs, oracle runs and comparisons."""
from __future__ import annotations

import functools
import math

import numpy as np
import torch

from bsa_synth import WORKLOADS, Workload, generate_difficulty, generate_qkv
from oracle import bsa_oracle as O

# Tolerances of the GPU path against the fp64 oracle (attention output relative L2 and max
# abs error on bf16-rounded inputs; natural-log LSE absolute error).
O_REL_L2 = 5e-3
O_MAX_ABS = 2e-2
LSE_ABS = 1e-3
# The output is bf16, and the P.V product takes bf16 probabilities (each rounded by up to
# 2^-9 of itself). Where half a bf16 ulp of |O| is well under the max-abs bound (|O| < 4:
# at most 2^-7) the bound is held literally: 2e-2. Above that, half an ulp (2^-6 and up)
# takes most of the bound by itself, and the literal bound would leave less computation
# error than the rounding of bf16 probabilities implies; there the bound is half an ulp
# plus the computation error the literal bound allows at |O| just below 4:
#   max(O_MAX_ABS, half_ulp_bf16(O) + O_PRE_ROUNDING),  O_PRE_ROUNDING = 2e-2 - 2^-7.
O_PRE_ROUNDING = O_MAX_ABS - 2.0 ** -7

SMALL_D128 = {
    "small128": Workload("small128", B=1, H=2, d=128, T=8, Hs=16, Ws=16, seed=1010,
                         window_kind=1, radius=1, topk=2, dense_fraction=0.25),
    "ragged128": Workload("ragged128", B=2, H=3, d=128, T=7, Hs=13, Ws=10, seed=1011,
                          window_kind=0, radius=1, topk=3, dense_fraction=0.2),
    "budget128": Workload("budget128", B=1, H=2, d=128, T=12, Hs=16, Ws=20, seed=1012,
                          window_kind=1, radius=0, topk=0, dense_fraction=0.0,
                          budget_mode=1, budget_target=0.19),
    "mass128": Workload("mass128", B=2, H=2, d=128, T=8, Hs=14, Ws=20, seed=1013,
                        window_kind=0, radius=1, topk=0, dense_fraction=0.2,
                        budget_mode=2, budget_target=0.5),
    # token-level circular support (window kind 2, radius in tokens): fixed top-k on the
    # 8 x 16 x 16 grid, cumulative mass on a ragged grid
    "token128": Workload("token128", B=1, H=2, d=128, T=8, Hs=16, Ws=16, seed=1016,
                         window_kind=2, radius=6, topk=3, dense_fraction=0.25),
    "token_mass": Workload("token_mass", B=2, H=2, d=64, T=7, Hs=13, Ws=10, seed=1017,
                           window_kind=2, radius=5, topk=0, dense_fraction=0.2,
                           budget_mode=2, budget_target=0.5),
    # edge cases: a grid of one (partial) tile, and the largest supported tile count
    "one_tile": Workload("one_tile", B=1, H=2, d=64, T=3, Hs=3, Ws=3, seed=1014,
                         window_kind=0, radius=1, topk=2, dense_fraction=0.0),
    "max_tiles": Workload("max_tiles", B=1, H=1, d=64, T=64, Hs=64, Ws=64, seed=1015,
                          window_kind=0, radius=1, topk=4, dense_fraction=0.05),
}


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    """Half a bfloat16 ulp at |x|: the rounding error of the bf16 output format itself.

    The output is bf16 (rounded to nearest even from fp32), so no implementation can be
    closer than this to the exact value; the max-abs bound applies on top of it.
    """
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def workload(name: str) -> Workload:
    return WORKLOADS[name] if name in WORKLOADS else SMALL_D128[name]


@functools.lru_cache(maxsize=8)
def inputs(name: str, overrides: tuple = ()):
    """bf16 q, k, v [B,N,H,d] (CPU), difficulty [B,NQT] fp32 (CPU) and float64 copies."""
    w = workload(name).with_(**dict(overrides))
    q, k, v = generate_qkv(w)
    diff = generate_difficulty(w)
    return w, q, k, v, diff


def geometry(w: Workload):
    from block_sparse_attention_major_b200 import Geometry
    return Geometry(w.B, w.H, w.d, w.T, w.Hs, w.Ws)


def params(w: Workload):
    from block_sparse_attention_major_b200 import MaskParams
    return MaskParams(w.window_kind, w.radius, w.topk, w.dense_fraction, w.budget_mode,
                      w.budget_target)


def oracle_mask(w: Workload, qt64: np.ndarray, kt64: np.ndarray, diff: np.ndarray) -> dict:
    return O.build_mask(qt64, kt64, diff, T=w.T, Hs=w.Hs, Ws=w.Ws, window_kind=w.window_kind,
                        radius=w.radius, topk=w.topk, dense_fraction=w.dense_fraction,
                        budget_mode=w.budget_mode, budget_target=w.budget_target)


def gpu_mask_bool(mask_i32: torch.Tensor, NKT: int) -> np.ndarray:
    bits = mask_i32.cpu().numpy().view(np.uint32)
    return O.unpack_bitmask(bits, NKT)


def compare_masks(gpu: np.ndarray, ref: dict) -> dict:
    """Row-wise comparison; disagreements are allowed only in rows the oracle flags."""
    diff_rows = np.any(gpu != ref["mask"], axis=-1)
    unflagged = diff_rows & ~ref["near_tie"]
    return dict(n_rows=int(diff_rows.size), n_diff=int(diff_rows.sum()),
                n_unflagged=int(unflagged.sum()), n_flagged=int(ref["near_tie"].sum()),
                diff_rows=diff_rows)


def max_abs_bound(want: np.ndarray) -> np.ndarray:
    """Per-element max-abs bound (see O_PRE_ROUNDING)."""
    return np.maximum(O_MAX_ABS, bf16_half_ulp(want) + O_PRE_ROUNDING)


def mask_for_reference(oracle_mask: np.ndarray, gpu_mask: np.ndarray, diff_rows: np.ndarray) -> np.ndarray:
    """The mask the oracle attends through: its own rows, except rows where the GPU's mask
    differs (allowed only at flagged near-ties), which take the GPU's row so that those rows
    are still checked, against the oracle run under the GPU's own mask."""
    return np.where(diff_rows[..., None], gpu_mask, oracle_mask)


def compare_attention(w: Workload, out: torch.Tensor, lse: torch.Tensor | None, ref: dict) -> dict:
    """GPU out [B,N,H,d] / lse [B,H,N] against oracle per-tile results {(b,h,i): entry}.

    Reports the raw max abs error, the |O| where it occurs, and the largest ratio of an
    element's error to its bound (max_abs_bound); the assertion is on that ratio."""
    src = O.slot_tokens(w.T, w.Hs, w.Ws)
    out64 = out.float().cpu().numpy().astype(np.float64)
    lse64 = lse.cpu().numpy().astype(np.float64) if lse is not None else None
    num = den = 0.0
    max_abs = 0.0
    at_abs = 0.0
    worst_ratio = 0.0
    max_lse = 0.0
    worst_tile = 0.0
    compared = 0
    for (b, h, i), e in ref.items():
        toks = src[i][e["valid"]]
        got = out64[b, toks, h, :]
        want = e["o"][e["valid"]]
        dn = float(((got - want) ** 2).sum())
        dd = float((want ** 2).sum())
        num += dn
        den += dd
        worst_tile = max(worst_tile, math.sqrt(dn / max(dd, 1e-300)))
        err = np.abs(got - want)
        k = np.unravel_index(int(np.argmax(err)), err.shape)
        if err[k] > max_abs:
            max_abs, at_abs = float(err[k]), float(abs(want[k]))
        worst_ratio = max(worst_ratio, float((err / max_abs_bound(want)).max()))
        if lse64 is not None:
            max_lse = max(max_lse, float(np.abs(lse64[b, h, toks] - e["lse"][e["valid"]]).max()))
        compared += 1
    return dict(rel_l2=math.sqrt(num / max(den, 1e-300)), worst_tile_rel_l2=worst_tile,
                max_abs=max_abs, max_abs_at_abs_o=at_abs, max_abs_over_bound=worst_ratio,
                max_lse=max_lse, tiles=compared)


def assert_attention_close(stats: dict) -> None:
    assert stats["tiles"] > 0
    assert stats["rel_l2"] <= O_REL_L2, stats
    assert stats["worst_tile_rel_l2"] <= O_REL_L2, stats
    assert stats["max_abs_over_bound"] <= 1.0, stats
    assert stats["max_lse"] <= LSE_ABS, stats
