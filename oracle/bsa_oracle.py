"""CPU oracle for heterogeneous block-sparse video attention (test infrastructure only).

This module is test infrastructure. Only the tests, the smoke check and the CPU baseline
leg of the benchmark may import it; the product path never does. It shares no code with
the CUDA path: it imports numpy (and torch only to read bfloat16 tensors), nothing else.

It computes, plainly and in float64, what the method defines:

  * the tile-major token layout of Token Radius Attention ("Efficient execution" step:
    tokens regrouped into contiguous tiles so the mask is block-sparse);
  * mean pooling of Q and K per tile (VORTA summary, ablation table, "average pooling");
  * pooled scores qbar . kbar / sqrt(d);
  * heterogeneous routing of HetA-DiT (Abstract: uncertain regions get dense global
    attention, reliable ones local attention; a single knob sets the dense share);
  * a 3D tile window, optionally with temporal distance decay (Token Radius Attention,
    "Radius construction"; VORTA "sliding-tile attention"), plus the top-k key tiles by
    pooled score, ties to the lower key index;
  * the entropy-to-budget-to-radius rule (Token Radius Attention, "Entropy-guided
    budgeting" and "Radius construction");
  * a cumulative-mass variant of the extra tiles: beyond the window, the key tiles of
    highest pooled probability until the row's retained pooled mass reaches a target
    (Token Radius Attention summary: the keys needed to capture a target attention mass);
  * masked softmax attention over the retained tiles' valid keys, with a natural-log LSE,
    written back in raster token order.

Readings of points the pages leave open (tile shape, padding, routing granularity, the
entropy budget formula, near-tie bands) are listed with the function that takes them.

Parity status: every function below is pinned by tests/test_oracle_pins.py against closed
forms, brute force, a library routine or invariants. Fidelity to the pages' own learned or
tuned methods (HetA-DiT's uncertainty branch, TRA's analytic entropy approximation, VORTA's
router) is parity unpinned: the pages print no formula or number for them.
"""
from __future__ import annotations

import math

import numpy as np

TILE_EDGE = 4
TILE_TOKENS = 64
NEAR_TIE_REL = 1e-4
MASS_NEAR_TIE = 1e-5


# ----------------------------------------------------------------------------------------
# Geometry: raster tokens, tile-major slots
# ----------------------------------------------------------------------------------------
def tile_grid(T: int, Hs: int, Ws: int) -> tuple[int, int, int]:
    """Tiles per axis (nT, nY, nX) for 4x4x4 cubes; edge tiles are partial (zero padded)."""
    return (-(-T // TILE_EDGE), -(-Hs // TILE_EDGE), -(-Ws // TILE_EDGE))


def tile_coords(T: int, Hs: int, Ws: int) -> np.ndarray:
    """[NT, 3] (tt, ty, tx) of every tile, tile index j = (tt*nY + ty)*nX + tx."""
    nT, nY, nX = tile_grid(T, Hs, Ws)
    out = np.zeros((nT * nY * nX, 3), dtype=np.int64)
    j = 0
    for tt in range(nT):
        for ty in range(nY):
            for tx in range(nX):
                out[j] = (tt, ty, tx)
                j += 1
    return out


def slot_tokens(T: int, Hs: int, Ws: int) -> np.ndarray:
    """[NT, 64] raster token index held by each tile slot, or -1 for a padding slot.

    Tile-major layout (Token Radius Attention, "Efficient execution"): tile j holds the
    4x4x4 cube starting at (4*tt, 4*ty, 4*tx); slot r = (dt*4 + dy)*4 + dx inside it.
    """
    coords = tile_coords(T, Hs, Ws)
    out = np.full((coords.shape[0], TILE_TOKENS), -1, dtype=np.int64)
    for j, (tt, ty, tx) in enumerate(coords):
        for dt in range(TILE_EDGE):
            for dy in range(TILE_EDGE):
                for dx in range(TILE_EDGE):
                    t, y, x = 4 * tt + dt, 4 * ty + dy, 4 * tx + dx
                    if t < T and y < Hs and x < Ws:
                        out[j, (dt * 4 + dy) * 4 + dx] = (t * Hs + y) * Ws + x
    return out


def slot_valid(T: int, Hs: int, Ws: int) -> np.ndarray:
    """[NT, 64] bool: the slot holds a real token."""
    return slot_tokens(T, Hs, Ws) >= 0


def reorder(x: np.ndarray, T: int, Hs: int, Ws: int) -> np.ndarray:
    """[B, N, H, d] raster -> [B, H, NT, 64, d] tile-major, padding slots zero."""
    B, N, H, d = x.shape
    assert N == T * Hs * Ws
    src = slot_tokens(T, Hs, Ws)
    NT = src.shape[0]
    out = np.zeros((B, H, NT, TILE_TOKENS, d), dtype=x.dtype)
    for j in range(NT):
        for r in range(TILE_TOKENS):
            n = src[j, r]
            if n >= 0:
                out[:, :, j, r, :] = x[:, n, :, :]
    return out


def unreorder(xt: np.ndarray, T: int, Hs: int, Ws: int) -> np.ndarray:
    """Inverse of reorder: [B, H, NT, 64, d] -> [B, N, H, d]; padding slots are dropped."""
    B, H, NT, R, d = xt.shape
    src = slot_tokens(T, Hs, Ws)
    out = np.zeros((B, T * Hs * Ws, H, d), dtype=xt.dtype)
    for j in range(NT):
        for r in range(TILE_TOKENS):
            n = src[j, r]
            if n >= 0:
                out[:, n, :, :] = xt[:, :, j, r, :]
    return out


# ----------------------------------------------------------------------------------------
# Mask construction
# ----------------------------------------------------------------------------------------
def pool(xt: np.ndarray, T: int, Hs: int, Ws: int) -> np.ndarray:
    """Mean over the valid tokens of each tile (VORTA, "average pooling"): [B, H, NT, d].

    Reading: padding slots are excluded from the mean (divide by the valid count).
    """
    valid = slot_valid(T, Hs, Ws).astype(np.float64)                  # [NT, 64]
    x = np.asarray(xt, dtype=np.float64)
    s = np.einsum("bhjrd,jr->bhjd", x, valid)
    return s / valid.sum(axis=1)[None, None, :, None]


def pooled_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Pooled tile scores qbar_i . kbar_j / sqrt(d): [B, H, NQT, NKT]."""
    d = qbar.shape[-1]
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / math.sqrt(d)


def n_dense(rho: float, NQT: int) -> int:
    """Number of query tiles routed to dense attention: round-half-up of rho * NQT.

    rho is taken at float32 precision (the precision in which the boundary receives it).
    """
    return int(math.floor(float(np.float32(rho)) * NQT + 0.5))


def route_dense(difficulty: np.ndarray, rho: float) -> np.ndarray:
    """HetA-DiT routing (Abstract): the most difficult query tiles go to dense attention.

    Reading: routing is per query tile and shared by all heads of a batch item; the dense
    set is the n_dense(rho) tiles of highest difficulty, ties to the lower tile index.
    Returns bool [B, NQT].
    """
    B, NQT = difficulty.shape
    out = np.zeros((B, NQT), dtype=bool)
    nd = n_dense(rho, NQT)
    for b in range(B):
        dvals = np.asarray(difficulty[b], dtype=np.float64)
        order = np.lexsort((np.arange(NQT), -dvals))                 # by (-difficulty, index)
        out[b, order[:nd]] = True
    return out


def window(kind: int, r: int, T: int, Hs: int, Ws: int) -> np.ndarray:
    """Local support of every query tile, bool [NQT, NKT] (no wrap at grid edges).

    kind 0 (cube, sliding-tile reading): max(|dt|, |dy|, |dx|) <= r, in tile units.
    kind 1 (temporal distance decay, Token Radius Attention "Radius construction"):
        |dt| <= r and max(|dy|, |dx|) <= r - |dt|: the spatial radius shrinks by one per
        frame-tile of distance.
    kind 2 (token-level circular support of radius r in tokens, see in_token_support):
        the key tiles that hold a token of some query token's support; attention inside
        these tiles is then masked token by token (attention_tiles, token_rho).
    """
    c = tile_coords(T, Hs, Ws)
    dt = np.abs(c[:, None, 0] - c[None, :, 0])
    dy = np.abs(c[:, None, 1] - c[None, :, 1])
    dx = np.abs(c[:, None, 2] - c[None, :, 2])
    if kind == 0:
        return np.maximum(np.maximum(dt, dy), dx) <= r
    if kind == 1:
        return (dt <= r) & (np.maximum(dy, dx) <= r - dt)
    if kind == 2:
        return token_window(r, T, Hs, Ws)
    raise ValueError("window kind must be 0, 1 or 2")


def window_row(kind: int, r: int, i: int, T: int, Hs: int, Ws: int) -> np.ndarray:
    """Window of one query tile i as bool [NKT] (same definition as window())."""
    c = tile_coords(T, Hs, Ws)
    dt = np.abs(c[:, 0] - c[i, 0])
    dy = np.abs(c[:, 1] - c[i, 1])
    dx = np.abs(c[:, 2] - c[i, 2])
    if kind == 0:
        return np.maximum(np.maximum(dt, dy), dx) <= r
    return (dt <= r) & (np.maximum(dy, dx) <= r - dt)


def slot_coords(T: int, Hs: int, Ws: int) -> np.ndarray:
    """Token coordinates (t, y, x) of every slot of every tile, int [NT, 64, 3] (padding
    slots get the coordinates they would have; use slot_valid to drop them)."""
    c = tile_coords(T, Hs, Ws)
    r = np.arange(TILE_TOKENS)
    off = np.stack([r // 16, (r // 4) % 4, r % 4], axis=1)               # (dt, dy, dx)
    return c[:, None, :] * TILE_EDGE + off[None, :, :]


def in_token_support(n: np.ndarray, m: np.ndarray, rho: int) -> np.ndarray:
    """Whether key token m lies in the circular support of query token n (broadcasting over
    leading axes of the [..., 3] coordinate arrays).

    Reading of Token Radius Attention ("Radius construction": query-centred circular
    neighbourhoods whose base radius is applied across frames with temporal distance decay)
    at token level: frame distance |dt| <= rho and in-plane Euclidean distance at most
    rho - |dt|, i.e. dy^2 + dx^2 <= (rho - |dt|)^2.
    """
    dt = np.abs(m[..., 0] - n[..., 0])
    d2 = (m[..., 1] - n[..., 1]) ** 2 + (m[..., 2] - n[..., 2]) ** 2
    return (dt <= rho) & (d2 <= (rho - dt) ** 2)


def token_window(rho: int, T: int, Hs: int, Ws: int) -> np.ndarray:
    """Tile window of the token-level circular support, bool [NQT, NKT]: key tile j is in
    query tile i's window when some valid token of j lies in the support of some valid
    token of i (brute force over token pairs)."""
    xy = slot_coords(T, Hs, Ws)
    valid = slot_valid(T, Hs, Ws)
    NT = xy.shape[0]
    keys = xy[valid]                                                      # [Nvalid, 3]
    key_tile = np.repeat(np.arange(NT), valid.sum(axis=1))
    W = np.zeros((NT, NT), dtype=bool)
    for i in range(NT):
        q = xy[i][valid[i]]                                               # [nq, 3]
        hit = in_token_support(q[:, None, :], keys[None, :, :], rho).any(axis=0)
        W[i, np.unique(key_tile[hit])] = True
    return W


def top_outside(scores_row: np.ndarray, excluded: np.ndarray, m: int) -> np.ndarray:
    """Indices of the m highest scores among non-excluded key tiles, ties to lower index."""
    cand = np.nonzero(~excluded)[0]
    if m <= 0 or cand.size == 0:
        return np.zeros(0, dtype=np.int64)
    order = np.lexsort((cand, -scores_row[cand]))                      # (-score, index)
    return cand[order[:m]]


def boundary_near_tie(scores_row: np.ndarray, excluded: np.ndarray, m: int) -> bool:
    """True when the m-th and (m+1)-th best candidates are closer than the near-tie band.

    Reading of "score gaps below 1e-4 relative": the gap is measured against the largest
    |score| of the row, so that scores near zero (where a float32 evaluation has an error
    set by the magnitude of the terms, not of the result) are judged on the row's scale.
    """
    cand = np.nonzero(~excluded)[0]
    if m <= 0 or m >= cand.size:
        return False
    vals = np.sort(scores_row[cand])[::-1]
    scale = max(float(np.max(np.abs(scores_row))), 1e-30)
    return (vals[m - 1] - vals[m]) < NEAR_TIE_REL * scale


def row_entropy(scores: np.ndarray) -> np.ndarray:
    """Entropy (natural log) of softmax over the last axis of pooled scores.

    Token Radius Attention ("Entropy-guided budgeting") estimates a per-query budget from
    attention entropy; the reading here evaluates the entropy of the pooled tile scores.
    """
    s = np.asarray(scores, dtype=np.float64)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    p = e / e.sum(axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0, p * np.log(p), 0.0)
    return -plogp.sum(axis=-1)


def pooled_probabilities(scores: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (all key tiles) of pooled scores, in float64."""
    s = np.asarray(scores, dtype=np.float64)
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def mass_extra(p_row: np.ndarray, scores_row: np.ndarray, window_row_: np.ndarray,
               theta: float) -> tuple[int, bool]:
    """Number of tiles outside the window that the cumulative-mass rule adds.

    Reading of "the number of keys required to capture a target attention mass" (Token
    Radius Attention summary) at tile granularity: the window is always kept; the tiles
    outside it are taken in decreasing pooled score (ties to the lower index) until the
    pooled probability of the whole row reaches theta, i.e. the smallest m with
    mass(window) + mass(first m) >= theta (every tile outside the window when the target is
    not reached). Returns (m, near) where near flags a row whose cumulative mass passes
    within the band of the target at the crossing, where float32 sums may decide either
    way. The band is MASS_NEAR_TIE plus twice the worst-case relative error of a float32
    sum of NKT positive terms (about NKT * 2^-24 of the total, which is at most 1).
    """
    band = MASS_NEAR_TIE + p_row.shape[0] * 2.0 ** -23
    R = theta - float(p_row[window_row_].sum())
    cand = np.nonzero(~window_row_)[0]
    if R <= 0.0 or cand.size == 0:
        return 0, abs(R) < band
    order = cand[np.lexsort((cand, -scores_row[cand]))]
    cum = np.cumsum(p_row[order])
    m = int(np.searchsorted(cum, R, side="left")) + 1
    if m > cand.size:
        return int(cand.size), abs(cum[-1] - R) < band
    near = abs(cum[m - 1] - R) < band or (m >= 2 and abs(R - cum[m - 2]) < band) or (m == 1 and R < band)
    return m, bool(near)


def entropy_budgets(H_row: np.ndarray, tau: float, NKT: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-query-tile budgets of one (b, h): b_i proportional to exp(H_i).

    Reading (Token Radius Attention: retained density grows log-linearly with entropy):
    b_i = clamp(floor(tau * NKT * NQT * exp(H_i) / sum_i' exp(H_i') + 1/2), 1, NKT), so the
    budgets sum to about tau * NKT * NQT. Returns (budgets int64, pre-rounding values).
    """
    NQT = H_row.shape[0]
    tau64 = float(np.float32(tau))
    e = np.exp(np.asarray(H_row, dtype=np.float64))
    x = tau64 * NKT * NQT * e / e.sum()
    b = np.clip(np.floor(x + 0.5), 1, NKT).astype(np.int64)
    return b, x


def radius_for_budget(b: int, i: int, T: int, Hs: int, Ws: int) -> int:
    """Largest decayed-window radius r whose (edge-clipped) window at tile i fits in b.

    Token Radius Attention ("Radius construction"): budget -> base radius, applied across
    frames with temporal distance decay. Reading: the radius grows from 0 while the next
    window still fits the budget; it stops once the window covers the whole grid.
    """
    nT, nY, nX = tile_grid(T, Hs, Ws)
    NKT = nT * nY * nX
    r = 0
    while int(window_row(1, r, i, T, Hs, Ws).sum()) < NKT and \
            int(window_row(1, r + 1, i, T, Hs, Ws).sum()) <= b:
        r += 1
    return r


def build_mask(qt: np.ndarray, kt: np.ndarray, difficulty: np.ndarray, *, T: int, Hs: int,
               Ws: int, window_kind: int, radius: int, topk: int, dense_fraction: float,
               budget_mode: int = 0, budget_target: float = 0.0) -> dict:
    """Retained key tiles of every (b, h, query tile).

    Steps, in the pages' order: pool Q and K per tile; score; route the dense share
    (HetA-DiT); give every other query tile its local window plus extra tiles by pooled
    score (fixed top-k, or an entropy-derived budget, Token Radius Attention).

    Fixed mode (budget_mode 0): row = window(kind, radius) U top-k tiles outside the window
    (k capped at the number of tiles outside it). Entropy budget (1): row = decayed window
    of radius r_i U the top (b_i - |window|) tiles outside it. Cumulative mass (2): row =
    window(kind, radius) U the fewest best tiles outside it that bring the row's pooled
    probability to budget_target. Dense rows: every key tile.

    Returns dict(mask bool [B,H,NQT,NKT], count int [B,H,NQT], near_tie bool [B,H,NQT],
    qbar, kbar, scores, dense bool [B,NQT], budget, budget_x).
    """
    B, H, NT, R, d = qt.shape
    qbar = pool(qt, T, Hs, Ws)
    kbar = pool(kt, T, Hs, Ws)
    S = pooled_scores(qbar, kbar)
    NQT = NKT = NT
    dense = route_dense(np.asarray(difficulty), dense_fraction)
    mask = np.zeros((B, H, NQT, NKT), dtype=bool)
    near = np.zeros((B, H, NQT), dtype=bool)
    budget = np.zeros((B, H, NQT), dtype=np.int64)
    budget_x = np.zeros((B, H, NQT), dtype=np.float64)
    window_mask = np.zeros((NQT, NKT), dtype=bool)
    if budget_mode == 0:
        W = window(window_kind, radius, T, Hs, Ws)
        window_mask = W
        for b in range(B):
            for h in range(H):
                for i in range(NQT):
                    if dense[b, i]:
                        mask[b, h, i, :] = True
                        continue
                    m = min(topk, int(NKT - W[i].sum()))
                    row = W[i].copy()
                    row[top_outside(S[b, h, i], W[i], m)] = True
                    mask[b, h, i] = row
                    near[b, h, i] = boundary_near_tie(S[b, h, i], W[i], m)
    elif budget_mode == 1:
        if window_kind != 1:
            raise ValueError("the entropy budget uses the decayed window (window_kind 1)")
        Hent = row_entropy(S)
        for b in range(B):
            for h in range(H):
                bud, x = entropy_budgets(Hent[b, h], budget_target, NKT)
                budget[b, h] = bud
                budget_x[b, h] = x
                for i in range(NQT):
                    frac = x[i] - math.floor(x[i])
                    near_half = abs(frac - 0.5) < NEAR_TIE_REL * max(x[i], 1.0)
                    if dense[b, i]:
                        mask[b, h, i, :] = True
                        continue
                    r_i = radius_for_budget(int(bud[i]), i, T, Hs, Ws)
                    Wi = window_row(1, r_i, i, T, Hs, Ws)
                    m = int(bud[i]) - int(Wi.sum())
                    row = Wi.copy()
                    row[top_outside(S[b, h, i], Wi, m)] = True
                    mask[b, h, i] = row
                    near[b, h, i] = near_half or boundary_near_tie(S[b, h, i], Wi, m)
    elif budget_mode == 2:
        W = window(window_kind, radius, T, Hs, Ws)
        window_mask = W
        theta = float(np.float32(budget_target))
        P = pooled_probabilities(S)
        for b in range(B):
            for h in range(H):
                for i in range(NQT):
                    if dense[b, i]:
                        mask[b, h, i, :] = True
                        continue
                    m, near_mass = mass_extra(P[b, h, i], S[b, h, i], W[i], theta)
                    row = W[i].copy()
                    row[top_outside(S[b, h, i], W[i], m)] = True
                    mask[b, h, i] = row
                    near[b, h, i] = near_mass or boundary_near_tie(S[b, h, i], W[i], m)
    else:
        raise ValueError("budget_mode must be 0, 1 or 2")
    return dict(mask=mask, count=mask.sum(axis=-1).astype(np.int64), near_tie=near,
                qbar=qbar, kbar=kbar, scores=S, dense=dense, budget=budget,
                budget_x=budget_x, window=window_mask)


def pack_bitmask(mask: np.ndarray) -> np.ndarray:
    """bool [..., NKT] -> uint32 [..., ceil(NKT/32)], key tile j at bit j%32 of word j//32."""
    NKT = mask.shape[-1]
    W = -(-NKT // 32)
    out = np.zeros(mask.shape[:-1] + (W,), dtype=np.uint64)
    for j in range(NKT):
        out[..., j // 32] |= mask[..., j].astype(np.uint64) << np.uint64(j % 32)
    return out.astype(np.uint32)


def unpack_bitmask(bits: np.ndarray, NKT: int) -> np.ndarray:
    """Inverse of pack_bitmask."""
    out = np.zeros(bits.shape[:-1] + (NKT,), dtype=bool)
    b64 = bits.astype(np.uint64)
    for j in range(NKT):
        out[..., j] = ((b64[..., j // 32] >> np.uint64(j % 32)) & np.uint64(1)) == 1
    return out


# ----------------------------------------------------------------------------------------
# Masked attention
# ----------------------------------------------------------------------------------------
def attention_tiles(qt: np.ndarray, kt: np.ndarray, vt: np.ndarray, mask: np.ndarray,
                    rows: list[tuple[int, int, int]], *, T: int, Hs: int, Ws: int,
                    scale: float | None = None, return_weights: bool = False,
                    token_rho: int | None = None, window: np.ndarray | None = None,
                    dense: np.ndarray | None = None) -> dict:
    """Masked softmax attention for the listed (b, h, query tile) rows, in float64.

    For each valid query token of tile i: s = q . k * scale over the valid tokens of the
    retained key tiles; weights = softmax(s) (max subtracted); o = weights @ v;
    lse = log(sum exp(s)). Output per row: o [64, d] (padding slots zero), lse [64].

    With token_rho (window kind 2), a query token of a local (non-dense) row sees, in the
    key tiles of its tile's window (window [NQT, NKT]), only the tokens of its circular
    support (in_token_support); tiles retained outside the window (the extras) are seen
    whole. dense [B, NQT] marks rows that see every valid token.
    """
    d = qt.shape[-1]
    sc = (1.0 / math.sqrt(d)) if scale is None else scale
    valid = slot_valid(T, Hs, Ws)
    coords = slot_coords(T, Hs, Ws) if token_rho is not None else None
    res = {}
    for (b, h, i) in rows:
        kept = np.nonzero(mask[b, h, i])[0]
        keys = []
        vals = []
        key_ids = []
        for j in kept:
            vm = valid[j]
            keys.append(np.asarray(kt[b, h, j][vm], dtype=np.float64))
            vals.append(np.asarray(vt[b, h, j][vm], dtype=np.float64))
            key_ids.append(np.stack([np.full(vm.sum(), j), np.nonzero(vm)[0]], axis=1))
        K = np.concatenate(keys, axis=0)
        V = np.concatenate(vals, axis=0)
        q = np.asarray(qt[b, h, i], dtype=np.float64)
        s = (q @ K.T) * sc                                               # [64, nk]
        if token_rho is not None and not (dense is not None and dense[b, i]):
            ids = np.concatenate(key_ids, axis=0)                        # [nk, 2] (tile, slot)
            in_win = window[i, ids[:, 0]]
            kc = coords[ids[:, 0], ids[:, 1]]                            # [nk, 3]
            sup = in_token_support(coords[i][:, None, :], kc[None, :, :], token_rho)
            allowed = sup | ~in_win[None, :]
            allowed[~valid[i]] = True                                    # padding rows: any finite value
            s = np.where(allowed, s, -np.inf)
        mx = s.max(axis=1, keepdims=True)
        e = np.exp(s - mx)
        z = e.sum(axis=1, keepdims=True)
        w = e / z
        o = w @ V
        lse = (mx + np.log(z))[:, 0]
        vq = valid[i]
        o[~vq] = 0.0
        lse[~vq] = 0.0
        entry = dict(o=o, lse=lse, valid=vq)
        if return_weights:
            entry["weights"] = w
            entry["key_ids"] = np.concatenate(key_ids, axis=0)
        res[(b, h, i)] = entry
    return res


def attention(qt: np.ndarray, kt: np.ndarray, vt: np.ndarray, mask: np.ndarray, *, T: int,
              Hs: int, Ws: int, scale: float | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Full masked attention: O [B, N, H, d] and LSE [B, H, N] in raster token order."""
    B, H, NT, R, d = qt.shape
    rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(NT)]
    res = attention_tiles(qt, kt, vt, mask, rows, T=T, Hs=Hs, Ws=Ws, scale=scale)
    src = slot_tokens(T, Hs, Ws)
    N = T * Hs * Ws
    O = np.zeros((B, N, H, d), dtype=np.float64)
    L = np.zeros((B, H, N), dtype=np.float64)
    for (b, h, i), e in res.items():
        for r in range(TILE_TOKENS):
            n = src[i, r]
            if n >= 0:
                O[b, n, h] = e["o"][r]
                L[b, h, n] = e["lse"][r]
    return O, L


def forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, difficulty: np.ndarray, *, T: int,
            Hs: int, Ws: int, window_kind: int, radius: int, topk: int,
            dense_fraction: float, budget_mode: int = 0, budget_target: float = 0.0) -> dict:
    """The whole path: reorder -> mask -> masked attention -> raster order."""
    qt = reorder(q, T, Hs, Ws)
    kt = reorder(k, T, Hs, Ws)
    vt = reorder(v, T, Hs, Ws)
    mk = build_mask(qt, kt, difficulty, T=T, Hs=Hs, Ws=Ws, window_kind=window_kind,
                    radius=radius, topk=topk, dense_fraction=dense_fraction,
                    budget_mode=budget_mode, budget_target=budget_target)
    O, L = attention(qt, kt, vt, mk["mask"], T=T, Hs=Hs, Ws=Ws)
    mk.update(O=O, LSE=L, qt=qt, kt=kt, vt=vt)
    return mk


def to_f64(x) -> np.ndarray:
    """Exact float64 view of a (bfloat16 or float) torch tensor or numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)
