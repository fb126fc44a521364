"""GPU parity: every CUDA kernel against the fp64 CPU oracle, through the C ABI.

Reorder / unreorder must be bit-exact. Masks must be bit-exact except in rows the oracle
flags as near-ties (score gaps below 1e-4 of the row's score scale), which are counted.
Attention output must be within relative L2 5e-3 and max abs 2e-2 of the oracle, LSE
within 1e-3.
"""
import numpy as np
import pytest
import torch

import _cases as C
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "tiny_s", "tiny_ragged", "small128", "ragged128", "budget128", "mass128"]


def _bsa():
    import block_sparse_attention_major_b200 as bsa
    return bsa


def _i16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy()


# ----------------------------------------------------------------------------- reorder
@pytest.mark.parametrize("name", SMALL + ["wan13b"])
def test_reorder_bit_exact(name):
    bsa = _bsa()
    w, q, k, v, _ = C.inputs(name)
    g = C.geometry(w)
    for x in (q, k, v):
        xt = bsa.reorder(g, x.cuda())
        ref = O.reorder(_i16(x), w.T, w.Hs, w.Ws)
        assert np.array_equal(_i16(xt), ref)


@pytest.mark.parametrize("name", SMALL + ["wan13b"])
def test_unreorder_round_trip_bit_exact(name):
    bsa = _bsa()
    w, q, _, _, _ = C.inputs(name)
    g = C.geometry(w)
    x = q.cuda()
    back = bsa.unreorder(g, bsa.reorder(g, x))
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
    # unreorder of arbitrary tile-major data equals the oracle's (padding ignored)
    xt = torch.randn((g.B, g.H, g.NT, 64, g.d), device="cuda").to(torch.bfloat16)
    ref = O.unreorder(_i16(xt), w.T, w.Hs, w.Ws)
    assert np.array_equal(_i16(bsa.unreorder(g, xt)), ref)


@pytest.mark.parametrize("name", SMALL + ["wan13b"])
def test_reorder_pool(name):
    """The fused reorder writes the same tile-major tensor as the reorder (bit-exact) and the
    per-tile means of the valid tokens, within fp32 summation error of the oracle's."""
    bsa = _bsa()
    w, q, k, _, _ = C.inputs(name)
    g = C.geometry(w)
    for x in (q, k):
        xt, xbar = bsa.reorder_pool(g, x.cuda())
        torch.cuda.synchronize()
        assert np.array_equal(_i16(xt), O.reorder(_i16(x), w.T, w.Hs, w.Ws))
        x64 = O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws)
        ref = O.pool(x64, w.T, w.Hs, w.Ws)
        # 64 fp32 additions of bf16 values: error below 64 * 2^-24 of the largest magnitude
        bound = 64 * 2.0 ** -24 * np.abs(x64).max(axis=(3, 4))[..., None] + 1e-30
        err = np.abs(xbar.double().cpu().numpy() - ref)
        assert (err <= bound).all(), float((err / bound).max())


# ----------------------------------------------------------------------------- mask
def _mask_case(name, heads=None, overrides=()):
    bsa = _bsa()
    w, q, k, _, diff = C.inputs(name, overrides)
    g = C.geometry(w)
    qt = bsa.reorder(g, q.cuda())
    kt = bsa.reorder(g, k.cuda())
    ws = bsa.alloc_workspace(g)
    mask, cnt = bsa.build_mask(g, C.params(w), qt, kt, diff.cuda(), ws=ws)
    torch.cuda.synchronize()
    assert bsa.read_error(ws) == 0
    gm = C.gpu_mask_bool(mask, g.NT)
    gc = cnt.cpu().numpy()
    hsel = list(range(w.H)) if heads is None else heads
    qt64 = O.reorder(O.to_f64(q), w.T, w.Hs, w.Ws)[:, hsel]
    kt64 = O.reorder(O.to_f64(k), w.T, w.Hs, w.Ws)[:, hsel]
    ref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    gm = gm[:, hsel]
    cmp = C.compare_masks(gm, ref)
    assert np.array_equal(gc[:, hsel], gm.sum(-1)), "kv_count is not the popcount of the row"
    return w, g, gm, ref, cmp, mask, cnt


@pytest.mark.parametrize("name", SMALL + ["wan13b"])
def test_mask_bit_exact(name):
    w, g, gm, ref, cmp, _, _ = _mask_case(name)
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp
    print(f"{name}: rows={cmp['n_rows']} differing={cmp['n_diff']} flagged={cmp['n_flagged']} "
          f"retained={gm.mean():.4f}")


@pytest.mark.parametrize("rho", [0.0, 0.1, 0.2, 0.4, 1.0])
def test_mask_wan5b_rho_sweep(rho):
    w, g, gm, ref, cmp, _, _ = _mask_case("wan5b", heads=[0, 11, 23],
                                          overrides=(("dense_fraction", rho),))
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp
    assert ref["dense"].sum() == O.n_dense(rho, g.NT)


def test_mask_wan14b_heads():
    w, g, gm, ref, cmp, _, _ = _mask_case("wan14b", heads=[0, 39])
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp


@pytest.mark.parametrize("theta", [0.3, 0.7])
def test_mask_mass_wan13b_heads(theta):
    """Cumulative-mass selection on the 1.3B-shaped call (its window, rho = 0.2)."""
    w, g, gm, ref, cmp, _, _ = _mask_case("wan13b", heads=[0, 11],
                                          overrides=(("budget_mode", 2), ("budget_target", theta)))
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp
    print(f"theta={theta}: retained={gm.mean():.4f} flagged={cmp['n_flagged']} differing={cmp['n_diff']}")


@pytest.mark.parametrize("tau", [0.09, 0.19])
def test_mask_hunyuan_budget_heads(tau):
    w, g, gm, ref, cmp, _, _ = _mask_case("hunyuan", heads=[0, 23],
                                          overrides=(("budget_target", tau),))
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp
    retained = gm.mean()
    assert abs(retained - tau) < 0.05, retained


def test_mask_deterministic():
    bsa = _bsa()
    w, q, k, _, diff = C.inputs("wan13b")
    g = C.geometry(w)
    qt, kt = bsa.reorder(g, q.cuda()), bsa.reorder(g, k.cuda())
    m1, c1 = bsa.build_mask(g, C.params(w), qt, kt, diff.cuda())
    m2, c2 = bsa.build_mask(g, C.params(w), qt, kt, diff.cuda())
    assert torch.equal(m1, m2) and torch.equal(c1, c2)


# ----------------------------------------------------------------------------- attention
def _attn_with_mask(w, q, k, v, mask_bool, rows=None):
    """GPU attention given a mask computed here (never from the GPU), plus oracle rows."""
    bsa = _bsa()
    g = C.geometry(w)
    qt, kt, vt = (bsa.reorder(g, x.cuda()) for x in (q, k, v))
    bits = O.pack_bitmask(mask_bool).view(np.int32)
    mask = torch.from_numpy(bits.copy()).cuda()
    cnt = torch.from_numpy(mask_bool.sum(-1).astype(np.int32)).cuda()
    ws = bsa.alloc_workspace(g)
    out, lse = bsa.sparse_attn_fwd(g, qt, kt, vt, mask, cnt, ws=ws)
    torch.cuda.synchronize()
    assert bsa.read_error(ws) == 0
    if rows is None:
        rows = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(g.NT)]
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    ref = O.attention_tiles(qt64, kt64, vt64, mask_bool, rows, T=w.T, Hs=w.Hs, Ws=w.Ws)
    return out, lse, ref


@pytest.mark.parametrize("name", SMALL)
def test_attention_oracle_mask(name):
    w, q, k, v, diff = C.inputs(name)
    qt64, kt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    out, lse, ref = _attn_with_mask(w, q, k, v, mref["mask"])
    st = C.compare_attention(w, out, lse, ref)
    print(name, st)
    C.assert_attention_close(st)


@pytest.mark.parametrize("pattern", ["random", "single", "all", "alternate", "last_only"])
@pytest.mark.parametrize("name", ["ragged128", "tiny_ragged"])
def test_attention_mask_patterns(name, pattern):
    w, q, k, v, _ = C.inputs(name)
    NT = w.NT
    rng = np.random.default_rng(17)
    if pattern == "random":
        m = rng.random((w.B, w.H, NT, NT)) < 0.35
        m[..., np.arange(NT), np.arange(NT)] = True
    elif pattern == "single":
        m = np.zeros((w.B, w.H, NT, NT), dtype=bool)
        m[..., np.arange(NT), rng.integers(0, NT, NT)] = True
    elif pattern == "all":
        m = np.ones((w.B, w.H, NT, NT), dtype=bool)
    elif pattern == "alternate":
        m = np.zeros((w.B, w.H, NT, NT), dtype=bool)
        m[..., 0::2, 0::2] = True      # even query tiles see even key tiles, odd see odd
        m[..., 1::2, 1::2] = True
    else:
        m = np.zeros((w.B, w.H, NT, NT), dtype=bool)
        m[..., :, NT - 1] = True       # every row keeps only the last (partial) tile
    out, lse, ref = _attn_with_mask(w, q, k, v, m)
    st = C.compare_attention(w, out, lse, ref)
    C.assert_attention_close(st)


@pytest.mark.parametrize("name", ["ragged128", "tiny_ragged"])
def test_attention_empty_rows(name):
    """Rows of a caller mask that retain nothing: zeros in O, -inf LSE, BSA_KERR_BAD_MASK;
    the other rows, including those sharing a work unit with the empty ones, as the oracle.
    Query tiles 0 and 1 (one whole query block of the first unit) and a lone query tile 5
    retain nothing."""
    bsa = _bsa()
    w, q, k, v, _ = C.inputs(name)
    g = C.geometry(w)
    NT = w.NT
    rng = np.random.default_rng(29)
    m = rng.random((w.B, w.H, NT, NT)) < 0.35
    m[..., np.arange(NT), np.arange(NT)] = True
    empty = [i for i in (0, 1, 5) if i < NT]
    m[..., empty, :] = False
    qt, kt, vt = (bsa.reorder(g, x.cuda()) for x in (q, k, v))
    mask = torch.from_numpy(O.pack_bitmask(m).view(np.int32).copy()).cuda()
    cnt = torch.from_numpy(m.sum(-1).astype(np.int32)).cuda()
    ws = bsa.alloc_workspace(g)
    out, lse = bsa.sparse_attn_fwd(g, qt, kt, vt, mask, cnt, ws=ws)
    torch.cuda.synchronize()
    assert bsa.read_error(ws) & bsa.KERR_BAD_MASK
    rows = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(NT) if i not in empty]
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    ref = O.attention_tiles(qt64, kt64, vt64, m, rows, T=w.T, Hs=w.Hs, Ws=w.Ws)
    st = C.compare_attention(w, out, lse, ref)
    C.assert_attention_close(st)
    # the empty rows' valid tokens: O = 0, LSE = -inf
    src, valid = O.slot_tokens(w.T, w.Hs, w.Ws), O.slot_valid(w.T, w.Hs, w.Ws)
    toks = np.concatenate([src[i][valid[i]] for i in empty])
    o = out.float().cpu().numpy()
    l = lse.float().cpu().numpy()
    assert np.all(o[:, toks] == 0.0)
    assert np.all(np.isneginf(l[:, :, toks]))


def test_attention_all_retained_equals_dense():
    """All tiles retained: equals dense softmax attention over the raster sequence."""
    bsa = _bsa()
    w, q, k, v, _ = C.inputs("ragged128")
    NT = w.NT
    m = np.ones((w.B, w.H, NT, NT), dtype=bool)
    out, lse, _ = _attn_with_mask(w, q, k, v, m, rows=[])
    tq, tk, tv = (x.double().permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3)
    got = out.double().cpu()
    rel = ((got - ref).norm() / ref.norm()).item()
    ratio = (got - ref).abs().numpy() / C.max_abs_bound(ref.numpy())
    assert rel <= C.O_REL_L2 and ratio.max() <= 1.0, (rel, ratio.max())
    s = torch.einsum("bhnd,bhmd->bhnm", tq, tk) / np.sqrt(w.d)
    assert (lse.double().cpu() - torch.logsumexp(s, -1)).abs().max().item() <= C.LSE_ABS


def test_attention_invariants():
    """V = 1 gives O = 1; V changes in unretained tiles leave O bit-identical."""
    bsa = _bsa()
    w, q, k, v, _ = C.inputs("ragged128")
    g = C.geometry(w)
    NT = w.NT
    rng = np.random.default_rng(5)
    m = rng.random((w.B, w.H, NT, NT)) < 0.3
    m[..., np.arange(NT), np.arange(NT)] = True
    unret_set = [3, 7, 11, 17]                 # key tiles no query tile of head 0 retains
    m[0, 0, :, unret_set] = False
    m[0, 0, unret_set, 0] = True
    mask = torch.from_numpy(O.pack_bitmask(m).view(np.int32).copy()).cuda()
    cnt = torch.from_numpy(m.sum(-1).astype(np.int32)).cuda()
    qt, kt = bsa.reorder(g, q.cuda()), bsa.reorder(g, k.cuda())
    ones = torch.ones((g.B, g.H, NT, 64, g.d), dtype=torch.bfloat16, device="cuda")
    out, _ = bsa.sparse_attn_fwd(g, qt, kt, ones, mask, cnt)
    assert (out.float() - 1).abs().max().item() < 1e-2
    vt = bsa.reorder(g, v.cuda())
    o1, l1 = bsa.sparse_attn_fwd(g, qt, kt, vt, mask, cnt)
    # perturb V in tiles that no query tile of head 0 retains
    unret = ~m[0, 0].any(axis=0)
    vt2 = vt.clone()
    idx = torch.from_numpy(np.nonzero(unret)[0]).cuda()
    if idx.numel() == 0:
        pytest.skip("every tile retained somewhere")
    vt2[0, 0, idx] = vt2[0, 0, idx] * 3 + 1
    o2, l2 = bsa.sparse_attn_fwd(g, qt, kt, vt2, mask, cnt)
    assert torch.equal(o1[0, :, 0].view(torch.int16), o2[0, :, 0].view(torch.int16))
    assert torch.equal(l1, l2)


def test_attention_zero_query_mean_of_values():
    bsa = _bsa()
    w, q, k, v, _ = C.inputs("tiny_ragged")
    NT = w.NT
    rng = np.random.default_rng(6)
    m = rng.random((w.B, w.H, NT, NT)) < 0.4
    m[..., np.arange(NT), np.arange(NT)] = True
    qz = torch.zeros_like(q)
    out, lse, ref = _attn_with_mask(w, qz, k, v, m)
    st = C.compare_attention(w, out, lse, ref)
    C.assert_attention_close(st)
    valid = O.slot_valid(w.T, w.Hs, w.Ws)
    src = O.slot_tokens(w.T, w.Hs, w.Ws)
    for i in range(NT):
        nk = int(sum(valid[j].sum() for j in np.nonzero(m[0, 0, i])[0]))
        toks = src[i][valid[i]]
        assert np.allclose(lse[0, 0, toks].cpu().numpy(), np.log(nk), atol=1e-5)


def test_attention_wan13b_sampled_rows():
    """Full 1.3B-shaped call; oracle on sampled dense and local query tiles."""
    w, q, k, v, diff = C.inputs("wan13b")
    qt64, kt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    rng = np.random.default_rng(3)
    dense_i = np.nonzero(mref["dense"][0])[0]
    local_i = np.nonzero(~mref["dense"][0])[0]
    rows = [(0, int(rng.integers(w.H)), int(i)) for i in rng.choice(dense_i, 6, replace=False)]
    rows += [(0, int(rng.integers(w.H)), int(i)) for i in rng.choice(local_i, 18, replace=False)]
    rows += [(0, w.H - 1, w.NT - 1), (0, 0, 0)]
    out, lse, ref = _attn_with_mask(w, q, k, v, mref["mask"], rows=rows)
    st = C.compare_attention(w, out, lse, ref)
    print(st)
    C.assert_attention_close(st)


# ----------------------------------------------------------------------------- whole path
@pytest.mark.parametrize("name", ["tiny_ragged", "small128", "budget128", "mass128", "wan13b"])
def test_forward_path(name):
    """reorder -> build_mask -> sparse attention on the GPU vs the oracle's whole path."""
    bsa = _bsa()
    w, q, k, v, diff = C.inputs(name)
    g = C.geometry(w)
    b = bsa.forward(g, C.params(w), q.cuda(), k.cuda(), v.cuda(), diff.cuda())
    torch.cuda.synchronize()
    assert bsa.read_error(b.ws) == 0
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    gm = C.gpu_mask_bool(b.mask, g.NT)
    cmp = C.compare_masks(gm, mref)
    assert cmp["n_unflagged"] == 0, cmp
    if name == "wan13b":
        rng = np.random.default_rng(11)
        rows = [(0, int(rng.integers(w.H)), int(rng.integers(g.NT))) for _ in range(20)]
    else:
        rows = [(bb, h, i) for bb in range(w.B) for h in range(w.H) for i in range(g.NT)]
    rows += [tuple(int(x) for x in r) for r in np.argwhere(cmp["diff_rows"])][:8]
    used = C.mask_for_reference(mref["mask"], gm, cmp["diff_rows"])
    ref = O.attention_tiles(qt64, kt64, vt64, used, rows, T=w.T, Hs=w.Hs, Ws=w.Ws)
    st = C.compare_attention(w, b.out, b.lse, ref)
    print(name, st, cmp["n_diff"])
    C.assert_attention_close(st)


def test_forward_path_one_tile():
    """A grid of a single partial tile (27 tokens): one mask word, one query tile per unit,
    no second sub-unit; the whole path against the oracle on every row."""
    bsa = _bsa()
    w, q, k, v, diff = C.inputs("one_tile")
    g = C.geometry(w)
    assert g.NT == 1
    b = bsa.forward(g, C.params(w), q.cuda(), k.cuda(), v.cuda(), diff.cuda())
    torch.cuda.synchronize()
    assert bsa.read_error(b.ws) == 0
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    assert np.array_equal(C.gpu_mask_bool(b.mask, g.NT), mref["mask"])
    rows = [(0, h, 0) for h in range(w.H)]
    ref = O.attention_tiles(qt64, kt64, vt64, mref["mask"], rows, T=w.T, Hs=w.Hs, Ws=w.Ws)
    C.assert_attention_close(C.compare_attention(w, b.out, b.lse, ref))


def test_forward_path_max_tiles():
    """The largest supported grid (4096 tiles: 128 mask words per row, rows spanning four
    selection warps, union lists at their limit): masks on every row, attention on
    sampled rows."""
    bsa = _bsa()
    w, q, k, v, diff = C.inputs("max_tiles")
    g = C.geometry(w)
    assert g.NT == 4096
    b = bsa.forward(g, C.params(w), q.cuda(), k.cuda(), v.cuda(), diff.cuda())
    torch.cuda.synchronize()
    assert bsa.read_error(b.ws) == 0
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    gm = C.gpu_mask_bool(b.mask, g.NT)
    cmp = C.compare_masks(gm, mref)
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp
    rng = np.random.default_rng(17)
    dense_rows = np.nonzero(mref["dense"][0])[0]
    rows = [(0, 0, int(i)) for i in rng.integers(g.NT, size=12)] + [(0, 0, int(dense_rows[0]))]
    rows += [tuple(int(x) for x in r) for r in np.argwhere(cmp["diff_rows"])][:4]
    used = C.mask_for_reference(mref["mask"], gm, cmp["diff_rows"])
    ref = O.attention_tiles(qt64, kt64, vt64, used, rows, T=w.T, Hs=w.Hs, Ws=w.Ws)
    st = C.compare_attention(w, b.out, b.lse, ref)
    C.assert_attention_close(st)


@pytest.mark.parametrize("name,overrides", [("wan14b", ()), ("hunyuan", (("budget_target", 0.14),))])
def test_forward_path_full_size(name, overrides):
    """Whole path on the 14B- and Hunyuan-shaped calls; the oracle checks two heads."""
    bsa = _bsa()
    w, q, k, v, diff = C.inputs(name, overrides)
    g = C.geometry(w)
    b = bsa.forward(g, C.params(w), q.cuda(), k.cuda(), v.cuda(), diff.cuda())
    torch.cuda.synchronize()
    assert bsa.read_error(b.ws) == 0
    heads = [0, w.H - 1]
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x[:, :, heads]), w.T, w.Hs, w.Ws) for x in (q, k, v))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    gm = C.gpu_mask_bool(b.mask, g.NT)[:, heads]
    cmp = C.compare_masks(gm, mref)
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp
    rng = np.random.default_rng(23)
    rows = [(0, int(rng.integers(2)), int(rng.integers(g.NT))) for _ in range(10)]
    rows += [tuple(int(x) for x in r) for r in np.argwhere(cmp["diff_rows"])][:4]
    used = C.mask_for_reference(mref["mask"], gm, cmp["diff_rows"])
    ref = O.attention_tiles(qt64, kt64, vt64, used, rows, T=w.T, Hs=w.Hs, Ws=w.Ws)
    # map the oracle's head slots back to the call's heads
    ref = {(bb, heads[h], i): e for (bb, h, i), e in ref.items()}
    st = C.compare_attention(w, b.out, b.lse, ref)
    print(name, st, cmp["n_diff"], "retained", float(gm.mean()))
    C.assert_attention_close(st)


# ----------------------------------------------------------------------------- window kind 2
@pytest.mark.parametrize("name,overrides", [
    ("token128", ()), ("token_mass", ()),
    ("wan13b", (("window_kind", 2), ("radius", 6))),          # 4 r + 2 tokens for r = 1
])
def test_mask_token_window(name, overrides):
    """Masks whose local support is the token-level circular support (radius in tokens):
    bit-exact against the oracle, whose window is a brute force over token pairs."""
    heads = [0, 11] if name == "wan13b" else None
    w, g, gm, ref, cmp, _, _ = _mask_case(name, heads=heads, overrides=overrides)
    assert cmp["n_unflagged"] == 0, cmp
    assert cmp["n_diff"] <= max(1, cmp["n_rows"] // 200), cmp
    local = ~ref["dense"][:, None, :, None]
    assert np.all(gm >= (ref["window"][None, None] & local)), "a window tile is missing"
    print(f"{name}: retained={gm.mean():.4f} window={ref['window'].mean():.4f} "
          f"flagged={cmp['n_flagged']} differing={cmp['n_diff']}")


def test_forward_mask_reuse():
    """forward(rebuild_mask=False) attends a new call's inputs through the mask an earlier
    call built: against the oracle's attention on the new inputs under the oracle's mask of
    the earlier inputs (rows where the GPU's earlier mask differs at a near-tie skipped)."""
    bsa = _bsa()
    wa, qa, ka, va, da = C.inputs("small128")
    wb, qb, kb, vb, db = C.inputs("small128", (("seed", wa.seed + 7),))
    g = C.geometry(wa)
    p = C.params(wa)
    b = bsa.forward(g, p, qa.cuda(), ka.cuda(), va.cuda(), da.cuda())
    mask_a, cnt_a = b.mask.clone(), b.kv_count.clone()
    n0 = bsa.launch_count()
    bsa.forward(g, p, qb.cuda(), kb.cuda(), vb.cuda(), db.cuda(), bufs=b, rebuild_mask=False)
    torch.cuda.synchronize()
    assert bsa.launch_count() - n0 == bsa.launches_per_forward(p, rebuild_mask=False)
    assert torch.equal(b.mask, mask_a) and torch.equal(b.kv_count, cnt_a)
    assert bsa.read_error(b.ws) == 0
    qa64, ka64 = (O.reorder(O.to_f64(x), wa.T, wa.Hs, wa.Ws) for x in (qa, ka))
    mref = C.oracle_mask(wa, qa64, ka64, da.numpy())
    gm = C.gpu_mask_bool(mask_a, g.NT)
    cmp = C.compare_masks(gm, mref)
    assert cmp["n_unflagged"] == 0, cmp
    qb64, kb64, vb64 = (O.reorder(O.to_f64(x), wb.T, wb.Hs, wb.Ws) for x in (qb, kb, vb))
    rows = [(bb, h, i) for bb in range(wb.B) for h in range(wb.H) for i in range(g.NT)]
    used = C.mask_for_reference(mref["mask"], gm, cmp["diff_rows"])
    ref = O.attention_tiles(qb64, kb64, vb64, used, rows, T=wb.T, Hs=wb.Hs, Ws=wb.Ws)
    st = C.compare_attention(wb, b.out, b.lse, ref)
    print(st)
    C.assert_attention_close(st)


# ----------------------------------------------------------------------------- score kernel
def _ws_offsets(g):
    """Byte offsets of the pooled means and the scores in the workspace. This mirrors the
    library's workspace layout (256-byte aligned regions in a fixed order)."""
    a = lambda x: (x + 255) // 256 * 256
    off = 256
    pooled = g.B * g.H * g.NT * g.d * 4
    qbar = off; off = a(off + pooled)
    kbar = off; off = a(off + pooled)
    off = a(off + g.B * g.NT)                                   # route flags
    off = a(off + g.B * g.H * g.NT * 4)                         # entropy
    off = a(off + g.B * g.H * g.NT * 8)                         # budget plan
    off = a(off + g.B * g.H * 16)                               # per-(b, h) counts
    off = a(off + g.B * g.H * (g.NT // 4 + 2) * 32)             # work units
    return qbar, kbar, off


@pytest.mark.parametrize("name", ["small128", "ragged128", "wan13b"])
def test_scores_against_exact_products(name):
    """The tensor-core scores against the exact products of the GPU's own pooled means:
    within 1e-5 of each row's score scale (3xTF32), a tenth of the selection's near-tie
    band of 1e-4, so that only rows the oracle flags can select differently."""
    bsa = _bsa()
    w, q, k, _, diff = C.inputs(name)
    g = C.geometry(w)
    qt, kt = bsa.reorder(g, q.cuda()), bsa.reorder(g, k.cuda())
    ws = bsa.alloc_workspace(g)
    assert ws.numel() == bsa.workspace_bytes(g)
    bsa.build_mask(g, C.params(w), qt, kt, diff.cuda(), ws=ws)
    torch.cuda.synchronize()
    assert bsa.read_error(ws) == 0
    oq, ok_, os_ = _ws_offsets(g)
    n = g.B * g.H * g.NT * g.d
    qbar = ws[oq:oq + 4 * n].view(torch.float32).view(g.B * g.H, g.NT, g.d).double().cpu().numpy()
    kbar = ws[ok_:ok_ + 4 * n].view(torch.float32).view(g.B * g.H, g.NT, g.d).double().cpu().numpy()
    nktp = (g.NT + 3) // 4 * 4
    S = ws[os_:os_ + 4 * g.B * g.H * g.NT * nktp].view(torch.float32).view(g.B * g.H, g.NT, nktp)
    S = S[:, :, :g.NT].double().cpu().numpy()
    exact = np.einsum("bid,bjd->bij", qbar, kbar)
    scale = np.abs(exact).max(axis=2, keepdims=True)
    err = float((np.abs(S - exact) / scale).max())
    print(name, "max relative score error", err)
    assert err < 1e-5


# ----------------------------------------------------------------------------- token support
def _attn_token(w, q, k, v, mask_bool, dense, rho, rows=None):
    """GPU attention under a token-level support, given a mask and route flags computed
    here (never from the GPU), and the oracle's rows."""
    bsa = _bsa()
    g = C.geometry(w)
    qt, kt, vt = (bsa.reorder(g, x.cuda()) for x in (q, k, v))
    bits = O.pack_bitmask(mask_bool).view(np.int32)
    mask = torch.from_numpy(bits.copy()).cuda()
    cnt = torch.from_numpy(mask_bool.sum(-1).astype(np.int32)).cuda()
    dflags = torch.from_numpy(dense.astype(np.uint8)).cuda()
    ws = bsa.alloc_workspace(g)
    out, lse = bsa.sparse_attn_fwd_token(g, qt, kt, vt, mask, cnt, dflags, rho, ws=ws)
    torch.cuda.synchronize()
    assert bsa.read_error(ws) == 0
    if rows is None:
        rows = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(g.NT)]
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    ref = O.attention_tiles(qt64, kt64, vt64, mask_bool, rows, T=w.T, Hs=w.Hs, Ws=w.Ws, token_rho=rho,
                            window=O.token_window(rho, w.T, w.Hs, w.Ws), dense=dense)
    return out, lse, ref


@pytest.mark.parametrize("name", ["token128", "token_mass"])
def test_attention_token_support_oracle_mask(name):
    """Token-level support inside window tiles, on the oracle's kind-2 mask and route flags."""
    w, q, k, v, diff = C.inputs(name)
    qt64, kt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    out, lse, ref = _attn_token(w, q, k, v, mref["mask"], mref["dense"], w.radius)
    st = C.compare_attention(w, out, lse, ref)
    print(name, st)
    C.assert_attention_close(st)


@pytest.mark.parametrize("rho", [0, 3, 6, 11])
def test_attention_token_support_random_masks(rho):
    """Random tile masks (window tiles and extras alike) and random route flags on a
    ragged grid, across radii from the tile itself (0) to most of the grid."""
    w, q, k, v, diff = C.inputs("ragged128")
    g = C.geometry(w)
    rng = np.random.default_rng(40 + rho)
    m = rng.random((w.B, w.H, g.NT, g.NT)) < 0.4
    m |= np.eye(g.NT, dtype=bool)[None, None]                 # every row keeps its own tile
    dense = rng.random((w.B, g.NT)) < 0.2
    m[dense[:, None, :, None].repeat(w.H, 1).repeat(g.NT, 3)] = True
    out, lse, ref = _attn_token(w, q, k, v, m, dense, rho)
    st = C.compare_attention(w, out, lse, ref)
    print(rho, st)
    C.assert_attention_close(st)


@pytest.mark.parametrize("name,overrides", [("token128", ()), ("token_mass", ()),
                                            ("wan13b", (("window_kind", 2), ("radius", 6)))])
def test_forward_path_token_support(name, overrides):
    """The whole path with window kind 2: GPU mask against the oracle, then the GPU output
    against the oracle's token-masked attention (rows whose GPU mask differs at a flagged
    near-tie under the GPU's own mask)."""
    bsa = _bsa()
    w, q, k, v, diff = C.inputs(name, overrides)
    g = C.geometry(w)
    b = bsa.forward(g, C.params(w), q.cuda(), k.cuda(), v.cuda(), diff.cuda())
    torch.cuda.synchronize()
    assert bsa.read_error(b.ws) == 0
    heads = [0, w.H - 1] if name == "wan13b" else list(range(w.H))
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x[:, :, heads]), w.T, w.Hs, w.Ws) for x in (q, k, v))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    gm = C.gpu_mask_bool(b.mask, g.NT)[:, heads]
    cmp = C.compare_masks(gm, mref)
    assert cmp["n_unflagged"] == 0, cmp
    assert np.array_equal(bsa.route_flags(g, b.ws).cpu().numpy().astype(bool), mref["dense"])
    if name == "wan13b":
        rng = np.random.default_rng(29)
        rows = [(0, int(rng.integers(2)), int(rng.integers(g.NT))) for _ in range(16)]
    else:
        rows = [(bb, h, i) for bb in range(w.B) for h in range(len(heads)) for i in range(g.NT)]
    used = C.mask_for_reference(mref["mask"], gm, cmp["diff_rows"])
    ref = O.attention_tiles(qt64, kt64, vt64, used, rows, T=w.T, Hs=w.Hs, Ws=w.Ws,
                            token_rho=w.radius, window=O.token_window(w.radius, w.T, w.Hs, w.Ws),
                            dense=mref["dense"])
    ref = {(bb, heads[h], i): e for (bb, h, i), e in ref.items()}
    st = C.compare_attention(w, b.out, b.lse, ref)
    print(name, st, "retained", float(gm.mean()))
    C.assert_attention_close(st)
