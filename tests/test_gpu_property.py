"""GPU property tests: the whole path against the oracle on random small grids (hypothesis,
derandomised so that every run checks the same examples), ragged and degenerate axes
included (1 to 13 tokens per axis), with random head dimension, batch, heads and mask
rule. Reorder must be bit-exact, masks bit-exact outside rows the oracle flags as near-ties,
attention within the parity tolerances on the rows whose masks agree.
"""
import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import _cases as C
from bsa_synth import Workload, generate_difficulty, generate_qkv
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu

SETTINGS = settings(max_examples=12, deadline=None, derandomize=True)
axis = st.integers(min_value=1, max_value=13)


def _run(w: Workload, forward: bool):
    import block_sparse_attention_major_b200 as bsa
    q, k, v = generate_qkv(w)
    diff = generate_difficulty(w)
    g = C.geometry(w)
    p = C.params(w)
    if forward:
        b = bsa.forward(g, p, q.cuda(), k.cuda(), v.cuda(), diff.cuda())
        qt, mask, ws = b.qt, b.mask, b.ws
    else:
        qt, kt = bsa.reorder(g, q.cuda()), bsa.reorder(g, k.cuda())
        ws = bsa.alloc_workspace(g)
        mask, _ = bsa.build_mask(g, p, qt, kt, diff.cuda(), ws=ws)
        b = None
    torch.cuda.synchronize()
    assert bsa.read_error(ws) == 0
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    assert np.array_equal(qt.view(torch.int16).cpu().numpy(),
                          O.reorder(q.view(torch.int16).numpy(), w.T, w.Hs, w.Ws))
    mref = C.oracle_mask(w, qt64, kt64, diff.numpy())
    gm = C.gpu_mask_bool(mask, g.NT)
    cmp = C.compare_masks(gm, mref)
    assert cmp["n_unflagged"] == 0, cmp
    mref["used"] = C.mask_for_reference(mref["mask"], gm, cmp["diff_rows"])
    return b, mref, cmp, (qt64, kt64, vt64)


@SETTINGS
@given(T=axis, Hs=axis, Ws=axis, d=st.sampled_from([64, 128]), B=st.integers(1, 2), H=st.integers(1, 2),
       kind=st.sampled_from([0, 1]), radius=st.integers(0, 3), topk=st.integers(0, 5),
       rho=st.sampled_from([0.0, 0.3]), seed=st.integers(0, 2**16))
def test_forward_matches_oracle_on_random_grids(T, Hs, Ws, d, B, H, kind, radius, topk, rho, seed):
    w = Workload("gpu_property", B=B, H=H, d=d, T=T, Hs=Hs, Ws=Ws, seed=seed, window_kind=kind,
                 radius=radius, topk=topk, dense_fraction=rho)
    b, mref, cmp, (qt64, kt64, vt64) = _run(w, forward=True)
    rows = [(bb, h, i) for bb in range(B) for h in range(H) for i in range(w.NT)]
    ref = O.attention_tiles(qt64, kt64, vt64, mref["used"], rows, T=T, Hs=Hs, Ws=Ws)
    st_ = C.compare_attention(w, b.out, b.lse, ref)
    C.assert_attention_close(st_)


@SETTINGS
@given(T=axis, Hs=axis, Ws=axis, rho=st.integers(0, 10), topk=st.integers(0, 4),
       mass=st.booleans(), seed=st.integers(0, 2**16))
def test_token_support_matches_oracle_on_random_grids(T, Hs, Ws, rho, topk, mass, seed):
    w = Workload("gpu_property_token", B=1, H=2, d=64, T=T, Hs=Hs, Ws=Ws, seed=seed, window_kind=2,
                 radius=rho, topk=topk, dense_fraction=0.25, budget_mode=2 if mass else 0,
                 budget_target=0.5 if mass else 0.0)
    b, mref, cmp, (qt64, kt64, vt64) = _run(w, forward=True)
    rows = [(0, h, i) for h in range(w.H) for i in range(w.NT)]
    ref = O.attention_tiles(qt64, kt64, vt64, mref["used"], rows, T=T, Hs=Hs, Ws=Ws, token_rho=rho,
                            window=O.token_window(rho, T, Hs, Ws), dense=mref["dense"])
    st_ = C.compare_attention(w, b.out, b.lse, ref)
    C.assert_attention_close(st_)
