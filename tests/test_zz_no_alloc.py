"""The attention entry point that allocates nothing (its scratch is the library's own
fixed device array), checked against the workspace entry point through the C ABI.

Who needs it: callers that cannot allocate device memory, for example a plug-in that
receives tensors from a host application which owns all device memory through its own
allocator, or a serving loop that forbids cudaMalloc after start-up because it can block
and synchronise the device. This file is collected last so that a run which stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import _cases as C
from oracle import bsa_oracle as O

pytestmark = pytest.mark.gpu


def _inputs(name):
    import block_sparse_attention_major_b200 as bsa
    w, q, k, v, diff = C.inputs(name)
    g = C.geometry(w)
    qt, kt, vt = (bsa.reorder(g, x.cuda()) for x in (q, k, v))
    mask, cnt = bsa.build_mask(g, C.params(w), qt, kt, diff.cuda())
    return g, qt, kt, vt, mask, cnt


def _identical(a_out, a_lse, b_out, b_lse):
    # both entry points run the same deterministic kernels on the same work list, so their
    # results agree bit for bit
    assert torch.equal(a_out.view(torch.int16), b_out.view(torch.int16))
    assert torch.equal(a_lse.view(torch.int32), b_lse.view(torch.int32))


def test_fixed_scratch_matches_workspace_entry_point_two_calls_in_a_row():
    import block_sparse_attention_major_b200 as bsa
    # two different geometries back to back: the second call must not see the first's
    # leftovers in the shared scratch array
    for name in ("ragged128", "small128"):
        g, qt, kt, vt, mask, cnt = _inputs(name)
        ref_out, ref_lse = bsa.sparse_attn_fwd(g, qt, kt, vt, mask, cnt)
        out = torch.empty_like(ref_out)
        lse = torch.empty_like(ref_lse)
        errs = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        n0 = bsa.launch_count()
        bsa.sparse_attn_fwd_fixed_scratch(g, qt, kt, vt, mask, cnt, out=out, lse=lse, kernel_errors=errs)
        torch.cuda.synchronize()
        assert bsa.launch_count() - n0 == 4
        assert int(errs.item()) == 0
        _identical(out, lse, ref_out, ref_lse)


def test_fixed_scratch_matches_oracle():
    """Directly against the oracle's attention under the same mask, on every row."""
    import block_sparse_attention_major_b200 as bsa
    w, q, k, v, _ = C.inputs("ragged128")
    g, qt, kt, vt, mask, cnt = _inputs("ragged128")
    out, lse = bsa.sparse_attn_fwd_fixed_scratch(g, qt, kt, vt, mask, cnt)
    torch.cuda.synchronize()
    gm = C.gpu_mask_bool(mask, g.NT)
    qt64, kt64, vt64 = (O.reorder(O.to_f64(x), w.T, w.Hs, w.Ws) for x in (q, k, v))
    rows = [(bb, h, i) for bb in range(w.B) for h in range(w.H) for i in range(g.NT)]
    ref = O.attention_tiles(qt64, kt64, vt64, gm, rows, T=w.T, Hs=w.Hs, Ws=w.Ws)
    st = C.compare_attention(w, out, lse, ref)
    print(st)
    C.assert_attention_close(st)


def test_fixed_scratch_repeated_call_is_identical():
    import block_sparse_attention_major_b200 as bsa
    g, qt, kt, vt, mask, cnt = _inputs("ragged128")
    o1, l1 = bsa.sparse_attn_fwd_fixed_scratch(g, qt, kt, vt, mask, cnt)
    o2, l2 = bsa.sparse_attn_fwd_fixed_scratch(g, qt, kt, vt, mask, cnt)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_fixed_scratch_rejects_calls_larger_than_its_array():
    import block_sparse_attention_major_b200 as bsa
    # 40 heads x 4 batch items of 1440 tiles need about 1.85 MB of scratch (> 1 MiB)
    g = bsa.Geometry(4, 40, 128, 21, 45, 80)
    t = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    lib = bsa.load_library()
    st = lib.bsa_sparse_attn_fwd_fixed_scratch(
        __import__("ctypes").byref(g.c()), bsa._ptr(t), bsa._ptr(t), bsa._ptr(t), bsa._ptr(t),
        bsa._ptr(t), __import__("ctypes").c_float(0.088), bsa._ptr(t), None, None, None)
    assert st == bsa.BSA_OK + 2           # BSA_ERR_WORKSPACE, nothing launched
