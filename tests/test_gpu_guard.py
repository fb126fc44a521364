"""Out-of-bounds write checks without a sanitizer: every tensor a call writes is carved out
of one device buffer, with guard regions filled with a byte pattern between and around
them; after the call the guard bytes must be unchanged. This covers every kernel's stores
(reorder, unreorder, the mask builder's kernels and workspace, the scheduler, attention
output, LSE and its workspace) on ragged, one-tile and degenerate grids. Reads need no such
check: the attention kernel reads through TMA, whose tensor maps bound every access, and
the other kernels' loads are indexed by the same arithmetic that these stores share.
"""
import math

import numpy as np
import pytest
import torch

import _cases as C
from bsa_synth import Workload, generate_difficulty, generate_qkv

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes of pattern before, between and after the tensors
PATTERN = 0xA5


class Carved:
    """Tensors carved from one guarded buffer (256-byte aligned, contiguous)."""

    def __init__(self, specs):
        sizes = [math.prod(shape) * torch.empty((), dtype=dt).element_size() for shape, dt in specs]
        offs, off = [], GUARD
        for n in sizes:
            offs.append(off)
            off = (off + n + GUARD + 255) // 256 * 256
        self.buf = torch.full((off + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.views = [self.buf[o:o + n].view(dt).view(shape)
                      for o, n, (shape, dt) in zip(offs, sizes, specs)]
        self.spans = [(o, o + n) for o, n in zip(offs, sizes)]

    def guards_intact(self) -> bool:
        host = self.buf.cpu().numpy()
        keep = np.ones(host.size, dtype=bool)
        for a, b in self.spans:
            keep[a:b] = False
        return bool(np.all(host[keep] == PATTERN))


def _whole_path(w: Workload, token: bool = False):
    import block_sparse_attention_major_b200 as bsa
    q, k, v = generate_qkv(w)
    diff = generate_difficulty(w)
    g = C.geometry(w)
    p = C.params(w)
    tiled = (g.B, g.H, g.NT, 64, g.d)
    raster = (g.B, g.N, g.H, g.d)
    pooled = (g.B, g.H, g.NT, g.d)
    c = Carved([(raster, torch.bfloat16)] * 3 + [(tiled, torch.bfloat16)] * 3 +
               [((g.B, g.NT), torch.float32), ((g.B, g.H, g.NT, g.NW), torch.int32),
                ((g.B, g.H, g.NT), torch.int32), (raster, torch.bfloat16), ((g.B, g.H, g.N), torch.float32),
                ((bsa.workspace_bytes(g),), torch.uint8), (raster, torch.bfloat16),
                (pooled, torch.float32), (pooled, torch.float32)])
    qd, kd, vd, qt, kt, vt, dd, mask, cnt, out, lse, ws, back, qbar, kbar = c.views
    for dst, src in ((qd, q), (kd, k), (vd, v), (dd, diff)):
        dst.copy_(src)
    ws.zero_()
    # both mask paths: from the tile-major tensors, then from the fused reorder's means
    for x, xt in ((qd, qt), (kd, kt), (vd, vt)):
        bsa.reorder(g, x, xt)
    bsa.build_mask(g, p, qt, kt, dd, mask, cnt, ws)
    bsa.reorder_pool(g, qd, qt, qbar)
    bsa.reorder_pool(g, kd, kt, kbar)
    bsa.build_mask_pooled(g, p, qbar, kbar, dd, mask, cnt, ws)
    if token:
        bsa.sparse_attn_fwd_token(g, qt, kt, vt, mask, cnt, bsa.route_flags(g, ws), w.radius, None, out, lse, ws)
    else:
        bsa.sparse_attn_fwd(g, qt, kt, vt, mask, cnt, None, out, lse, ws)
    bsa.unreorder(g, vt, back)
    torch.cuda.synchronize()
    assert bsa.read_error(ws) == 0
    assert torch.equal(back, vd)                       # the round trip, through guarded buffers
    assert c.guards_intact(), "a kernel wrote outside its tensor"


@pytest.mark.parametrize("name", ["tiny_ragged", "ragged128", "one_tile", "budget128", "mass128"])
def test_no_writes_outside_tensors(name):
    _whole_path(C.workload(name))


@pytest.mark.parametrize("grid", [(1, 13, 1), (13, 1, 2), (1, 1, 1), (5, 9, 3)])
def test_no_writes_outside_tensors_degenerate_grids(grid):
    T, Hs, Ws = grid
    _whole_path(Workload("guard", B=2, H=2, d=64, T=T, Hs=Hs, Ws=Ws, seed=77, window_kind=1, radius=1,
                         topk=2, dense_fraction=0.3))


def test_no_writes_outside_tensors_token_support():
    _whole_path(C.workload("token128"), token=True)


def test_fixed_scratch_no_writes_outside_tensors():
    import block_sparse_attention_major_b200 as bsa
    w = C.workload("ragged128")
    q, k, v = generate_qkv(w)
    diff = generate_difficulty(w)
    g = C.geometry(w)
    qt, kt, vt = (bsa.reorder(g, x.cuda()) for x in (q, k, v))
    mask, cnt = bsa.build_mask(g, C.params(w), qt, kt, diff.cuda())
    c = Carved([((g.B, g.N, g.H, g.d), torch.bfloat16), ((g.B, g.H, g.N), torch.float32), ((1,), torch.int32)])
    out, lse, err = c.views
    err.zero_()
    bsa.sparse_attn_fwd_fixed_scratch(g, qt, kt, vt, mask, cnt, None, out, lse, kernel_errors=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert c.guards_intact()
