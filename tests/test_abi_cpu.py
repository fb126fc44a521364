"""CPU checks of the C ABI: the library loads, exports every symbol the header declares,
and its host-only entry points and argument validation behave as documented. No call here
reaches a CUDA device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_major_b200 import _build
    import block_sparse_attention_major_b200 as bsa
    _build.build()
    return bsa.load_library()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("bsa_reorder", "bsa_unreorder", "bsa_build_mask", "bsa_sparse_attn_fwd",
                 "bsa_workspace_bytes", "bsa_status_string"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.bsa_status_string(0) == b"BSA_OK"
    assert lib.bsa_status_string(1) == b"BSA_ERR_INVALID_ARG"
    assert lib.bsa_status_string(99) == b"BSA_ERR_UNKNOWN"


def test_tile_grid_and_workspace(lib):
    import block_sparse_attention_major_b200 as bsa
    g = bsa.Geometry(1, 12, 128, 21, 30, 52)
    out = [ctypes.c_int() for _ in range(4)]
    assert lib.bsa_tile_grid(ctypes.byref(g.c()), *[ctypes.byref(o) for o in out]) == 0
    assert [o.value for o in out] == [6, 8, 13, 624]
    n = bsa.workspace_bytes(g)
    pooled = 12 * 624 * 128 * 4          # qbar and kbar, fp32
    scores = 12 * 624 * 624 * 4          # pooled scores, fp32, rows padded to 4
    assert n >= 2 * pooled + scores + 256 and n % 256 == 0
    assert n < 2 * pooled + scores + 4 * 1024 * 1024


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(d=0), dict(B=0), dict(H=0), dict(T=0), dict(Ws=-1),
    dict(T=400, Hs=400, Ws=400),                      # more than 4096 tiles
    dict(T=4096, Hs=4096, Ws=4096),                   # token count beyond int range
    dict(T=4097),                                     # more than 4096 per axis
    dict(B=2, H=40000),                               # B*H above the 65535 grid limit
])
def test_invalid_geometry_rejected_on_host(lib, bad):
    import block_sparse_attention_major_b200 as bsa
    base = dict(B=1, H=2, d=64, T=8, Hs=16, Ws=16)
    base.update(bad)
    g = bsa.bsa_geom(base["B"], base["H"], base["d"], base["T"], base["Hs"], base["Ws"])
    assert lib.bsa_workspace_bytes(ctypes.byref(g), None) == 0
    assert lib.bsa_tile_grid(ctypes.byref(g), None, None, None, None) == 1
    buf = ctypes.create_string_buffer(64)
    assert lib.bsa_reorder(ctypes.byref(g), buf, buf, None) == 1
    assert lib.bsa_unreorder(ctypes.byref(g), buf, buf, None) == 1


def test_largest_head_count_accepted_on_host(lib):
    """B*H = 65535 heads of one tile is a valid geometry (the grid limit is inclusive)."""
    import block_sparse_attention_major_b200 as bsa
    g = bsa.bsa_geom(1, 65535, 64, 4, 4, 4)
    nt = ctypes.c_int(0)
    assert lib.bsa_tile_grid(ctypes.byref(g), None, None, None, ctypes.byref(nt)) == 0
    assert nt.value == 1
    assert lib.bsa_workspace_bytes(ctypes.byref(g), None) > 0


def test_null_and_misaligned_pointers_rejected_on_host(lib):
    import block_sparse_attention_major_b200 as bsa
    g = bsa.Geometry(1, 2, 64, 8, 16, 16).c()
    assert lib.bsa_reorder(ctypes.byref(g), None, None, None) == 1
    odd = ctypes.c_void_p(0x1001)
    al = ctypes.c_void_p(0x1000)
    assert lib.bsa_reorder(ctypes.byref(g), odd, al, None) == 1
    p = bsa.MaskParams(0, 1, 1, 0.25).c()
    # missing workspace
    assert lib.bsa_build_mask(ctypes.byref(g), ctypes.byref(p), al, al, al, al, al, None, 0, None) == 2
    # workspace too small
    assert lib.bsa_build_mask(ctypes.byref(g), ctypes.byref(p), al, al, al, al, al,
                              ctypes.c_void_p(0x10000), 16, None) == 2
    assert lib.bsa_sparse_attn_fwd(ctypes.byref(g), al, al, al, al, al, ctypes.c_float(0.125), al,
                                   None, None, 0, None) == 2
    assert lib.bsa_sparse_attn_fwd(ctypes.byref(g), al, al, al, al, al, ctypes.c_float(-1.0), al,
                                   None, ctypes.c_void_p(0x10000), 1 << 30, None) == 1


@pytest.mark.parametrize("bad", [
    dict(dense_fraction=1.5), dict(dense_fraction=-0.1), dict(window_kind=-1), dict(radius=-1),
    dict(topk=-3), dict(budget_mode=2), dict(budget_mode=1, window_kind=0, budget_target=0.1),
    dict(budget_mode=1, window_kind=1, budget_target=0.0),
    dict(budget_mode=3, budget_target=0.5), dict(budget_mode=2, budget_target=1.5),
    dict(budget_mode=2, budget_target=0.5, radius=-1), dict(budget_mode=2, budget_target=0.5, window_kind=3),
    dict(window_kind=2, radius=32768), dict(window_kind=2, radius=-1), dict(window_kind=3),
    dict(budget_mode=1, window_kind=2, budget_target=0.2),
    dict(budget_mode=2, budget_target=0.5, window_kind=2, radius=40000),
])
def test_invalid_mask_params_rejected_on_host(lib, bad):
    import block_sparse_attention_major_b200 as bsa
    g = bsa.Geometry(1, 2, 64, 8, 16, 16).c()
    base = dict(window_kind=0, radius=1, topk=1, dense_fraction=0.25, budget_mode=0,
                budget_target=0.0)
    base.update(bad)
    p = bsa.bsa_mask_params(base["window_kind"], base["radius"], base["topk"],
                            base["dense_fraction"], base["budget_mode"], base["budget_target"])
    al = ctypes.c_void_p(0x1000)
    assert lib.bsa_build_mask(ctypes.byref(g), ctypes.byref(p), al, al, al, al, al,
                              ctypes.c_void_p(0x10000), 1 << 30, None) == 1


def test_token_attention_rejects_bad_arguments_on_host(lib):
    """Null route flags and radii outside [0, 32767] are refused before any device call."""
    import block_sparse_attention_major_b200 as bsa
    g = bsa.Geometry(1, 2, 64, 8, 16, 16).c()
    al = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x10000)
    for dense, rho in ((None, 6), (al, -1), (al, 32768)):
        assert lib.bsa_sparse_attn_fwd_token(ctypes.byref(g), al, al, al, al, al, dense, rho,
                                             ctypes.c_float(0.125), al, None, ws, 1 << 30, None) == 1
    bad = bsa.Geometry(1, 2, 96, 8, 16, 16).c()
    assert lib.bsa_sparse_attn_fwd_token(ctypes.byref(bad), al, al, al, al, al, al, 6,
                                         ctypes.c_float(0.125), al, None, ws, 1 << 30, None) == 1


def test_route_flags_offset(lib):
    """The route flags sit inside the workspace, after the pooled Q and K, and a flags
    region of B*NQT bytes fits before the workspace ends."""
    import block_sparse_attention_major_b200 as bsa
    g = bsa.Geometry(2, 3, 128, 7, 13, 10)
    off = lib.bsa_route_flags_offset(ctypes.byref(g.c()))
    pooled = g.B * g.H * g.NT * g.d * 4
    assert off >= 256 + 2 * pooled and off % 256 == 0
    assert off + g.B * g.NT <= lib.bsa_workspace_bytes(ctypes.byref(g.c()), None)
    assert lib.bsa_route_flags_offset(ctypes.byref(bsa.Geometry(1, 1, 96, 4, 4, 4).c())) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    import block_sparse_attention_major_b200 as bsa
    with pytest.raises(RuntimeError):
        bsa.load_library(str(tmp_path / "missing.so"))


def test_binding_refuses_mixed_devices():
    """Tensors of one call must share a device: the library launches on the current device
    with the pointers it is given, so a tensor elsewhere is refused before any call."""
    import torch
    import block_sparse_attention_major_b200 as bsa
    a = torch.zeros(4)
    m = torch.empty(4, device="meta")
    assert bsa._device_of(a, None, a) == torch.device("cpu")
    with pytest.raises(ValueError, match="share one device"):
        bsa._device_of(a, m)
    with pytest.raises(ValueError, match="share one device"):
        bsa._device_of(None, None)


@pytest.mark.parametrize("ws", ["host", "float", "2d", "strided"])
def test_binding_refuses_a_bad_workspace(ws):
    """The workspace must be device memory: a host tensor, or one of another dtype or shape,
    is refused by the binding before the library sees its pointer."""
    import torch
    import block_sparse_attention_major_b200 as bsa
    t = {"host": torch.zeros(1024, dtype=torch.uint8),
         "float": torch.zeros(256, dtype=torch.float32),
         "2d": torch.zeros(4, 256, dtype=torch.uint8),
         "strided": torch.zeros(2048, dtype=torch.uint8)[::2]}[ws]
    with pytest.raises(ValueError, match="ws must be"):
        bsa._need_ws(t)
    with pytest.raises(ValueError, match="ws must be"):
        bsa.clear_error(t)


def test_binding_wrappers_marshal_every_entry_point(monkeypatch):
    """Every wrapper, driven on the CPU through a fake library and a fake current stream:
    each reaches its C entry point once, with the stream of the tensors' device and the
    pointers of the tensors it was given."""
    import contextlib
    import torch
    import block_sparse_attention_major_b200 as bsa

    calls = []

    class FakeLib:
        def __getattr__(self, name):
            def f(*args):
                calls.append((name, args))
                return 0
            return f

    class FakeStream:
        device = torch.device("cpu")
        cuda_stream = 0x5000

    monkeypatch.setattr(bsa, "load_library", lambda path=None: FakeLib())
    monkeypatch.setattr(bsa, "_need", lambda t, dtype, shape, name: None)
    monkeypatch.setattr(bsa, "_need_ws", lambda ws: None)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda d=None: FakeStream())
    g = bsa.Geometry(1, 2, 64, 8, 16, 16)
    p = bsa.MaskParams(1, 2, 3, 0.25, 0, 0.0)
    tiled = torch.zeros(g.B, g.H, g.NT, 64, g.d, dtype=torch.bfloat16)
    raster = torch.zeros(g.B, g.N, g.H, g.d, dtype=torch.bfloat16)
    mask = torch.zeros(g.B, g.H, g.NT, g.NW, dtype=torch.int32)
    cnt = torch.zeros(g.B, g.H, g.NT, dtype=torch.int32)
    diff = torch.zeros(g.B, g.NT)
    ws = torch.zeros(4096, dtype=torch.uint8)
    out = torch.zeros_like(raster)
    lse = torch.zeros(g.B, g.H, g.N)
    err = torch.zeros(1, dtype=torch.int32)

    bsa.reorder(g, raster, tiled)
    bsa.unreorder(g, tiled, raster)
    bsa.build_mask(g, p, tiled, tiled, diff, mask, cnt, ws)
    bsa.sparse_attn_fwd(g, tiled, tiled, tiled, mask, cnt, None, out, lse, ws)
    bsa.sparse_attn_fwd_fixed_scratch(g, tiled, tiled, tiled, mask, cnt, None, out, lse, err)
    bsa.clear_error(ws)
    bsa.selftest_bounded_wait(err)
    pooled = torch.zeros(g.B, g.H, g.NT, g.d)
    bsa.reorder_pool(g, raster, tiled, pooled)
    bsa.build_mask_pooled(g, p, pooled, pooled, diff, mask, cnt, ws)
    dense = torch.zeros(g.B, g.NT, dtype=torch.uint8)
    bsa.sparse_attn_fwd_token(g, tiled, tiled, tiled, mask, cnt, dense, 6, None, out, lse, ws)
    names = [c[0] for c in calls]
    assert names == ["bsa_reorder", "bsa_unreorder", "bsa_build_mask", "bsa_sparse_attn_fwd",
                     "bsa_sparse_attn_fwd_fixed_scratch", "bsa_clear_error", "bsa_selftest_bounded_wait",
                     "bsa_reorder_pool", "bsa_build_mask_pooled", "bsa_sparse_attn_fwd_token"]
    tk = calls[9][1]
    assert tk[6].value == dense.data_ptr() and tk[7].value == 6 and abs(tk[8].value - 0.125) < 1e-7
    assert [a.value for a in (tk[9], tk[10], tk[11])] == [out.data_ptr(), lse.data_ptr(), ws.data_ptr()]
    assert [a.value for a in calls[7][1][1:4]] == [raster.data_ptr(), tiled.data_ptr(), pooled.data_ptr()]
    assert [a.value for a in calls[8][1][2:8]] == [pooled.data_ptr(), pooled.data_ptr(), diff.data_ptr(),
                                                  mask.data_ptr(), cnt.data_ptr(), ws.data_ptr()]
    for name, args in calls:
        assert args[-1].value == FakeStream.cuda_stream, name
    ptr = lambda t: t.data_ptr()
    assert [a.value for a in calls[0][1][1:3]] == [ptr(raster), ptr(tiled)]
    assert [a.value for a in calls[1][1][1:3]] == [ptr(tiled), ptr(raster)]
    bm = calls[2][1]
    assert [a.value for a in bm[2:8]] == [ptr(tiled), ptr(tiled), ptr(diff), ptr(mask), ptr(cnt), ptr(ws)]
    assert bm[8].value == ws.numel()
    fw = calls[3][1]
    assert abs(fw[6].value - 0.125) < 1e-7                 # 1/sqrt(64)
    assert [a.value for a in (fw[7], fw[8], fw[9])] == [ptr(out), ptr(lse), ptr(ws)]
    assert calls[4][1][9].value == ptr(err)

    # a tensor of another device in the same call is refused before the library is called
    calls.clear()
    with pytest.raises(ValueError, match="share one device"):
        bsa.sparse_attn_fwd(g, tiled, tiled, tiled.to("meta"), mask, cnt, None, out, lse, ws)
    assert calls == []

    # so is a stream of another device
    class OtherStream(FakeStream):
        device = torch.device("meta")
    with pytest.raises(ValueError, match="stream is on"):
        bsa.reorder(g, raster, tiled, stream=OtherStream())
    assert calls == []


def test_forward_mask_reuse_skips_the_build(monkeypatch):
    """forward(rebuild_mask=False) reorders and attends through the buffers' mask without
    calling the mask builder; without earlier buffers it refuses."""
    import contextlib
    import types
    import torch
    import block_sparse_attention_major_b200 as bsa

    calls = []

    class FakeLib:
        def __getattr__(self, name):
            return lambda *args: calls.append(name) or 0

    class FakeStream:
        device = torch.device("cpu")
        cuda_stream = 0x5000

    monkeypatch.setattr(bsa, "load_library", lambda path=None: FakeLib())
    monkeypatch.setattr(bsa, "_need", lambda t, dtype, shape, name: None)
    monkeypatch.setattr(bsa, "_need_ws", lambda ws: None)
    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "current_stream", lambda d=None: FakeStream())
    g = bsa.Geometry(1, 2, 64, 8, 16, 16)
    p = bsa.MaskParams(1, 1, 2, 0.25)
    t = lambda *shape, dt=torch.bfloat16: torch.zeros(*shape, dtype=dt)
    b = types.SimpleNamespace(qt=t(1, 2, g.NT, 64, 64), kt=t(1, 2, g.NT, 64, 64), vt=t(1, 2, g.NT, 64, 64),
                              qbar=t(1, 2, g.NT, 64, dt=torch.float32), kbar=t(1, 2, g.NT, 64, dt=torch.float32),
                              mask=t(1, 2, g.NT, g.NW, dt=torch.int32), kv_count=t(1, 2, g.NT, dt=torch.int32),
                              out=t(1, g.N, 2, 64), lse=t(1, 2, g.N, dt=torch.float32),
                              ws=t(4096, dt=torch.uint8))
    x = t(1, g.N, 2, 64)
    d = t(1, g.NT, dt=torch.float32)
    bsa.forward(g, p, x, x, x, d, bufs=b)
    assert calls == ["bsa_reorder_pool"] * 2 + ["bsa_reorder", "bsa_build_mask_pooled", "bsa_sparse_attn_fwd"]
    calls.clear()
    bsa.forward(g, p, x, x, x, d, bufs=b, rebuild_mask=False)
    assert calls == ["bsa_reorder"] * 3 + ["bsa_sparse_attn_fwd"]
    assert bsa.launches_per_forward(p, rebuild_mask=False) == bsa.launches_per_forward(p) - 3
    with pytest.raises(ValueError, match="earlier call"):
        bsa.forward(g, p, x, x, x, d, rebuild_mask=False)


def test_launch_counter_starts_at_zero_without_launches(lib):
    assert lib.bsa_launch_count() == 0


def test_selftest_arguments_rejected_on_host(lib):
    al = ctypes.c_void_p(0x1000)
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(1000), None, None) == 1
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(1000), ctypes.c_void_p(0x1002), None) == 1
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(0), al, None) == 1
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(5_000_000_000), al, None) == 1
