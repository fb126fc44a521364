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
    dict(dense_fraction=1.5), dict(dense_fraction=-0.1), dict(window_kind=2), dict(radius=-1),
    dict(topk=-3), dict(budget_mode=2), dict(budget_mode=1, window_kind=0, budget_target=0.1),
    dict(budget_mode=1, window_kind=1, budget_target=0.0),
    dict(budget_mode=3, budget_target=0.5), dict(budget_mode=2, budget_target=1.5),
    dict(budget_mode=2, budget_target=0.5, radius=-1), dict(budget_mode=2, budget_target=0.5, window_kind=2),
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


def test_binding_fails_loudly_without_library(tmp_path):
    import block_sparse_attention_major_b200 as bsa
    with pytest.raises(RuntimeError):
        bsa.load_library(str(tmp_path / "missing.so"))


def test_launch_counter_starts_at_zero_without_launches(lib):
    assert lib.bsa_launch_count() == 0


def test_selftest_arguments_rejected_on_host(lib):
    al = ctypes.c_void_p(0x1000)
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(1000), None, None) == 1
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(1000), ctypes.c_void_p(0x1002), None) == 1
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(0), al, None) == 1
    assert lib.bsa_selftest_bounded_wait(ctypes.c_longlong(5_000_000_000), al, None) == 1
