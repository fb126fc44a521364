"""Failure handling on the GPU without a fault: a bounded wait that nothing completes gives
up, reports through the error word, and leaves the CUDA context usable."""
import time

import pytest
import torch

import _cases as C

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    import block_sparse_attention_major_b200 as bsa
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    bsa.selftest_bounded_wait(err, limit_cycles=20_000_000)        # about 10 ms of SM clock
    torch.cuda.synchronize()
    assert int(err.item()) & bsa.KERR_WAIT_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    # the same context runs the whole path afterwards, error-free
    w, q, k, v, diff = C.inputs("tiny_ragged")
    g = C.geometry(w)
    b = bsa.forward(g, C.params(w), q.cuda(), k.cuda(), v.cuda(), diff.cuda())
    torch.cuda.synchronize()
    assert bsa.read_error(b.ws) == 0
    assert torch.isfinite(b.out.float()).all()
