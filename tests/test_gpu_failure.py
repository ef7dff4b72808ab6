"""Bounded device waits (the one every grid barrier of the library uses): a wait on a
flag that nothing sets runs out after its limit, the timeout status reaches the host
through the error word, and the context stays usable. Nothing faults or hangs."""
import time

import pytest
import torch

import lookahead_sparse_kv_lsa_b200 as lsa

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports(cuda_ok):
    dev = torch.device("cuda")
    flag = torch.zeros(1, dtype=torch.int32, device=dev)   # nothing ever sets it
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    lsa.lsa_wait_selftest(flag, 1, 50_000_000, err)        # 50 ms
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(err.item()) == lsa._lib.DEVERR_TIMEOUT
    assert 0.04 <= dt < 5.0, dt
    # the context is still usable
    x = torch.arange(1024, device=dev, dtype=torch.float32)
    assert float((2 * x).sum().item()) == 2.0 * sum(range(1024))


def test_wait_on_a_set_flag_returns_at_once(cuda_ok):
    dev = torch.device("cuda")
    flag = torch.full((1,), 3, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    lsa.lsa_wait_selftest(flag, 3, 1_000_000_000, err)     # would allow 1 s
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert time.perf_counter() - t0 < 0.5
