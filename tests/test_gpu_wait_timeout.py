"""Failure detection on the GPU without a fault: every wait inside the kernels is bounded, and a
wait that runs out records a code in the device error word and lets its kernel return.

The library's wait self-test waits on an mbarrier that nothing ever arrives on, so the bound is
what ends it; the tests check the reported code, that the call ends in about the bound, and that
the context stays usable (a forward pass afterwards matches the float64 oracle).
"""
import time

import pytest
import torch

import memory_efficient_attention_b200 as mea
from memory_efficient_attention_b200 import _lib
import oracle
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv

pytestmark = pytest.mark.gpu


def test_completed_wait_reports_nothing():
    mea.device_error(clear=True)
    mea.wait_selftest(timeout_ns=50_000_000, arrive=True)
    torch.cuda.synchronize()
    assert mea.device_error() == 0


def test_wait_on_a_barrier_nothing_completes_times_out_and_reports():
    mea.device_error(clear=True)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    mea.wait_selftest(timeout_ns=200_000_000, arrive=False)   # 0.2 s bound
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert mea.device_error(clear=True) == _lib.MEA_SELFTEST_WAIT_CODE
    assert 0.15 <= took < 5.0, took
    assert mea.device_error() == 0                            # cleared


def test_context_usable_after_a_timed_out_wait():
    mea.wait_selftest(timeout_ns=10_000_000, arrive=False)
    assert mea.device_error(clear=True) == _lib.MEA_SELFTEST_WAIT_CODE
    lens = [130, 77]
    q, k, v = make_qkv(lens, lens, 8, 2, 128, torch.bfloat16, 4242)
    slopes = alibi_slope_values(8)
    cu = cu_seqlens(lens).cuda()
    out, lse = mea.attention_packed(q.cuda(), k.cuda(), v.cuda(), cu, cu, max(lens), causal=True,
                                    alibi_slopes=slopes.cuda(), scale=0.1)
    torch.cuda.synchronize()
    ref, lref = oracle.attention(q, k, v, cu_seqlens(lens).tolist(), cu_seqlens(lens).tolist(),
                                 0.1, True, slopes.double())
    err = (out.cpu().double() - ref).abs() - (8e-3 + 2e-2 * ref.abs())
    assert float(err.max()) <= 0.0
    assert float((lse.cpu().double() - lref).abs().max()) <= 1e-3
    assert mea.device_error() == 0


def test_default_bound_is_used_when_zero_is_passed():
    mea.set_wait_timeout_ns(30_000_000)
    try:
        mea.wait_selftest(timeout_ns=0, arrive=False)
        assert mea.device_error(clear=True) == _lib.MEA_SELFTEST_WAIT_CODE
    finally:
        mea.set_wait_timeout_ns(2_000_000_000)
    assert mea.device_error() == 0
