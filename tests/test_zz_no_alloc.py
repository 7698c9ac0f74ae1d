"""The decode entry point that allocates nothing (mea_decode_splitkv_noalloc).

Some callers of this library cannot allocate device memory: a plugin inside a host runtime that
reserved all of its device memory up front and only hands over input/output tensors, or a
serving loop that cannot afford an allocation on every decode step. For them the library keeps
the split-KV partials in a fixed array of its own instead of a caller workspace. These tests call
that entry point through the C ABI and check it against mea_decode_splitkv (with a workspace) on
two calls in a row, plus its size limit. The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import memory_efficient_attention_b200 as mea
from memory_efficient_attention_b200 import _lib
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv

pytestmark = pytest.mark.gpu

ATOL, RTOL = 8e-3, 2e-2   # bf16 tolerance used by every parity test
LSE_TOL = 1e-3


def _case(seed, lk, hq, hkv, d=128, dtype=torch.bfloat16):
    _, k, v = make_qkv([1], lk, hq, hkv, d, dtype, seed)
    q = make_qkv([len(lk)], [1], hq, hkv, d, dtype, seed + 1)[0]
    return q.cuda(), k.cuda(), v.cuda(), cu_seqlens(lk).cuda()


def _close(a, b, la, lb, what):
    a, b = a.double(), b.double()
    assert not torch.isnan(a).any(), what
    assert bool(((a - b).abs() <= ATOL + RTOL * b.abs()).all()), f"{what}: out differs"
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin), f"{what}: -inf pattern differs"
    assert float((la[fin] - lb[fin]).abs().max()) <= LSE_TOL, f"{what}: lse differs"


def test_noalloc_matches_workspace_decode_two_calls_in_a_row():
    cases = [(700, [513, 64, 4000, 1, 0, 2500], 64, 8, 0, True),
             (710, [33, 1500, 128, 9000], 32, 4, 256, False)]
    for call, (seed, lk, hq, hkv, split, alibi) in enumerate(cases):
        q, k, v, cu = _case(seed, lk, hq, hkv)
        slopes = alibi_slope_values(hq).cuda() if alibi else None
        ref_o, ref_l = mea.decode_splitkv(q, k, v, cu, max(lk), alibi_slopes=slopes, scale=0.09,
                                          split_keys=split)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((hq, len(lk)), float("nan"), dtype=torch.float32, device="cuda")
        mea.decode_splitkv_noalloc(q, k, v, cu, max(lk), out, lse, alibi_slopes=slopes,
                                   scale=0.09, split_keys=split)
        torch.cuda.synchronize()
        _close(out, ref_o, lse, ref_l, f"call {call}")
    assert mea.device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib.load()
    a = 0x10000  # never dereferenced: the size check fails before anything is launched
    # 10M keys in 64-key chunks -> ~156k partial slots x 64 heads x 129 floats >> 32 MiB
    rc = lib.mea_decode_splitkv_noalloc(a, a, a, a, a, a, 1, 10_000_000, 10_000_000, 64, 8, 128,
                                        0.1, 1, None, 1, 64, None)
    assert rc == _lib.MEA_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.status_string(rc)
