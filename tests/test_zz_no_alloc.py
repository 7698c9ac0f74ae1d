"""The decode entry point that allocates nothing (mea_decode_splitkv_noalloc).

Some callers of this library cannot allocate device memory: a plugin inside a host runtime that
reserved all of its device memory up front and only hands over input/output tensors, or a
serving loop that cannot afford an allocation on every decode step. For them the library keeps
the split-KV partials in a fixed array of its own instead of a caller workspace. These tests call
that entry point through the C ABI, on two calls in a row, and check it against the float64
oracle (the same tolerance as every decode parity test) and against mea_decode_splitkv with a
workspace. They also drive the automatic chunk doubling that keeps large problems inside the
array, and its size limit. The file is named so that pytest collects it last.
"""
import pytest
import torch

import memory_efficient_attention_b200 as mea
import oracle
from memory_efficient_attention_b200 import _lib
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv, randn

pytestmark = pytest.mark.gpu

ATOL, RTOL = 8e-3, 2e-2   # bf16 tolerance used by every parity test
LSE_TOL = 1e-3
SCRATCH = 32 * 1024 * 1024  # MEA_DECODE_NOALLOC_SCRATCH_BYTES


def _case(seed, lk, hq, hkv, d=128, dtype=torch.bfloat16):
    _, k, v = make_qkv([1], lk, hq, hkv, d, dtype, seed)
    q = make_qkv([len(lk)], [1], hq, hkv, d, dtype, seed + 1)[0]
    return q, k, v, cu_seqlens(lk)


def _close(a, b, la, lb, what):
    a, b = a.double().cpu(), b.double().cpu()
    la, lb = la.double().cpu(), lb.double().cpu()
    assert not torch.isnan(a).any(), what
    assert bool(((a - b).abs() <= ATOL + RTOL * b.abs()).all()), f"{what}: out differs"
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin), f"{what}: -inf pattern differs"
    if fin.any():
        assert float((la[fin] - lb[fin]).abs().max()) <= LSE_TOL, f"{what}: lse differs"


def _noalloc(q, k, v, cu, max_k, slopes, scale, split):
    out = torch.full_like(q, float("nan"))
    lse = torch.full((q.shape[1], q.shape[0]), float("nan"), dtype=torch.float32,
                     device=q.device)
    mea.decode_splitkv_noalloc(q, k, v, cu, max_k, out, lse, alibi_slopes=slopes, scale=scale,
                               split_keys=split)
    return out, lse


def test_noalloc_matches_oracle_and_workspace_decode_two_calls_in_a_row():
    cases = [(700, [513, 64, 4000, 1, 0, 2500], 64, 8, 0, True),
             (710, [33, 1500, 128, 9000], 32, 4, 256, False)]
    for call, (seed, lk, hq, hkv, split, alibi) in enumerate(cases):
        q, k, v, cu = _case(seed, lk, hq, hkv)
        slopes = alibi_slope_values(hq) if alibi else None
        qd, kd, vd, cud = q.cuda(), k.cuda(), v.cuda(), cu.cuda()
        sd = slopes.cuda() if alibi else None
        out, lse = _noalloc(qd, kd, vd, cud, max(lk), sd, 0.09, split)
        ref_o, ref_l = mea.decode_splitkv(qd, kd, vd, cud, max(lk), alibi_slopes=sd, scale=0.09,
                                          split_keys=split)
        torch.cuda.synchronize()
        oo, ol = oracle.decode(q, k, v, cu.tolist(), 0.09,
                               None if slopes is None else slopes.double())
        _close(out, oo, lse, ol, f"call {call} vs oracle")
        _close(out, ref_o, lse, ref_l, f"call {call} vs mea_decode_splitkv")
    assert mea.device_error() == 0


def _auto_chunk(n, tk, hq, hkv, d):
    """The library's automatic chunk for mea_decode_splitkv (the workspace size identifies it:
    it falls strictly as the chunk doubles)."""
    ws = mea.decode_workspace_size(n, tk, hq, hkv, d, 0)
    for c in (128, 256, 512, 1024, 2048):
        if mea.decode_workspace_size(n, tk, hq, hkv, d, c) == ws:
            return c
    raise AssertionError("automatic chunk not identified")


def test_noalloc_doubles_its_chunk_to_fit_the_scratch():
    # MQA, 128 query heads, ~1.4M keys: at the automatic chunk the partials exceed the fixed
    # array, so the entry point doubles the chunk (past the 2048 the workspace path ever picks)
    n, per, hq, hkv, d = 12, 131072, 128, 1, 128
    lk = [per] * n
    lk[3] = per - 1000
    lk[5] = 700
    tk = sum(lk)
    chunk = _auto_chunk(n, tk, hq, hkv, d)
    while mea.decode_workspace_size(n, tk, hq, hkv, d, chunk) > SCRATCH:
        chunk *= 2
    assert chunk > 2048
    k = randn((tk, hkv, d), 7101, torch.bfloat16, device="cuda")
    v = randn((tk, hkv, d), 7102, torch.bfloat16, device="cuda")
    q = randn((n, hq, d), 7103, torch.bfloat16, device="cuda")
    cu = cu_seqlens(lk)
    cud = cu.cuda()
    for call in range(2):
        out, lse = _noalloc(q, k, v, cud, max(lk), None, 0.088, 0)
        ref_o, ref_l = mea.decode_splitkv(q, k, v, cud, max(lk), scale=0.088, split_keys=chunk)
        torch.cuda.synchronize()
        # same chunking, same kernels: identical bits
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l), f"call {call}"
    c = cu.tolist()
    for b in (3, 5):  # a long request and the short one, against the oracle
        ro, rl = oracle.decode(q[b:b + 1].cpu(), k[c[b]:c[b + 1]].cpu(), v[c[b]:c[b + 1]].cpu(),
                               [0, lk[b]], 0.088)
        _close(out[b:b + 1], ro, lse[:, b:b + 1], rl, f"request {b} vs oracle")
    assert mea.device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib.load()
    # 70,000 keys in 64-key chunks: 1,095 partial slots x 64 heads x 129 floats > 32 MiB. The
    # buffers have exactly the sizes the arguments describe, so even if the size check ever
    # came after the launches, every access would stay inside them.
    tk, hq, hkv, d = 70_000, 64, 8, 128
    q = torch.zeros((1, hq, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((tk, hkv, d), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    lse = torch.zeros((hq, 1), dtype=torch.float32, device="cuda")
    cu = torch.tensor([0, tk], dtype=torch.int32, device="cuda")
    assert mea.decode_workspace_size(1, tk, hq, hkv, d, 64) > SCRATCH
    rc = lib.mea_decode_splitkv_noalloc(q.data_ptr(), kv.data_ptr(), kv.data_ptr(),
                                        out.data_ptr(), lse.data_ptr(), cu.data_ptr(), 1, tk, tk,
                                        hq, hkv, d, 0.1, 1, None, 1, 64, None)
    assert rc == _lib.MEA_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.status_string(rc)
    torch.cuda.synchronize()
    assert mea.device_error() == 0
