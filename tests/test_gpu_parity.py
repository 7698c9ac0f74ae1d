"""GPU parity: the CUDA path (through the C ABI) against the float64 CPU oracle.

Tolerances: |out - ref| <= 2e-3 + 1e-2 |ref| for fp16 and 8e-3 + 2e-2 |ref| for bf16; lse within
1e-3 absolute; -inf lse (no admissible key) must match exactly. Output buffers are pre-filled
with NaN and followed by a canary region, so rows the kernel never writes and writes past the
end are both caught.
"""
import math

import pytest
import torch

import memory_efficient_attention_b200 as mea
import oracle
from mea_workloads import (alibi_slope_values, cu_seqlens, make_qkv, randn, sample_rows,
                           workload)

pytestmark = pytest.mark.gpu

TOL = {torch.float16: (2e-3, 1e-2), torch.bfloat16: (8e-3, 2e-2)}
LSE_TOL = 1e-3
CANARY = 4096


def _alloc_out(shape, dtype):
    n = math.prod(shape)
    buf = torch.full((n + CANARY,), float("nan"), dtype=dtype, device="cuda")
    buf[n:] = 7.0
    return buf, buf[:n].view(shape)


def _alloc_lse(shape):
    n = math.prod(shape)
    buf = torch.full((n + CANARY,), float("nan"), dtype=torch.float32, device="cuda")
    buf[n:] = 7.0
    return buf, buf[:n].view(shape)


def _check_canary(buf, n):
    tail = buf[n:].float()
    assert torch.all(tail == 7.0), "write past the end of an output buffer"


def assert_close(out, ref, lse=None, lse_ref=None, dtype=torch.bfloat16, what=""):
    atol, rtol = TOL[dtype]
    o = out.double().cpu()
    r = ref.double()
    assert not torch.isnan(o).any(), f"{what}: NaN in output (unwritten rows?)"
    err = (o - r).abs()
    bound = atol + rtol * r.abs()
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.numel()} elements out of "
                           f"tolerance, max excess {float((err - bound).max()):.3e}")
    if lse is not None:
        l = lse.double().cpu()
        lr = lse_ref.double()
        inf_ref = torch.isinf(lr)
        assert torch.equal(torch.isinf(l), inf_ref), f"{what}: -inf pattern of lse differs"
        if (~inf_ref).any():
            d = (l[~inf_ref] - lr[~inf_ref]).abs().max()
            assert float(d) <= LSE_TOL, f"{what}: lse max err {float(d):.3e}"


def run_packed(seqlens_q, seqlens_k, hq, hkv, d, dtype, causal, alibi, scale, seed,
               max_seqlen_q=None):
    q, k, v = make_qkv(seqlens_q, seqlens_k, hq, hkv, d, dtype, seed)
    cu_q, cu_k = cu_seqlens(seqlens_q), cu_seqlens(seqlens_k)
    slopes = alibi_slope_values(hq) if alibi else None
    tq = q.shape[0]
    obuf, out = _alloc_out((tq, hq, d), dtype)
    lbuf, lse = _alloc_lse((hq, tq))
    mea.attention_packed(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(),
                         max_seqlen_q if max_seqlen_q is not None else max(seqlens_q),
                         causal=causal, alibi_slopes=None if slopes is None else slopes.cuda(),
                         scale=scale, out=out, lse=lse)
    torch.cuda.synchronize()
    _check_canary(obuf, out.numel())
    _check_canary(lbuf, lse.numel())
    return (q, k, v, cu_q, cu_k, slopes), out, lse


def check_packed(seqlens_q, seqlens_k, hq, hkv, d, dtype, causal, alibi, scale, seed, **kw):
    (q, k, v, cu_q, cu_k, slopes), out, lse = run_packed(seqlens_q, seqlens_k, hq, hkv, d, dtype,
                                                         causal, alibi, scale, seed, **kw)
    ref, lref = oracle.attention(q, k, v, cu_q.tolist(), cu_k.tolist(), scale, causal,
                                 None if slopes is None else slopes.double())
    assert_close(out, ref, lse, lref, dtype,
                 f"q{seqlens_q[:6]} k{seqlens_k[:6]} H{hq}/{hkv} D{d} {dtype} causal={causal} "
                 f"alibi={alibi}")


# ------------------------------------------------------------------ the five workloads

@pytest.mark.parametrize("causal", [False, True])
def test_workload0_packed_varlen(causal):
    w = workload(0)
    check_packed(w.seqlens_q, w.seqlens_k, 8, 8, 64, w.dtype, causal, False, w.scale, w.seed)


@pytest.mark.parametrize("causal", [False, True])
def test_workload1_bmghk(causal):
    w = workload(1)
    b, m, g, hq, kd = w.extra["bmghk"]
    qg = randn((b, m, g, hq, kd), w.seed * 3, w.dtype)
    kg = randn((b, m, g, 1, kd), w.seed * 3 + 1, w.dtype)
    vg = randn((b, m, g, 1, kd), w.seed * 3 + 2, w.dtype)
    bias = mea.LowerTriangularMask() if causal else None
    out = mea.memory_efficient_attention(qg.cuda(), kg.cuda(), vg.cuda(), attn_bias=bias,
                                         scale=w.scale)
    torch.cuda.synchronize()
    assert tuple(out.shape) == (b, m, g, hq, kd)
    ref, _ = oracle.attention(qg.reshape(b * m, g * hq, kd), kg.reshape(b * m, g, kd),
                              vg.reshape(b * m, g, kd), [0, m, 2 * m], [0, m, 2 * m], w.scale,
                              causal)
    assert_close(out.reshape(b * m, g * hq, kd), ref, dtype=w.dtype, what="BMGHK")


def test_workload2_packed_causal_gqa_alibi_full():
    w = workload(2)
    assert w.total_q == 32768
    check_packed(w.seqlens_q, w.seqlens_k, 32, 8, 128, w.dtype, True, True, w.scale, w.seed)


def test_head_dim_256_long_causal_sampled():
    # the 16384-token causal prefill at head dim 256 (64/8 heads, scale 1/16), one launch of the
    # 256-wide kernel at the size the bench times, on sampled rows
    w = workload(3)
    (q, k, v, cu_q, cu_k, _), out, lse = run_packed(w.seqlens_q, w.seqlens_k, 64, 8, 256,
                                                    w.dtype, True, False, 1.0 / 16, w.seed + 256)
    rows = sample_rows(w.seed + 256, 256, 64, w.total_q, must_tokens=(0, 1, 127, 128, 16383))
    ro, rl = oracle.attention_rows(q, k, v, cu_q.tolist(), cu_k.tolist(), 1.0 / 16, True, None,
                                   rows)
    got = torch.stack([out[t, h].cpu() for h, t in rows])
    gl = torch.stack([lse[h, t].cpu() for h, t in rows])
    assert_close(got, ro, gl, rl, w.dtype, "head dim 256, 16384 tokens, sampled rows")


def test_workload3_long_causal_sampled():
    w = workload(3)
    (q, k, v, cu_q, cu_k, _), out, lse = run_packed(w.seqlens_q, w.seqlens_k, 64, 8, 128,
                                                    w.dtype, True, False, w.scale, w.seed)
    rows = sample_rows(w.seed, 512, 64, w.total_q, must_tokens=(0, 15, 16, 127, 128, 16383))
    ro, rl = oracle.attention_rows(q, k, v, cu_q.tolist(), cu_k.tolist(), w.scale, True, None,
                                   rows)
    got = torch.stack([out[t, h].cpu() for h, t in rows])
    gl = torch.stack([lse[h, t].cpu() for h, t in rows])
    assert_close(got, ro, gl, rl, w.dtype, "workload 3 sampled rows")


def test_workload4_decode_sampled():
    w = workload(4)
    hq, hkv, d = 64, 8, 128
    tk = w.total_k
    k = randn((tk, hkv, d), w.seed * 3 + 1, w.dtype, device="cuda")
    v = randn((tk, hkv, d), w.seed * 3 + 2, w.dtype, device="cuda")
    q = randn((len(w.seqlens_k), hq, d), w.seed * 3, w.dtype, device="cuda")
    cu_k = cu_seqlens(w.seqlens_k)
    out, lse = mea.decode_splitkv(q, k, v, cu_k.cuda(), max(w.seqlens_k), scale=w.scale)
    torch.cuda.synchronize()
    # oracle on a seeded sample of requests (all their heads), copied back to the host
    import numpy as np
    rng = np.random.default_rng(w.seed)
    reqs = set(int(x) for x in rng.choice(len(w.seqlens_k), 8, replace=False))
    # always the longest request (the most chunks) and the shortest one
    reqs |= {int(np.argmax(w.seqlens_k)), int(np.argmin(w.seqlens_k))}
    reqs = sorted(reqs)
    for b in reqs:
        a, e = int(cu_k[b]), int(cu_k[b + 1])
        ro, rl = oracle.decode(q[b:b + 1].cpu(), k[a:e].cpu(), v[a:e].cpu(), [0, e - a], w.scale)
        assert_close(out[b:b + 1], ro, lse[:, b:b + 1], rl, w.dtype, f"decode request {b}")


# ------------------------------------------------------------------ edge cases, forward

@pytest.mark.parametrize("lens", [[1], [127], [128], [129], [1, 127, 128, 129, 2, 255, 257],
                                  [300, 5, 640]])
@pytest.mark.parametrize("causal", [False, True])
def test_tile_edges(lens, causal):
    check_packed(lens, lens, 4, 4, 64, torch.float16, causal, False, 0.125, 11 + sum(lens))


@pytest.mark.parametrize("hq,hkv", [(1, 1), (2, 1), (4, 1), (8, 1), (16, 2), (8, 8), (32, 2),
                                    (6, 2), (12, 4), (3, 1), (64, 1), (128, 1), (256, 2)])
def test_gqa_packing(hq, hkv):
    lens = [70, 200, 33]
    check_packed(lens, lens, hq, hkv, 64, torch.bfloat16, True, hq <= 32, 0.125, 100 + hq)


@pytest.mark.parametrize("d", [32, 64, 96, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal,alibi", [(False, False), (True, False), (True, True),
                                          (False, True)])
def test_dtypes_dims_masks(d, dtype, causal, alibi):
    lens = [190, 1, 64, 385]
    check_packed(lens, lens, 8, 2, d, dtype, causal, alibi, 1.0 / math.sqrt(d), 300 + d)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal,alibi", [(False, False), (True, False), (True, True),
                                          (False, True)])
def test_head_dim_256(dtype, causal, alibi):
    # the 256-wide kernel: one 128-row tile per item, S double-buffered in tensor memory
    lens = [190, 1, 64, 385, 129]
    check_packed(lens, lens, 8, 2, 256, dtype, causal, alibi, 1.0 / 16, 360)


@pytest.mark.parametrize("hq,hkv", [(1, 1), (4, 1), (6, 2), (32, 2), (128, 1)])
def test_head_dim_256_gqa_and_edges(hq, hkv):
    lens = [1, 127, 128, 129, 300, 5]
    check_packed(lens, lens, hq, hkv, 256, torch.bfloat16, True, hq <= 32, 0.07, 370 + hq)


def test_head_dim_256_lq_ne_lk_and_empty():
    lq = [5, 130, 40, 0, 17]
    lk = [300, 140, 10, 9, 0]
    for causal in (False, True):
        check_packed(lq, lk, 8, 4, 256, torch.bfloat16, causal, True, 0.06, 380)


@pytest.mark.parametrize("d", [136, 192, 200, 248])
def test_head_dims_between_128_and_256(d):
    lens = [130, 7, 300]
    check_packed(lens, lens, 8, 2, d, torch.bfloat16, True, True, 1.0 / math.sqrt(d), 390 + d)


def test_head_dim_256_long_segments_many_items():
    # several thousand keys per row: long runs of the S double buffer, rescales of O
    lens = [3000, 2100, 700]
    check_packed(lens, lens, 16, 4, 256, torch.bfloat16, True, True, 0.0625, 395)
    check_packed(lens, lens, 16, 4, 256, torch.float16, True, False, 0.125, 396)


@pytest.mark.parametrize("d", [8, 16, 40, 72, 80, 120])
def test_other_head_dims(d):
    # any multiple of 8 up to 128: the 64- or 128-wide kernel with zero-filled columns
    lens = [130, 7, 300]
    check_packed(lens, lens, 8, 2, d, torch.bfloat16, True, True, 1.0 / math.sqrt(d), 350 + d)
    check_packed(lens, lens, 4, 4, d, torch.float16, False, False, 1.0 / math.sqrt(d), 351 + d)


def test_lq_ne_lk_bottom_right_and_empty():
    # L_q < L_k (prefix in cache), L_q > L_k (first rows see no key), L_k = 0, L_q = 0
    lq = [5, 130, 40, 0, 17]
    lk = [300, 140, 10, 9, 0]
    for causal in (False, True):
        check_packed(lq, lk, 8, 4, 128, torch.bfloat16, causal, True, 0.09, 77)


@pytest.mark.parametrize("n_seqs", [255, 256, 257, 300, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_many_segments(n_seqs, causal):
    # the forward ranks up to 256 segments by length on chip and walks longer lists in segment
    # order; both sides of the limit, with GQA (R = 3) and some empty segments
    g = torch.Generator().manual_seed(n_seqs)
    lens = torch.randint(0, 161, (n_seqs,), generator=g).tolist()
    lens[0] = max(lens[0], 1)
    check_packed(lens, lens, 6, 2, 64, torch.float16, causal, False, 0.125, 900 + n_seqs)


def test_max_seqlen_upper_bound():
    lens = [50, 20]
    check_packed(lens, lens, 4, 2, 64, torch.float16, True, False, 0.125, 5, max_seqlen_q=70)


@pytest.mark.parametrize("max_seqlen_q", [1, 100])
def test_max_seqlen_below_true_maximum_still_complete(max_seqlen_q):
    # max_seqlen_q only sizes the grid: every row is produced from the true lengths
    lens = [700, 3, 260]
    check_packed(lens, lens, 8, 2, 128, torch.bfloat16, True, True, 0.09, 6,
                 max_seqlen_q=max_seqlen_q)


def test_out_16_byte_offset():
    # out 16-byte but not 32-byte aligned: whole tiles still go through TMA stores (which need
    # 16 bytes), partial ones through the 16-byte store path
    lens = [100, 37]
    hq, hkv, d, dtype = 8, 2, 128, torch.bfloat16
    q, k, v = make_qkv(lens, lens, hq, hkv, d, dtype, 31)
    cu = cu_seqlens(lens)
    n = q.numel()
    buf = torch.full((n + 8 + CANARY,), float("nan"), dtype=dtype, device="cuda")
    buf[n + 8:] = 7.0
    out = buf[8:n + 8].view(q.shape)
    assert out.data_ptr() % 32 == 16
    mea.attention_packed(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), cu.cuda(), 100, causal=True,
                         scale=0.09, out=out)
    torch.cuda.synchronize()
    assert torch.isnan(buf[:8].float()).all(), "write before the start of out"
    _check_canary(buf, n + 8)
    ref, _ = oracle.attention(q, k, v, cu.tolist(), cu.tolist(), 0.09, True)
    assert_close(out, ref, dtype=dtype, what="out at a 16-byte offset")


def test_extreme_scores_no_overflow():
    # large scale -> scores far beyond the lazy-rescale threshold; output must stay finite/exact
    lens = [256, 300]
    check_packed(lens, lens, 4, 2, 64, torch.bfloat16, True, False, 2.0, 9)
    check_packed(lens, lens, 4, 2, 64, torch.float16, False, True, 1.5, 10)


def test_packed_equals_per_segment_on_gpu():
    lens = [37, 120, 8, 200]
    (q, k, v, cu_q, cu_k, _), out, lse = run_packed(lens, lens, 8, 8, 64, torch.float16, True,
                                                    False, 0.125, 1)
    c = cu_q.tolist()
    for s in range(len(lens)):
        a, b = c[s], c[s + 1]
        o1, l1 = mea.attention_packed(q[a:b].cuda(), k[a:b].cuda(), v[a:b].cuda(),
                                      torch.tensor([0, b - a], dtype=torch.int32, device="cuda"),
                                      torch.tensor([0, b - a], dtype=torch.int32, device="cuda"),
                                      b - a, causal=True, scale=0.125)
        assert torch.equal(o1, out[a:b]) and torch.equal(l1, lse[:, a:b])


def test_block_diagonal_mask_api_and_split():
    lens = [37, 120, 8, 200]
    q, k, v = make_qkv(lens, lens, 8, 8, 64, torch.float16, 1000)
    for cls, causal in ((mea.BlockDiagonalMask, False), (mea.BlockDiagonalCausalMask, True)):
        bias = cls.from_seqlens(lens)
        out = mea.memory_efficient_attention(q[None].cuda(), k[None].cuda(), v[None].cuda(),
                                             attn_bias=bias, scale=0.125)
        assert tuple(out.shape) == (1, 365, 8, 64)
        parts = bias.split(out)
        assert [tuple(p.shape) for p in parts] == [(1, 37, 8, 64), (1, 120, 8, 64),
                                                   (1, 8, 8, 64), (1, 200, 8, 64)]
        ref, _ = oracle.attention(q, k, v, cu_seqlens(lens).tolist(), cu_seqlens(lens).tolist(),
                                  0.125, causal)
        assert_close(out[0], ref, dtype=torch.float16, what=cls.__name__)


def test_gqa_equals_repeat_interleave_on_gpu():
    lens = [100, 60]
    q, k, v = make_qkv(lens, lens, 16, 4, 128, torch.bfloat16, 12)
    cu = cu_seqlens(lens).cuda()
    o1, l1 = mea.attention_packed(q.cuda(), k.cuda(), v.cuda(), cu, cu, 100, causal=True)
    o2, l2 = mea.attention_packed(q.cuda(), k.repeat_interleave(4, 1).cuda(),
                                  v.repeat_interleave(4, 1).cuda(), cu, cu, 100, causal=True)
    assert_close(o1, o2.double().cpu(), l1, l2.double().cpu(), torch.bfloat16, "gqa vs rep")


# ------------------------------------------------------------------ edge cases, decode

@pytest.mark.parametrize("lk,split", [([1, 64, 65, 0, 200], 64), ([513, 1024, 1025, 7], 0),
                                      ([4000, 3, 129], 128), ([2048], 2048), ([10, 20], 0)])
@pytest.mark.parametrize("hq,hkv", [(64, 8), (8, 8), (32, 1), (12, 2), (16, 1)])
def test_decode_edges(lk, split, hq, hkv):
    d = 128
    dtype = torch.bfloat16
    tk = sum(lk)
    _, k, v = make_qkv([1], lk, hq, hkv, d, dtype, 400 + tk)
    q = make_qkv([len(lk)], [1], hq, hkv, d, dtype, 401 + tk)[0]
    slopes = alibi_slope_values(hq)
    obuf, out = _alloc_out((len(lk), hq, d), dtype)
    lbuf, lse = _alloc_lse((hq, len(lk)))
    mea.decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu_seqlens(lk).cuda(), max(lk),
                       alibi_slopes=slopes.cuda(), scale=0.088, split_keys=split, out=out,
                       lse=lse)
    torch.cuda.synchronize()
    _check_canary(obuf, out.numel())
    _check_canary(lbuf, lse.numel())
    ro, rl = oracle.decode(q, k, v, cu_seqlens(lk).tolist(), 0.088, slopes.double())
    assert_close(out, ro, lse, rl, dtype, f"decode lk={lk} split={split} H{hq}/{hkv}")


@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.float16),
                                     (64, torch.bfloat16), (8, torch.bfloat16),
                                     (40, torch.float16), (96, torch.bfloat16),
                                     (120, torch.bfloat16), (256, torch.bfloat16),
                                     (256, torch.float16), (200, torch.bfloat16)])
def test_decode_dims(d, dtype):
    lk = [300, 1000, 65]
    _, k, v = make_qkv([1], lk, 16, 4, d, dtype, 500)
    q = make_qkv([3], [1], 16, 4, d, dtype, 501)[0]
    out, lse = mea.decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu_seqlens(lk).cuda(), 1000,
                                  scale=1 / math.sqrt(d), split_keys=256)
    torch.cuda.synchronize()
    ro, rl = oracle.decode(q, k, v, cu_seqlens(lk).tolist(), 1 / math.sqrt(d))
    assert_close(out, ro, lse, rl, dtype, f"decode D{d} {dtype}")


@pytest.mark.parametrize("hq,hkv", [(64, 8), (16, 1), (12, 2)])
def test_decode_head_dim_256_edges(hq, hkv):
    lk = [1, 64, 65, 0, 2000, 129]
    _, k, v = make_qkv([1], lk, hq, hkv, 256, torch.bfloat16, 410 + hq)
    q = make_qkv([len(lk)], [1], hq, hkv, 256, torch.bfloat16, 411 + hq)[0]
    slopes = alibi_slope_values(hq)
    obuf, out = _alloc_out((len(lk), hq, 256), torch.bfloat16)
    lbuf, lse = _alloc_lse((hq, len(lk)))
    mea.decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu_seqlens(lk).cuda(), max(lk),
                       alibi_slopes=slopes.cuda(), scale=0.0625, split_keys=128, out=out,
                       lse=lse)
    torch.cuda.synchronize()
    _check_canary(obuf, out.numel())
    _check_canary(lbuf, lse.numel())
    ro, rl = oracle.decode(q, k, v, cu_seqlens(lk).tolist(), 0.0625, slopes.double())
    assert_close(out, ro, lse, rl, torch.bfloat16, f"decode D256 H{hq}/{hkv}")


def test_decode_matches_forward():
    # decode == forward with one query per segment (bottom-right causal)
    lk = [777, 64, 1500]
    _, k, v = make_qkv([1], lk, 32, 8, 128, torch.bfloat16, 600)
    q = make_qkv([3], [1], 32, 8, 128, torch.bfloat16, 601)[0]
    cu_k = cu_seqlens(lk).cuda()
    o1, l1 = mea.decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu_k, 1500, split_keys=256)
    o2, l2 = mea.attention_packed(q.cuda(), k.cuda(), v.cuda(),
                                  torch.arange(4, dtype=torch.int32, device="cuda"), cu_k, 1,
                                  causal=True)
    assert_close(o1, o2.double().cpu(), l1, l2.double().cpu(), torch.bfloat16, "decode vs fwd")


def test_no_device_error_recorded():
    torch.cuda.synchronize()
    assert mea.device_error(clear=True) == 0
