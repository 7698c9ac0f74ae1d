"""GPU parity of the FP8 forward (mea_forward_fp8 through the C ABI) against the float64 oracle.

Inputs: seeded N(0,1) values divided by their descale and rounded to e4m3; the oracle is the
attention of the decoded values (oracle.e4m3_decode, pinned to the format definition) times the
descales, in float64.

Tolerance, from the arithmetic: the scores are exact products of e4m3 values summed in fp32;
the only rounding of consequence is P to e4m3 before P V (relative error <= 2^-4 for normal
values, absolute <= 2^-10 for subnormals in the kernel's units, which are never smaller than the
row-max-normalised ones), then out to bf16/f16. Per element, with pi the oracle's softmax
probabilities of the row:
    |out - ref| <= sum_j max(2^-4 pi_ij, 2^-10 max_j pi_ij) |v_j| + 2^-8 |ref| + 1e-5,
and |lse - lse_ref| <= 1e-3 (it uses the fp32 P).
"""
import math

import pytest
import torch

import memory_efficient_attention_b200 as mea
import oracle
from mea_workloads import alibi_slope_values, cu_seqlens, randn, workload

pytestmark = pytest.mark.gpu

QD, KD, VD = 0.5, 0.25, 2.0   # per-tensor descales


def _quantized(shape, seed, descale):
    x = randn(shape, seed, torch.float32) / descale
    return x.to(torch.float8_e4m3fn)


def _run(seqlens, hq, hkv, causal, alibi, scale, seed, out_dtype=torch.bfloat16, d=128):
    """The kernel on seeded e4m3 inputs; returns the host e4m3 codes, the slopes and out, lse."""
    tq = sum(seqlens)
    q8 = _quantized((tq, hq, d), seed, QD)
    k8 = _quantized((tq, hkv, d), seed + 1, KD)
    v8 = _quantized((tq, hkv, d), seed + 2, VD)
    slopes = alibi_slope_values(hq) if alibi else None
    cu = cu_seqlens(seqlens)
    out, lse = mea.attention_packed_fp8(q8.cuda(), k8.cuda(), v8.cuda(), cu.cuda(), cu.cuda(),
                                        max(seqlens), causal=causal,
                                        alibi_slopes=None if slopes is None else slopes.cuda(),
                                        scale=scale, q_descale=QD, k_descale=KD, v_descale=VD,
                                        out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert mea.device_error() == 0
    return (q8, k8, v8, slopes, cu), out, lse


def _check(q8, k8, v8, slopes, seqlens, scale, causal, out, lse):
    """out [T, Hq, D] / lse [Hq, T] (host or device) of the given e4m3 codes against the oracle
    of the decoded values, with the bound of the module docstring."""
    hq, hkv = q8.shape[1], k8.shape[1]
    q = oracle.e4m3_decode(q8.view(torch.uint8)) * QD
    k = oracle.e4m3_decode(k8.view(torch.uint8)) * KD
    v = oracle.e4m3_decode(v8.view(torch.uint8)) * VD
    c = cu_seqlens(seqlens).tolist()
    sl = None if slopes is None else slopes.double()
    ref, lref = oracle.attention(q, k, v, c, c, scale, causal, sl)
    probs = oracle.attention_probs(q, k, v, c, c, scale, causal, sl)
    r = hq // hkv
    bound = torch.zeros_like(ref)
    for s, pr in enumerate(probs):            # pr [Hq, L, L]
        if pr.numel() == 0:
            continue
        pmax = pr.amax(dim=-1, keepdim=True)
        w = torch.maximum(2.0 ** -4 * pr, 2.0 ** -10 * pmax)
        for h in range(hq):
            va = v[c[s]:c[s + 1], h // r].abs()
            bound[c[s]:c[s + 1], h] = w[h] @ va
    bound = bound + 2.0 ** -8 * ref.abs() + 1e-5
    o = out.cpu().double()
    assert torch.isfinite(o).all()
    err = (o - ref).abs()
    worst = float((err - bound).max())
    assert worst <= 0.0, f"max err {float(err.max()):.3e}, exceeds the bound by {worst:.3e}"
    fin = torch.isfinite(lref)
    lg = lse.cpu().double()
    assert torch.equal(torch.isfinite(lg), fin)
    assert float((lg[fin] - lref[fin]).abs().max()) <= 1e-3
    return float(err.max()), float((err / bound).max())


def _case(seqlens, hq, hkv, causal, alibi, scale, seed, out_dtype=torch.bfloat16, d=128):
    (q8, k8, v8, slopes, _), out, lse = _run(seqlens, hq, hkv, causal, alibi, scale, seed,
                                             out_dtype, d)
    return _check(q8, k8, v8, slopes, seqlens, scale, causal, out, lse)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("alibi", [False, True])
def test_fp8_packed_varlen(causal, alibi):
    _case([37, 120, 8, 200], 8, 2, causal, alibi, 1 / math.sqrt(128), 1500)


@pytest.mark.parametrize("hq,hkv", [(32, 8), (64, 8), (8, 8), (6, 2)])
def test_fp8_gqa_packing(hq, hkv):
    _case([130, 77, 300], hq, hkv, True, True, 0.088, 1510 + hq)


@pytest.mark.parametrize("lens", [[1], [128], [129], [255, 1, 257]])
def test_fp8_tile_edges(lens):
    _case(lens, 8, 4, True, False, 0.1, 1520 + sum(lens))


def test_fp8_half_output_and_longer_segments():
    _case([1000, 700], 8, 2, True, True, 1 / math.sqrt(128), 1530, out_dtype=torch.float16)


@pytest.mark.parametrize("d", [16, 64, 96])
def test_fp8_other_head_dims(d):
    _case([130, 77, 300], 8, 2, True, True, 1 / math.sqrt(d), 1540 + d, d=d)


def test_fp8_rejects_other_head_dims_and_dtypes():
    x = torch.zeros((4, 2, 72), dtype=torch.float8_e4m3fn, device="cuda")
    cu = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    with pytest.raises(mea.MeaError):
        mea.attention_packed_fp8(x, x, x, cu, cu, 4)
    y = torch.zeros((4, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mea.MeaError):
        mea.attention_packed_fp8(y, y, y, cu, cu, 4)


def test_fp8_packed_workload_full_size_sampled():
    """The packed prefill workload at full size (32768 tokens in 16 segments, 32/8 heads, D=128,
    causal + ALiBi) with e4m3 inputs, one launch as the bench runs it; checked whole segment by
    whole segment (the longest, the shortest and one between) for the four query heads of KV
    groups 0 and 7, each slice against the oracle with the bound above."""
    w = workload(2)
    hq, hkv = 32, 8
    r = hq // hkv
    (q8, k8, v8, slopes, cu), out, lse = _run(w.seqlens_q, hq, hkv, True, True, w.scale, w.seed)
    lens = w.seqlens_q
    segs = sorted({max(range(len(lens)), key=lambda i: lens[i]),
                   min(range(len(lens)), key=lambda i: lens[i]), len(lens) // 2})
    c = cu.tolist()
    for s in segs:
        a, e = c[s], c[s + 1]
        for g in (0, hkv - 1):
            hs = slice(g * r, (g + 1) * r)
            _check(q8[a:e, hs], k8[a:e, g:g + 1], v8[a:e, g:g + 1], slopes[hs], [e - a],
                   w.scale, True, out[a:e, hs], lse[hs, a:e])

