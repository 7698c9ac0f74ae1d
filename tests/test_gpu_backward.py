"""GPU parity of the backward pass (mea_backward through the C ABI) against the float64 oracle.

The CUDA backward takes the CUDA forward's out and lse (as a training step does); the oracle
differentiates the forward definition from q, k, v and dout alone. Gradients are compared
element by element. Tolerance (no gradient tolerance is stated for this method, so it is derived
from the arithmetic): P and dS enter the tensor cores rounded to 16 bits (relative 2^-8 for
bf16, 2^-11 for fp16), out (inside rowsum(dout * out)) is the 16-bit forward output and the
results are rounded to 16 bits once; each gradient element is a sum of such products, so its
error is a few unit roundoffs u times the typical magnitude of the terms (the largest seen over
these cases: 3.3e-2 = 8.5u for bf16, 4.3e-3 = 8.8u for fp16, relative to rms + |reference|). The
bound is 16u * (rms(reference) + |reference|) + 1e-5 per element, u = 2^-8 (bf16) or 2^-11
(fp16); the 1e-5 floor covers gradients that are zero by the mathematics (dq with a single key,
where the rounded rowsum(dout * out) and dout * v cancel only to the last bit).
"""
import math

import pytest
import torch

import memory_efficient_attention_b200 as mea
import oracle
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv, randn, workload

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: (16 * 2.0 ** -8, 16 * 2.0 ** -8),
       torch.float16: (16 * 2.0 ** -11, 16 * 2.0 ** -11)}


def _run(seqlens_q, seqlens_k, hq, hkv, d, dtype, causal, alibi, scale, seed):
    q, k, v = make_qkv(seqlens_q, seqlens_k, hq, hkv, d, dtype, seed)
    dout = randn((sum(seqlens_q), hq, d), seed + 7, dtype)
    slopes = alibi_slope_values(hq) if alibi else None
    cq, ck = cu_seqlens(seqlens_q), cu_seqlens(seqlens_k)
    dev = "cuda"
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    cqd, ckd = cq.to(dev), ck.to(dev)
    sd = slopes.to(dev) if alibi else None
    out, lse = mea.attention_packed(qd, kd, vd, cqd, ckd, max(seqlens_q), causal=causal,
                                    alibi_slopes=sd, scale=scale)
    dq, dk, dv = mea.attention_packed_backward(qd, kd, vd, out, lse, dod, cqd, ckd,
                                               max(seqlens_q), max(seqlens_k), causal=causal,
                                               alibi_slopes=sd, scale=scale)
    torch.cuda.synchronize()
    assert mea.device_error() == 0
    return (q, k, v, dout, cq, ck, slopes), (dq.cpu(), dk.cpu(), dv.cpu())


def _assert_grad_close(got, ref, dtype, what):
    atol, rtol = TOL[dtype]
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        a = a.double()
        assert torch.isfinite(a).all(), f"{what} {name}: non-finite values"
        rms = float(b.pow(2).mean().sqrt()) if b.numel() else 0.0
        err = (a - b).abs()
        bound = atol * rms + rtol * b.abs() + 1e-5
        worst = float((err - bound).max()) if b.numel() else 0.0
        assert worst <= 0.0, (f"{what} {name}: max err {float(err.max()):.3e} "
                              f"(rms ref {rms:.3e}) exceeds the bound by {worst:.3e}")


def _check(seqlens_q, seqlens_k, hq, hkv, d, dtype, causal, alibi, scale, seed):
    (q, k, v, dout, cq, ck, slopes), got = _run(seqlens_q, seqlens_k, hq, hkv, d, dtype, causal,
                                                alibi, scale, seed)
    ref = oracle.attention_backward(q, k, v, dout, cq.tolist(), ck.tolist(), scale, causal,
                                    None if slopes is None else slopes.double())
    _assert_grad_close(got, ref, dtype,
                       f"q{list(seqlens_q)[:5]} k{list(seqlens_k)[:5]} H{hq}/{hkv} D{d} {dtype} "
                       f"causal={causal} alibi={alibi}")


@pytest.mark.parametrize("causal", [False, True])
def test_backward_small_packed_workload(causal):
    w = workload(0)
    _check(w.seqlens_q, w.seqlens_k, 8, 8, 64, torch.float16, causal, False, w.scale, w.seed)


@pytest.mark.parametrize("hq,hkv", [(8, 2), (12, 4), (9, 3), (4, 1)])
def test_backward_gqa_causal_alibi(hq, hkv):
    _check([130, 77, 300], [130, 77, 300], hq, hkv, 128, torch.bfloat16, True, True,
           1 / math.sqrt(128), 900 + hq)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal,alibi", [(False, False), (True, False), (False, True),
                                          (True, True)])
def test_backward_dtypes_dims_masks(d, dtype, causal, alibi):
    _check([190, 65], [190, 65], 4, 2, d, dtype, causal, alibi, 0.11, 950)


@pytest.mark.parametrize("lens", [[63], [64], [65], [128], [129], [1], [2, 3]])
def test_backward_tile_edges(lens):
    _check(lens, lens, 4, 2, 128, torch.bfloat16, True, False, 0.09, 960 + sum(lens))


def test_backward_q_and_k_lengths_differ():
    _check([50, 200, 7], [120, 64, 7], 8, 4, 64, torch.bfloat16, True, True, 0.1, 970)
    _check([50, 200, 7], [120, 64, 7], 8, 4, 64, torch.bfloat16, False, False, 0.1, 971)


def test_backward_empty_segments():
    _check([0, 40, 30, 5], [20, 0, 50, 5], 4, 2, 64, torch.bfloat16, True, False, 0.1, 980)
    _check([0, 40, 30, 5], [20, 0, 50, 5], 4, 2, 64, torch.bfloat16, False, True, 0.1, 981)


def test_backward_packed_prefill_workload_one_kv_group():
    """The 32768-token packed causal GQA+ALiBi workload at full size through the CUDA path; the
    oracle checks KV group 0 (query heads 0-3 and KV head 0: dq of those heads, dk/dv of KV
    head 0 depend on nothing else)."""
    w = workload(2)
    (q, k, v, dout, cq, ck, slopes), (dq, dk, dv) = _run(w.seqlens_q, w.seqlens_k, 32, 8, 128,
                                                         torch.bfloat16, True, True, w.scale,
                                                         w.seed)
    ref = oracle.attention_backward(q[:, 0:4], k[:, 0:1], v[:, 0:1], dout[:, 0:4], cq.tolist(),
                                    ck.tolist(), w.scale, True, slopes[0:4].double())
    _assert_grad_close((dq[:, 0:4], dk[:, 0:1], dv[:, 0:1]), ref, torch.bfloat16,
                       "packed prefill workload, KV group 0")


def test_backward_is_deterministic():
    _, a = _run([300, 129], [300, 129], 8, 2, 128, torch.bfloat16, True, True, 0.09, 990)
    _, b = _run([300, 129], [300, 129], 8, 2, 128, torch.bfloat16, True, True, 0.09, 990)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
