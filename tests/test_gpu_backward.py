"""GPU parity of the backward pass (mea_backward through the C ABI) against the float64 oracle.

The CUDA backward takes the CUDA forward's out and lse (as a training step does); the oracle
differentiates the forward definition from q, k, v and dout alone. Gradients are compared
element by element against a bound derived beforehand from the arithmetic (no gradient
tolerance is stated for this method), evaluated with the oracle's own P, O and dS:

* the 16-bit output out of the forward is off by at most u|O| + u sum_j P_ij |v_j| per element
  (its own rounding, and P rounded to 16 bits before P V), so delta_i = sum_d dO_id out_id is
  off by at most Ddelta_i = u sum_d |dO_id| (|O_id| + sum_j P_ij |v_jd|);
* dS_ij = P_ij (dP_ij - delta_i) is formed in fp32 from that delta and rounded to 16 bits, so it
  is off by at most E_ij = P_ij Ddelta_i + u |dS_ij|;
* P is rounded to 16 bits before dV += P^T dO: off by at most u P_ij;
* then dq_i = scale sum_j dS_ij k_j, dk_j = scale sum_(h,i) dS_ij q_i and dv_j = sum_(h,i) P_ij dO_i
  (heads h of the KV group) inherit scale E|k|, scale E^T|q| and u P^T|dO|; the fp32
  accumulation of n terms adds (n + 2) 2^-24 times the sum of the terms' magnitudes; the result
  is rounded to 16 bits once more (u |g|).
u = 2^-8 for bf16 and 2^-11 for fp16, plus 2^-16 for the exponentials and the fp32 scores and
lse that P is recomputed from (a relative effect far below 2^-16 at these magnitudes). The
second-order products of these terms are covered by a factor 1 + 4u.
"""
import math

import pytest
import torch

import memory_efficient_attention_b200 as mea
import oracle
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv, randn, workload

pytestmark = pytest.mark.gpu

U16 = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


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


def grad_bounds(q, k, v, dout, cq, ck, scale, causal, slopes, dtype):
    """Per-element bounds on |gradient_gpu - gradient_exact| for dq, dk, dv (module docstring),
    from the oracle's softmax probabilities of each segment and head."""
    u = U16[dtype] + 2.0 ** -16
    hq, hkv = q.shape[1], k.shape[1]
    r = hq // hkv
    q64, k64, v64, do64 = (t.double() for t in (q, k, v, dout))
    bnd = [torch.zeros_like(q64), torch.zeros_like(k64), torch.zeros_like(v64)]
    mag = [torch.zeros_like(q64), torch.zeros_like(k64), torch.zeros_like(v64)]
    n_terms = [1, 1, 1]
    for s in range(len(cq) - 1):
        a, b, c, e = cq[s], cq[s + 1], ck[s], ck[s + 1]
        if b == a or e == c:
            continue
        probs = oracle.attention_probs(q[a:b], k[c:e], v[c:e], [0, b - a], [0, e - c], scale,
                                       causal, slopes)[0]
        n_terms = [max(n_terms[0], e - c), max(n_terms[1], (b - a) * r),
                   max(n_terms[2], (b - a) * r)]
        for h in range(hq):
            g = h // r
            pm, qq, kk, vv, do = probs[h], q64[a:b, h], k64[c:e, g], v64[c:e, g], do64[a:b, h]
            o = pm @ vv
            ds = pm * (do @ vv.T - (do * o).sum(-1, keepdim=True))
            ddelta = u * (do.abs() * (o.abs() + pm @ vv.abs())).sum(-1) \
                + (q.shape[2] + 2) * 2.0 ** -24 * (do * o).abs().sum(-1)
            err = pm * ddelta[:, None] + u * ds.abs()
            bnd[0][a:b, h] += scale * (err @ kk.abs())
            bnd[1][c:e, g] += scale * (err.T @ qq.abs())
            bnd[2][c:e, g] += u * (pm.T @ do.abs())
            mag[0][a:b, h] += scale * (ds.abs() @ kk.abs())
            mag[1][c:e, g] += scale * (ds.abs().T @ qq.abs())
            mag[2][c:e, g] += pm.T @ do.abs()
    u0 = U16[dtype]
    return [(1 + 4 * u0) * bb + (n + 2) * 2.0 ** -24 * mm
            for bb, mm, n in zip(bnd, mag, n_terms)], u0


def _assert_grad_close(got, ref, bounds, what):
    bnd, u = bounds
    for name, a, b, bb in zip(("dq", "dk", "dv"), got, ref, bnd):
        a = a.double()
        assert torch.isfinite(a).all(), f"{what} {name}: non-finite values"
        err = (a - b).abs()
        bound = bb + u * (1 + 4 * u) * b.abs() + 1e-7
        worst = float((err - bound).max()) if b.numel() else 0.0
        assert worst <= 0.0, (f"{what} {name}: max err {float(err.max()):.3e} "
                              f"exceeds the derived bound by {worst:.3e}")


def _check(seqlens_q, seqlens_k, hq, hkv, d, dtype, causal, alibi, scale, seed):
    (q, k, v, dout, cq, ck, slopes), got = _run(seqlens_q, seqlens_k, hq, hkv, d, dtype, causal,
                                                alibi, scale, seed)
    sl = None if slopes is None else slopes.double()
    ref = oracle.attention_backward(q, k, v, dout, cq.tolist(), ck.tolist(), scale, causal, sl)
    bounds = grad_bounds(q, k, v, dout, cq.tolist(), ck.tolist(), scale, causal, sl, dtype)
    _assert_grad_close(got, ref, bounds,
                       f"q{list(seqlens_q)[:5]} k{list(seqlens_k)[:5]} H{hq}/{hkv} D{d} {dtype} "
                       f"causal={causal} alibi={alibi}")


@pytest.mark.parametrize("causal", [False, True])
def test_backward_small_packed_workload(causal):
    w = workload(0)
    _check(w.seqlens_q, w.seqlens_k, 8, 8, 64, torch.float16, causal, False, w.scale, w.seed)


@pytest.mark.parametrize("hq,hkv", [(8, 2), (12, 4), (9, 3), (4, 1), (6, 2)])
def test_backward_gqa_causal_alibi(hq, hkv):
    _check([130, 77, 300], [130, 77, 300], hq, hkv, 128, torch.bfloat16, True, True,
           1 / math.sqrt(128), 900 + hq)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("causal,alibi", [(False, False), (True, False), (False, True),
                                          (True, True)])
def test_backward_dtypes_dims_masks(d, dtype, causal, alibi):
    _check([190, 65], [190, 65], 4, 2, d, dtype, causal, alibi, 0.11, 950)


@pytest.mark.parametrize("hq,hkv,d", [(6, 2, 64), (12, 4, 64), (1, 1, 128), (2, 1, 128),
                                      (3, 1, 128)])
def test_backward_row_term_paths(hq, hkv, d):
    # full-width rows are read as 512-byte warp loads when the heads fill them (a multiple of
    # 256 / D heads), else one lane per head: both forms, at both kernel widths
    _check([190, 65, 3], [190, 65, 3], hq, hkv, d, torch.bfloat16, True, True,
           1 / math.sqrt(d), 990 + hq + d)


def test_backward_outputs_16_byte_aligned_only():
    """dq, dk, dv whose base addresses are 16 but not 32 bytes aligned take the 16-byte store
    form of the epilogues: the same values, bit for bit, as 32-byte aligned outputs, and within
    the derived bound of the oracle."""
    lens, hq, hkv, d, scale = [190, 65, 3], 8, 2, 128, 1 / math.sqrt(128)
    (q, k, v, dout, cq, ck, slopes), ref_al = _run(lens, lens, hq, hkv, d, torch.bfloat16, True,
                                                   True, scale, 996)
    dev = "cuda"
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    cqd, ckd, sd = cq.to(dev), ck.to(dev), slopes.to(dev)
    out, lse = mea.attention_packed(qd, kd, vd, cqd, ckd, max(lens), causal=True,
                                    alibi_slopes=sd, scale=scale)

    def offset_empty(shape):
        n = math.prod(shape)
        buf = torch.empty(n + 8, dtype=torch.bfloat16, device=dev)  # 8 elements = 16 bytes
        t = buf[8:].view(shape)
        assert t.data_ptr() % 32 == 16
        return t

    dq, dk, dv = offset_empty(qd.shape), offset_empty(kd.shape), offset_empty(vd.shape)
    mea.attention_packed_backward(qd, kd, vd, out, lse, dod, cqd, ckd, max(lens), max(lens),
                                  causal=True, alibi_slopes=sd, scale=scale, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert mea.device_error() == 0
    got = (dq.cpu(), dk.cpu(), dv.cpu())
    for g, r in zip(got, ref_al):
        assert torch.equal(g, r)
    sl = slopes.double()
    ref = oracle.attention_backward(q, k, v, dout, cq.tolist(), ck.tolist(), scale, True, sl)
    bounds = grad_bounds(q, k, v, dout, cq.tolist(), ck.tolist(), scale, True, sl, torch.bfloat16)
    _assert_grad_close(got, ref, bounds, "16-byte aligned outputs")


@pytest.mark.parametrize("d", [8, 32, 40, 72, 96, 120])
def test_backward_other_head_dims(d):
    # multiples of 8 up to 128: the 64- or 128-wide kernels with zero-filled columns
    _check([190, 65], [190, 65], 4, 2, d, torch.bfloat16, True, True, 1 / math.sqrt(d), 955 + d)


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
    args = (q[:, 0:4], k[:, 0:1], v[:, 0:1], dout[:, 0:4], cq.tolist(), ck.tolist(), w.scale,
            True, slopes[0:4].double())
    ref = oracle.attention_backward(*args)
    _assert_grad_close((dq[:, 0:4], dk[:, 0:1], dv[:, 0:1]), ref,
                       grad_bounds(*args, torch.bfloat16), "packed prefill workload, KV group 0")


def test_backward_is_deterministic():
    _, a = _run([300, 129], [300, 129], 8, 2, 128, torch.bfloat16, True, True, 0.09, 990)
    _, b = _run([300, 129], [300, 129], 8, 2, 128, torch.bfloat16, True, True, 0.09, 990)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_many_segments_ranked_with_ties():
    """300 segments with repeated lengths: the pre kernel ranks them (ties by index) and the
    dK/dV and dQ grids launch them in that order."""
    import random
    rnd = random.Random(4242)
    lens = [rnd.choice([1, 17, 64, 65, 130, 200]) for _ in range(300)]
    _check(lens, lens, 4, 2, 64, torch.bfloat16, True, True, 0.125, 4242)


def test_backward_more_segments_than_ranked():
    """1100 segments (beyond the 1024 the pre kernel ranks): launched in index order."""
    import random
    rnd = random.Random(4343)
    lens = [rnd.randint(1, 6) for _ in range(1100)]
    _check(lens, lens, 2, 1, 32, torch.bfloat16, True, False, 0.2, 4343)
