"""The xformers-style entry point under autograd: memory_efficient_attention on BMHK / BMGHK
inputs that require grad runs mea_forward and, on .backward(), mea_backward; the gradients that
reach the user's tensors match the float64 oracle (same tolerance as the backward tests:
16u * (rms(ref) + |ref|) + 1e-5 with u = 2^-8 for bf16)."""
import pytest
import torch

import memory_efficient_attention_b200 as mea
import oracle
from mea_workloads import alibi_slope_values, randn

pytestmark = pytest.mark.gpu
U = 2.0 ** -8


def _close(got, ref, what):
    got = got.double().cpu()
    bound = 16 * U * (ref.pow(2).mean().sqrt() + ref.abs()) + 1e-5
    assert bool(((got - ref).abs() <= bound).all()), f"{what}: max err {float((got - ref).abs().max())}"


def test_bmghk_causal_alibi_gradients():
    b, m, g, hq, kd = 2, 160, 2, 4, 128
    q = randn((b, m, g, hq, kd), 2001, torch.bfloat16)
    k = randn((b, m, g, 1, kd), 2002, torch.bfloat16)
    v = randn((b, m, g, 1, kd), 2003, torch.bfloat16)
    do = randn((b, m, g, hq, kd), 2004, torch.bfloat16)
    sl = alibi_slope_values(g * hq)
    qd, kd_, vd = (t.cuda().requires_grad_() for t in (q, k, v))
    out = mea.memory_efficient_attention(qd, kd_, vd, mea.LowerTriangularMask(sl.cuda()),
                                         scale=0.09)
    (out.float() * do.cuda().float()).sum().backward()
    cu = [0, m, 2 * m]
    gq, gk, gv = oracle.attention_backward(q.reshape(b * m, g * hq, kd), k.reshape(b * m, g, kd),
                                           v.reshape(b * m, g, kd), do.reshape(b * m, g * hq, kd),
                                           cu, cu, 0.09, True, sl.double())
    _close(qd.grad.reshape(b * m, g * hq, kd), gq, "dq")
    _close(kd_.grad.reshape(b * m, g, kd), gk, "dk")
    _close(vd.grad.reshape(b * m, g, kd), gv, "dv")


def test_packed_block_diagonal_causal_gradients():
    lens = [37, 120, 8, 200]
    t, h, kd = sum(lens), 8, 64
    q = randn((1, t, h, kd), 2011, torch.bfloat16)
    k = randn((1, t, 2, kd), 2012, torch.bfloat16)
    v = randn((1, t, 2, kd), 2013, torch.bfloat16)
    do = randn((1, t, h, kd), 2014, torch.bfloat16)
    qd, kd_, vd = (x.cuda().requires_grad_() for x in (q, k, v))
    bias = mea.BlockDiagonalCausalMask.from_seqlens(lens)
    out = mea.memory_efficient_attention(qd, kd_, vd, bias, scale=0.125)
    (out.float() * do.cuda().float()).sum().backward()
    cu = [0]
    for x in lens:
        cu.append(cu[-1] + x)
    gq, gk, gv = oracle.attention_backward(q[0], k[0], v[0], do[0], cu, cu, 0.125, True)
    _close(qd.grad[0], gq, "dq")
    _close(kd_.grad[0], gk, "dk")
    _close(vd.grad[0], gv, "dv")


def test_no_grad_path_unchanged():
    q = randn((1, 64, 4, 64), 2021, torch.bfloat16).cuda()
    with torch.no_grad():
        a = mea.memory_efficient_attention(q, q, q)
    b = mea.memory_efficient_attention(q.requires_grad_(), q, q)
    assert torch.equal(a, b.detach())
