"""Pins for the oracle's backward pass (oracle.attention_backward).

Each check ties the gradients to something other than the function itself: central finite
differences of the (separately pinned) forward oracle, closed forms of the softmax derivative,
the shift invariance of the softmax (the key gradients of a segment sum to zero), and torch's
reverse-mode differentiation of the forward oracle as a library routine. Planted mistakes
(a dropped term, a wrong sign, a missing scale, GQA heads not summed, a wrong head index)
must each fail at least one pin.
"""
import pytest
import torch

import oracle
import oracle.core as oa

F64 = torch.float64


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=F64)


def _case(seed=0, hq=4, hkv=2, d=6, lq=(3, 5), lk=(4, 5)):
    q = _rand((sum(lq), hq, d), seed)
    k = _rand((sum(lk), hkv, d), seed + 1)
    v = _rand((sum(lk), hkv, d), seed + 2)
    do = _rand((sum(lq), hq, d), seed + 3)
    cq = [0]
    for x in lq:
        cq.append(cq[-1] + x)
    ck = [0]
    for x in lk:
        ck.append(ck[-1] + x)
    return q, k, v, do, cq, ck


# ------------------------------------------------------------------------------ pin checks
# Each takes a backward with the signature of oracle.attention_backward and returns True when
# the pin holds, so that mutants run through the same checks.

def pin_finite_differences(bwd):
    """Central differences of L = sum(attention(q, k, v) * dout) match the gradients (causal +
    ALiBi + GQA + two segments with L_q != L_k; and the non-causal form)."""
    ok = True
    for causal, alibi in ((True, True), (False, False), (False, True)):
        q, k, v, do, cq, ck = _case(seed=11 if causal else 21)
        sl = oracle.alibi_slopes(q.shape[1]) if alibi else None
        scale = 0.37
        dq, dk, dv = bwd(q, k, v, do, cq, ck, scale, causal, sl)

        def loss(qq, kk, vv):
            o, _ = oracle.attention(qq, kk, vv, cq, ck, scale, causal, sl)
            return float((o * do).sum())

        eps = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            num = torch.zeros_like(x)
            flat, nflat = x.view(-1), num.view(-1)
            for i in range(flat.numel()):
                old = float(flat[i])
                flat[i] = old + eps
                lp = loss(q, k, v)
                flat[i] = old - eps
                lm = loss(q, k, v)
                flat[i] = old
                nflat[i] = (lp - lm) / (2 * eps)
            ok &= bool(torch.allclose(g, num, atol=1e-6, rtol=1e-6))
    return ok


def pin_single_key_closed_form(bwd):
    """One key per segment and no causal mask: out = v_0 for every row whatever the bias, so
    dq = 0, dk = 0 and dv_0 = the sum of dout over the rows and heads that use it."""
    q, k, v, do, cq, ck = _case(seed=31, lq=(3, 2), lk=(1, 1))
    dq, dk, dv = bwd(q, k, v, do, cq, ck, 0.5, False, oracle.alibi_slopes(4))
    ok = bool(dq.abs().max() < 1e-12) and bool(dk.abs().max() < 1e-12)
    r = q.shape[1] // k.shape[1]
    for s in range(2):
        for g in range(k.shape[1]):
            want = do[cq[s]:cq[s + 1], g * r:(g + 1) * r].sum(dim=(0, 1))
            ok &= bool(torch.allclose(dv[ck[s], g], want, atol=1e-12))
    return ok


def pin_zero_scale_closed_form(bwd):
    """scale = 0, no bias, no mask: P is uniform 1/L_k, so dq = 0 and dv_j = (1/L_k) sum_i dout_i
    (summed over the group's heads); dk_j = 0 * ... = 0."""
    q, k, v, do, cq, ck = _case(seed=41, lq=(4,), lk=(6,))
    dq, dk, dv = bwd(q, k, v, do, cq, ck, 0.0, False, None)
    r = q.shape[1] // k.shape[1]
    ok = bool(dq.abs().max() < 1e-12) and bool(dk.abs().max() < 1e-12)
    for g in range(k.shape[1]):
        want = do[:, g * r:(g + 1) * r].sum(dim=(0, 1)) / 6.0
        ok &= bool(torch.allclose(dv[:, g], want.expand(6, -1), atol=1e-12))
    return ok


def pin_key_gradients_sum_to_zero(bwd):
    """Softmax is invariant to adding a constant to a row of scores, so sum_j dS_ij = 0 and the
    key gradients of a segment and KV head sum to zero (any mask or bias)."""
    q, k, v, do, cq, ck = _case(seed=51)
    _, dk, _ = bwd(q, k, v, do, cq, ck, 0.41, True, oracle.alibi_slopes(4))
    ok = True
    for s in range(2):
        ok &= bool(dk[ck[s]:ck[s + 1]].sum(dim=0).abs().max() < 1e-10)
    return ok


def pin_autograd(bwd):
    """torch reverse-mode differentiation of the forward oracle gives the same gradients."""
    q, k, v, do, cq, ck = _case(seed=61, lq=(5, 7), lk=(5, 9))
    sl = oracle.alibi_slopes(4)
    dq, dk, dv = bwd(q, k, v, do, cq, ck, 0.3, True, sl)
    qq, kk, vv = (t.clone().requires_grad_() for t in (q, k, v))
    o, _ = oracle.attention(qq, kk, vv, cq, ck, 0.3, True, sl)
    (o * do).sum().backward()
    return all(bool(torch.allclose(a, b.grad, atol=1e-12, rtol=1e-10))
               for a, b in ((dq, qq), (dk, kk), (dv, vv)))


PINS = [pin_finite_differences, pin_single_key_closed_form, pin_zero_scale_closed_form,
        pin_key_gradients_sum_to_zero, pin_autograd]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_backward_pin(pin):
    assert pin(oracle.attention_backward)


def test_backward_of_empty_segments_is_zero():
    q, k, v, do, cq, ck = _case(seed=71, lq=(0, 4, 3), lk=(2, 0, 3))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, cq, ck, 0.5, False, None)
    assert dq[0:4].abs().max() == 0          # segment 1 has no keys
    assert dk[0:2].abs().max() == 0 and dv[0:2].abs().max() == 0   # segment 0 has no queries


# ------------------------------------------------------------------------------ planted mistakes

def _mutant(kind):
    def bwd(q, k, v, dout, cu_q, cu_k, scale, causal, slopes=None):
        cu_q = list(cu_q)
        cu_k = list(cu_k)
        r = q.shape[1] // k.shape[1]
        dq, dk, dv = (torch.zeros_like(t) for t in (q, k, v))
        for s in range(len(cu_q) - 1):
            q0, q1, k0, k1 = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
            if q1 == q0 or k1 == k0:
                continue
            for h in range(q.shape[1]):
                g = h // r
                hd = g if kind == "wrong_head" else h
                qs, ks, vs, dos = q[q0:q1, h], k[k0:k1, g], v[k0:k1, g], dout[q0:q1, hd]
                sc = oa._segment_scores(qs, ks, scale, causal,
                                        None if slopes is None else slopes[h])
                pr, _ = oa._softmax_rows(sc)
                out = pr @ vs
                dp = dos @ vs.T
                delta = (dos * out).sum(dim=-1, keepdim=True)
                if kind == "no_delta":
                    ds = pr * dp
                elif kind == "delta_sign":
                    ds = pr * (dp + delta)
                else:
                    ds = pr * (dp - delta)
                sc_q = 1.0 if kind == "no_scale" else scale
                dq[q0:q1, h] = sc_q * (ds @ ks)
                upd_k = scale * (ds.T @ qs)
                upd_v = pr.T @ dos
                if kind == "gqa_overwrite":
                    dk[k0:k1, g] = upd_k
                    dv[k0:k1, g] = upd_v
                else:
                    dk[k0:k1, g] += upd_k
                    dv[k0:k1, g] += upd_v
        return dq, dk, dv
    return bwd


@pytest.mark.parametrize("kind", ["no_delta", "delta_sign", "no_scale", "gqa_overwrite",
                                  "wrong_head"])
def test_planted_backward_mistakes_are_caught(kind):
    results = {p.__name__: p(_mutant(kind)) for p in PINS}
    assert not all(results.values()), f"mutant {kind} passed every pin"


def test_unmutated_copy_passes_every_pin():
    assert all(p(_mutant("none")) for p in PINS)
