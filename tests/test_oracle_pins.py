"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources: closed forms and special cases of the softmax, invariants the pages state (packed ==
per-segment, 7minutos page section 4; GQA == repeat_interleave, "group query attention gqa"
snippets), a pure-Python brute force over an explicit mask matrix, and torch's float64 SDPA as a
textbook routine. ``test_planted_mistakes_are_caught`` plants plausible mistakes in the oracle
and shows that at least one pin fails for each.
"""
import json
import math
import os

import pytest
import torch

import oracle
import oracle.core as oa
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv, workload

F64 = torch.float64
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, dtype=torch.float16):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


# ----------------------------------------------------------------------------------------------
# Pin checks: each returns True when the oracle `att` satisfies it. `att` has the signature of
# oracle.attention so that mutants of it can be run through the same checks.
# ----------------------------------------------------------------------------------------------

def pin_single_key(att):
    """A segment with one key returns v_0 exactly, lse = scale <q, k_0> (distance 0, no bias)."""
    q, k, v = _rand((1, 4, 16), 1), _rand((1, 2, 16), 2), _rand((1, 2, 16), 3)
    slopes = torch.tensor([0.5, 0.25, 0.125, 0.0625], dtype=F64)
    ok = True
    for causal in (False, True):
        for sl in (None, slopes):
            out, lse = att(q, k, v, [0, 1], [0, 1], 0.3, causal, sl)
            for h in range(4):
                g = h // 2
                ok &= torch.equal(out[0, h], v[0, g].to(F64))
                ref = 0.3 * float((q[0, h].to(F64) * k[0, g].to(F64)).sum())
                ok &= abs(float(lse[h, 0]) - ref) < 1e-12
    return bool(ok)


def pin_causal_row0(att):
    """Causal row 0 sees only key 0: out_0 = v_0, lse_0 = scale <q_0, k_0> (with or without ALiBi)."""
    q, k, v = _rand((9, 2, 8), 4), _rand((9, 2, 8), 5), _rand((9, 2, 8), 6)
    ok = True
    for sl in (None, torch.tensor([0.7, 0.1], dtype=F64)):
        out, lse = att(q, k, v, [0, 9], [0, 9], 0.5, True, sl)
        for h in range(2):
            ok &= torch.equal(out[0, h], v[0, h].to(F64))
            ref = 0.5 * float((q[0, h].to(F64) * k[0, h].to(F64)).sum())
            ok &= abs(float(lse[h, 0]) - ref) < 1e-12
    return bool(ok)


def pin_zero_query_mean(att):
    """q = 0 and no bias: every admissible key has weight 1/|A_i|, so out_i is the mean of v over
    A_i and lse_i = ln |A_i| (causal: |A_i| = i + 1)."""
    lq = 7
    q = torch.zeros((lq, 1, 8), dtype=torch.float16)
    k, v = _rand((lq, 1, 8), 7), _rand((lq, 1, 8), 8)
    ok = True
    for causal in (False, True):
        out, lse = att(q, k, v, [0, lq], [0, lq], 1.0, causal, None)
        for i in range(lq):
            n = i + 1 if causal else lq
            mean = v[:n, 0].to(F64).mean(0)
            ok &= torch.allclose(out[i, 0], mean, atol=1e-12, rtol=0)
            ok &= abs(float(lse[0, i]) - math.log(n)) < 1e-12
    return bool(ok)


def pin_two_key_closed_form(att):
    """Two keys with scaled scores 0 and ln 3: weights 1/4 and 3/4, lse = ln 4."""
    q = torch.zeros((1, 1, 2), dtype=F64)
    q[0, 0, 0] = 1.0
    k = torch.zeros((2, 1, 2), dtype=F64)
    k[1, 0, 0] = math.log(3.0) / 0.5
    v = torch.tensor([[[1.0, -2.0]], [[5.0, 3.0]]], dtype=F64)
    out, lse = att(q, k, v, [0, 1], [0, 2], 0.5, False, None)
    want = (v[0, 0] + 3.0 * v[1, 0]) / 4.0
    return bool(torch.allclose(out[0, 0], want, atol=1e-13, rtol=0)
                and abs(float(lse[0, 0]) - math.log(4.0)) < 1e-13)


def pin_alibi_closed_form(att):
    """q = 0, ALiBi slope m. Causal row at p=1 over keys {0,1}: biases -m, 0, so the weights are
    e^-m/(1+e^-m) and 1/(1+e^-m), lse = ln(1 + e^-m). Non-causal middle row of 3 keys: biases
    -m, 0, -m (symmetric distance)."""
    m = 0.75
    sl = torch.tensor([m], dtype=F64)
    v = torch.tensor([[[1.0]], [[10.0]], [[100.0]]], dtype=F64)
    q = torch.zeros((3, 1, 1), dtype=F64)
    k = torch.zeros((3, 1, 1), dtype=F64)
    out, lse = att(q[:2], k[:2], v[:2], [0, 2], [0, 2], 1.0, True, sl)
    e = math.exp(-m)
    ok = abs(float(out[1, 0, 0]) - (e * 1.0 + 10.0) / (1.0 + e)) < 1e-12
    ok &= abs(float(lse[0, 1]) - math.log(1.0 + e)) < 1e-12
    out, lse = att(q, k, v, [0, 3], [0, 3], 1.0, False, sl)
    ok &= abs(float(out[1, 0, 0]) - (e * 1.0 + 10.0 + e * 100.0) / (1.0 + 2.0 * e)) < 1e-12
    ok &= abs(float(lse[0, 1]) - math.log(1.0 + 2.0 * e)) < 1e-12
    return bool(ok)


def pin_huge_alibi_slope(att):
    """A huge slope concentrates row i on the key at distance 0 (j = p_i): out_i -> v_i, causal or not."""
    n = 6
    q, k, v = _rand((n, 2, 8), 9), _rand((n, 2, 8), 10), _rand((n, 2, 8), 11)
    sl = torch.tensor([1e4, 1e4], dtype=F64)
    ok = True
    for causal in (True, False):
        out, _ = att(q, k, v, [0, n], [0, n], 0.1, causal, sl)
        ok &= torch.allclose(out, v.to(F64), atol=1e-9, rtol=0)
    return bool(ok)


def pin_rows_sum_to_one_and_constant_v(att):
    """Constant V rows give that constant (the softmax weights sum to 1), for every mask kind."""
    q, k = _rand((20, 4, 16), 12), _rand((20, 2, 16), 13)
    v = torch.full((20, 2, 16), 0.375, dtype=torch.float16)
    sl = alibi_slope_values(4).to(F64)
    ok = True
    for causal in (False, True):
        for s in (None, sl):
            out, _ = att(q, k, v, [0, 5, 20], [0, 5, 20], 0.25, causal, s)
            ok &= torch.allclose(out, torch.full_like(out, 0.375), atol=1e-12, rtol=0)
    return bool(ok)


def pin_packed_equals_segments(att):
    """Packed output equals attention run on each segment alone (7minutos page, section 4)."""
    lens = [5, 1, 12, 3]
    q, k, v = make_qkv(lens, lens, 4, 4, 16, torch.float16, 77)
    cu = cu_seqlens(lens).tolist()
    ok = True
    for causal in (False, True):
        out, lse = att(q, k, v, cu, cu, 0.25, causal, alibi_slope_values(4).to(F64))
        for s in range(len(lens)):
            a, b = cu[s], cu[s + 1]
            o1, l1 = att(q[a:b], k[a:b], v[a:b], [0, b - a], [0, b - a], 0.25, causal,
                         alibi_slope_values(4).to(F64))
            ok &= torch.allclose(out[a:b], o1, atol=1e-13, rtol=0)
            ok &= torch.allclose(lse[:, a:b], l1, atol=1e-13, rtol=0)
    return bool(ok)


def pin_gqa_equals_repeat_interleave(att):
    """GQA equals MHA on K/V repeat_interleave-d along heads ("group query attention gqa")."""
    lens = [9, 14]
    q, k, v = make_qkv(lens, lens, 8, 2, 16, torch.bfloat16, 78)
    cu = cu_seqlens(lens).tolist()
    ok = True
    for causal in (False, True):
        o1, l1 = att(q, k, v, cu, cu, 0.25, causal, None)
        o2, l2 = att(q, k.repeat_interleave(4, 1), v.repeat_interleave(4, 1), cu, cu, 0.25,
                     causal, None)
        ok &= torch.allclose(o1, o2, atol=1e-13, rtol=0) and torch.allclose(l1, l2, atol=1e-13)
    return bool(ok)


def pin_key_permutation(att):
    """Non-causal, no bias: permuting the keys (with their values) of a segment changes nothing."""
    n = 11
    q, k, v = _rand((n, 2, 8), 14), _rand((n, 2, 8), 15), _rand((n, 2, 8), 16)
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(3))
    o1, l1 = att(q, k, v, [0, n], [0, n], 0.3, False, None)
    o2, l2 = att(q, k[perm], v[perm], [0, n], [0, n], 0.3, False, None)
    return bool(torch.allclose(o1, o2, atol=1e-13) and torch.allclose(l1, l2, atol=1e-13))


def pin_bruteforce(att):
    """Agreement with pure-Python loops over an explicit [T_q, T_k] additive mask matrix."""
    cases = [
        ([3, 1, 4], [3, 1, 4], 2, 2, False, False),
        ([3, 1, 4], [3, 1, 4], 4, 2, True, True),
        ([2, 3], [4, 3], 2, 1, True, True),      # L_q < L_k: bottom-right alignment
        ([3, 2], [2, 0], 2, 2, True, False),     # causal rows with no admissible key; empty L_k
        ([1, 1], [5, 2], 4, 1, False, True),     # decode-shaped, MQA, non-causal ALiBi
    ]
    ok = True
    for i, (lq, lk, hq, hkv, causal, alibi) in enumerate(cases):
        q, k, v = make_qkv(lq, lk, hq, hkv, 4, torch.float16, 200 + i)
        sl = alibi_slope_values(hq).to(F64) if alibi else None
        out, lse = att(q, k, v, cu_seqlens(lq).tolist(), cu_seqlens(lk).tolist(), 0.4, causal, sl)
        bo, bl = oracle.attention_bruteforce(q, k, v, lq, lk, 0.4, causal,
                                             None if sl is None else sl.tolist())
        bo, bl = torch.tensor(bo, dtype=F64), torch.tensor(bl, dtype=F64)
        ok &= torch.allclose(out, bo, atol=1e-12, rtol=0)
        ok &= bool(((lse - bl).abs() < 1e-12).logical_or(lse == bl).all())
    return bool(ok)


def pin_sdpa(att):
    """Agreement with torch's float64 scaled_dot_product_attention given an explicit float mask
    (block-diagonal + causal + ALiBi), used as a textbook routine on small shapes."""
    lens = [6, 10]
    hq, hkv = 4, 2
    q, k, v = make_qkv(lens, lens, hq, hkv, 8, torch.float16, 300)
    sl = alibi_slope_values(hq).to(F64)
    tq = sum(lens)
    seg = torch.cat([torch.full((n,), s) for s, n in enumerate(lens)])
    pos = torch.cat([torch.arange(n) for n in lens])
    ok = True
    for causal in (False, True):
        mask = torch.zeros((hq, tq, tq), dtype=F64)
        allowed = seg[:, None] == seg[None, :]
        if causal:
            allowed &= pos[None, :] <= pos[:, None]
        dist = (pos[:, None] - pos[None, :]).abs().to(F64)
        mask = torch.where(allowed, -sl[:, None, None] * dist, torch.tensor(float("-inf"), dtype=F64))
        qh = q.to(F64).permute(1, 0, 2)
        kh = k.to(F64).repeat_interleave(hq // hkv, 1).permute(1, 0, 2)
        vh = v.to(F64).repeat_interleave(hq // hkv, 1).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask,
                                                               scale=0.35)
        out, _ = att(q, k, v, cu_seqlens(lens).tolist(), cu_seqlens(lens).tolist(), 0.35, causal, sl)
        ok &= torch.allclose(out.permute(1, 0, 2), ref, atol=1e-12, rtol=0)
    return bool(ok)


def pin_bottom_right_decode(att):
    """One query per segment against L_k keys, causal: the query is the newest token, so with
    q = 0 it averages all L_k values (bottom-right alignment at L_q = 1)."""
    lk = [5, 3]
    q = torch.zeros((2, 2, 4), dtype=torch.float16)
    k, v = _rand((8, 1, 4), 20), _rand((8, 1, 4), 21)
    out, lse = att(q, k, v, [0, 1, 2], cu_seqlens(lk).tolist(), 1.0, True, None)
    ok = torch.allclose(out[0, 0], v[:5, 0].to(F64).mean(0), atol=1e-12)
    ok &= torch.allclose(out[1, 1], v[5:, 0].to(F64).mean(0), atol=1e-12)
    ok &= abs(float(lse[0, 0]) - math.log(5)) < 1e-12 and abs(float(lse[1, 1]) - math.log(3)) < 1e-12
    return bool(ok)


def pin_empty_rows(att):
    """No admissible key: out = 0, lse = -inf (L_k = 0, and causal rows with p_i < 0)."""
    q, k, v = _rand((5, 1, 4), 22), _rand((2, 1, 4), 23), _rand((2, 1, 4), 24)
    out, lse = att(q, k, v, [0, 2, 5], [0, 0, 2], 1.0, True, None)
    # segment 0 has no keys; segment 1 has L_q = 3, L_k = 2 -> p = -1, 0, 1 -> row 0 empty
    ok = torch.equal(out[0:3], torch.zeros_like(out[0:3]))
    ok &= bool(torch.isneginf(lse[0, 0:3]).all())
    ok &= torch.equal(out[3, 0], v[0, 0].to(F64))
    return bool(ok)


PINS = [pin_single_key, pin_causal_row0, pin_zero_query_mean, pin_two_key_closed_form,
        pin_alibi_closed_form, pin_huge_alibi_slope, pin_rows_sum_to_one_and_constant_v,
        pin_packed_equals_segments, pin_gqa_equals_repeat_interleave, pin_key_permutation,
        pin_bruteforce, pin_sdpa, pin_bottom_right_decode, pin_empty_rows]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    assert pin(oracle.attention)


def test_alibi_slopes_closed_form():
    # H = 8: 2^-1 ... 2^-8 ; H = 32: 2^-(h+1)/4
    s8 = oracle.alibi_slopes(8)
    assert torch.equal(s8, torch.tensor([2.0 ** -(h + 1) for h in range(8)], dtype=F64))
    s32 = oracle.alibi_slopes(32)
    assert abs(float(s32[3]) - 0.5) < 1e-15 and abs(float(s32[31]) - 2.0 ** -8) < 1e-15
    assert torch.allclose(alibi_slope_values(32).to(F64), s32, rtol=1e-7, atol=0)


def test_rows_sum_to_one_probs():
    lens = [4, 7]
    q, k, v = make_qkv(lens, lens, 2, 1, 8, torch.float16, 31)
    for causal in (False, True):
        ps = oracle.attention_probs(q, k, v, [0, 4, 11], [0, 4, 11], 0.5, causal,
                                    oracle.alibi_slopes(2))
        for p in ps:
            assert torch.allclose(p.sum(-1), torch.ones(p.shape[:-1], dtype=F64), atol=1e-14)
            if causal:
                assert torch.equal(torch.triu(p, diagonal=1), torch.zeros_like(p))


def test_attention_rows_matches_full():
    lens = [13, 29, 4]
    q, k, v = make_qkv(lens, lens, 4, 2, 16, torch.bfloat16, 41)
    sl = oracle.alibi_slopes(4)
    cu = cu_seqlens(lens).tolist()
    for causal in (False, True):
        out, lse = oracle.attention(q, k, v, cu, cu, 0.2, causal, sl)
        rows = [(h, t) for h in range(4) for t in (0, 12, 13, 30, 41, 45)]
        ro, rl = oracle.attention_rows(q, k, v, cu, cu, 0.2, causal, sl, rows)
        for n, (h, t) in enumerate(rows):
            assert torch.allclose(ro[n], out[t, h], atol=1e-13)
            assert abs(float(rl[n] - lse[h, t])) < 1e-13


def test_split_merge_equals_unsplit():
    """Splitting the keys into chunks and merging by log-sum-exp reproduces the unsplit row
    (split-K of the 300% page, section 1) — this pins the merge step on the CPU."""
    lk = 301
    q, k, v = make_qkv([1], [lk], 1, 1, 32, torch.bfloat16, 51)
    bias = -0.01 * torch.arange(lk - 1, -1, -1, dtype=F64)
    sl = torch.tensor([0.01], dtype=F64)
    full_o, full_l = oracle.attention(q, k, v, [0, 1], [0, lk], 0.2, True, sl)
    for chunk in (1, 7, 64, 128, 301, 1000):
        lp, op = oracle.split_attention_chunks(q[0, 0], k[:, 0], v[:, 0], 0.2, chunk, bias)
        mo, ml = oracle.lse_merge(lp, op)
        assert torch.allclose(mo, full_o[0, 0], atol=1e-13), chunk
        assert abs(float(ml - full_l[0, 0])) < 1e-12, chunk
    # an all-empty merge is empty
    mo, ml = oracle.lse_merge(torch.full((3,), float("-inf"), dtype=F64), torch.zeros((3, 4)))
    assert torch.equal(mo, torch.zeros(4, dtype=F64)) and torch.isneginf(ml)


def test_decode_is_attention_with_one_query():
    lk = [17, 1, 40]
    b, hq, hkv, d = 3, 8, 2, 16
    _, k, v = make_qkv([1], lk, hq, hkv, d, torch.bfloat16, 61)
    q = make_qkv([b], [1], hq, hkv, d, torch.bfloat16, 62)[0]
    out, lse = oracle.decode(q, k, v, cu_seqlens(lk).tolist(), 0.25, oracle.alibi_slopes(hq))
    for i in range(b):
        a, e = int(cu_seqlens(lk)[i]), int(cu_seqlens(lk)[i + 1])
        o1, l1 = oracle.attention(q[i:i + 1], k[a:e], v[a:e], [0, 1], [0, e - a], 0.25, False,
                                  oracle.alibi_slopes(hq))
        assert torch.allclose(out[i], o1[0], atol=1e-13) and torch.allclose(lse[:, i], l1[:, 0])


def test_golden_packed_example_shapes():
    """Shapes printed by the packed and grouped examples (7minutos page, sections 4 and 5)."""
    with open(os.path.join(GOLDEN, "packed_example_shapes.json")) as f:
        g = json.load(f)
    w0 = workload(0)
    assert w0.seqlens_q == g["seqlens"] and w0.total_q == g["total"]
    q, k, v = make_qkv(w0.seqlens_q, w0.seqlens_k, 8, 8, 64, torch.float16, w0.seed)
    cu = cu_seqlens(w0.seqlens_q).tolist()
    out, _ = oracle.attention(q, k, v, cu, cu, 1 / 8, False)
    assert [1] + list(out.shape) == g["packed_out_shape"]
    parts = torch.split(out, w0.seqlens_q, dim=0)
    assert [[1] + list(p.shape) for p in parts] == g["split_shapes"]
    b, m, gg, hq, kk = g["bmghk_q_shape"]
    assert workload(1).extra["bmghk"] == (b, m, gg, hq, kk)
    assert g["bmghk_out_shape"] == [b, m, gg, hq, kk]


# ----------------------------------------------------------------------------------------------
# Planted mistakes: each mutant of the oracle must fail at least one pin.
# ----------------------------------------------------------------------------------------------

def _mutant_scores(kind):
    orig = oa._segment_scores

    def scores(q_s, k_s, scale, causal, slope):
        if kind == "no_scale":
            return orig(q_s, k_s, 1.0, causal, slope)
        if kind == "alibi_sign":
            return orig(q_s, k_s, scale, causal, None if slope is None else -slope)
        if kind == "top_left_causal":
            l_q, l_k = q_s.shape[0], k_s.shape[0]
            s = scale * (q_s @ k_s.T)
            i = torch.arange(l_q)[:, None]
            j = torch.arange(l_k)[None, :]
            if slope is not None:
                s = s - float(slope) * (i - j).abs().to(F64)
            return s.masked_fill(j > i, float("-inf")) if causal else s
        if kind == "strict_causal":
            l_q, l_k = q_s.shape[0], k_s.shape[0]
            s = orig(q_s, k_s, scale, False, slope)
            p = oa.segment_positions(l_q, l_k)
            return s.masked_fill(torch.arange(l_k)[None, :] >= p[:, None], float("-inf")) if causal else s
        if kind == "transposed_qk":
            s = orig(k_s, q_s, scale, causal, slope)
            return s.T if s.shape[0] != q_s.shape[0] else s.T.contiguous()
        raise AssertionError(kind)
    return scores


@pytest.mark.parametrize("kind", ["no_scale", "alibi_sign", "top_left_causal", "strict_causal",
                                  "transposed_qk", "wrong_group", "no_max_shift_lse",
                                  "no_block_diagonal"])
def test_planted_mistakes_are_caught(kind, monkeypatch):
    if kind == "wrong_group":
        # query head h reads key/value head h % Hkv instead of h // R
        def target(q, k, v, cu_q, cu_k, scale, causal, slopes=None):
            hq, hkv = q.shape[1], k.shape[1]
            r = hq // hkv
            idx = torch.tensor([(h % hkv) * r for h in range(hq)])
            return oa.attention(q, k.repeat_interleave(r, 1)[:, idx],
                                v.repeat_interleave(r, 1)[:, idx], cu_q, cu_k, scale, causal, slopes)
    elif kind == "no_max_shift_lse":
        orig_sm = oa._softmax_rows

        def sm(s):
            p, lse = orig_sm(s)
            m = s.max(dim=-1).values if s.shape[-1] else lse
            return p, torch.where(torch.isfinite(m), lse - m, lse)
        monkeypatch.setattr(oa, "_softmax_rows", sm)
        target = oa.attention
    elif kind == "no_block_diagonal":
        # segments attend across their boundaries (one big segment)
        def target(q, k, v, cu_q, cu_k, scale, causal, slopes=None):
            return oa.attention(q, k, v, [0, q.shape[0]], [0, k.shape[0]], scale, causal, slopes)
    else:
        monkeypatch.setattr(oa, "_segment_scores", _mutant_scores(kind))
        target = oa.attention
    results = {}
    for pin in PINS:
        try:
            results[pin.__name__] = pin(target)
        except Exception:  # a crash also counts as a caught mistake
            results[pin.__name__] = False
    assert not all(results.values()), f"mutant {kind} passed every pin"


def test_paged_gather_inverts_a_brute_force_scatter():
    """Scatter packed keys into a shuffled block cache with explicit loops, then gather them back
    with oracle.paged_gather: the packed tensor is recovered exactly (block sizes 16 and 64,
    requests that end mid-block, unused blocks holding NaN)."""
    g = torch.Generator().manual_seed(77)
    for bs in (16, 64):
        lens = [1, 17, 64, 100, 0, 33]
        packed = torch.randn((sum(lens), 3, 8), generator=g, dtype=F64)
        nblk = [-(-x // bs) for x in lens]
        num_blocks = sum(nblk) + 3
        perm = torch.randperm(num_blocks, generator=g).tolist()
        cache = torch.full((num_blocks, bs, 3, 8), float("nan"), dtype=F64)
        table = [[-1] * max(nblk) for _ in lens]
        nxt, off = 0, 0
        for b, length in enumerate(lens):
            for j in range(nblk[b]):
                table[b][j] = perm[nxt]
                nxt += 1
            for t in range(length):
                cache[table[b][t // bs], t % bs] = packed[off + t]
            off += length
        back = oracle.paged_gather(cache, table, lens)
        assert torch.equal(back, packed)


def test_e4m3_decode_matches_the_format_definition_and_torch():
    """E4M3 code points worked out by hand from the format (sign, 4-bit exponent bias 7, 3-bit
    mantissa, subnormals, no infinities), and agreement with torch's float8_e4m3fn decoding
    over all 256 codes (NaN codes 0x7F / 0xFF excepted)."""
    by_hand = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0x3C: 1.5, 0x7E: 448.0, 0xFE: -448.0,
               0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0xB8: -1.0}
    codes = torch.tensor(list(by_hand), dtype=torch.uint8)
    got = oracle.e4m3_decode(codes)
    for c, want in zip(by_hand, got.tolist()):
        assert want == by_hand[c], hex(c)
    allc = torch.arange(256, dtype=torch.uint8)
    dec = oracle.e4m3_decode(allc)
    assert torch.isnan(dec[0x7F]) and torch.isnan(dec[0xFF])
    tv = allc.view(torch.float8_e4m3fn).to(F64)
    ok = ~torch.isnan(dec)
    assert torch.equal(dec[ok], tv[ok])
