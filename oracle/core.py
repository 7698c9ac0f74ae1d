"""Oracle: a plain, slow, obviously correct CPU float64 statement of memory-efficient attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import this module. It shares no code with the CUDA path
(``memory_efficient_attention_b200``) and imports nothing from it.

Sources (the pages, cited by title and section):

* [7minutos §4] "Cómo construir transformadores con memoria eficiente con xFormers usando
  secuencias empaquetadas, GQA, ALiBi, SwiGLU y atención causal", section 4 "Lote empaquetado de
  longitud variable": packed ``[1, total, H, K]`` tensors, ``BlockDiagonalMask.from_seqlens``,
  ``BlockDiagonalCausalMask.from_seqlens``, ``split`` of the packed output, and the check that
  segment 0 of the packed output equals vanilla attention on segment 0 alone.
* [7minutos §5] same page, section 5 "Atención de consultas agrupadas (diseño BMGHK 5-D)":
  q ``[B, M, G, Hq, K]``, k/v ``[B, M, G, 1, K]``, output ``[B, M, G, Hq, K]``.
* [yifor 五大] "How to Build Memory-Efficient Transformers with xFormers Using Packed Sequences,
  GQA, ALiBi, SwiGLU, and Causal Attention" (yifor-blog summary), section "五大核心優化組合":
  item 1 packed sequences + block-diagonal mask, item 2 GQA, item 3 ALiBi (a per-head linear
  position penalty added to the scores), item 5 implicit lower-triangular causal mask; section
  "效能對比": outputs agree with the standard implementation.
* [mqa-snippets] "multi query attention代码" search snippets: ``self_attention`` computes
  ``matmul(query, key^T) / sqrt(d_k)``, masks, softmax, then weights the values.
* [gqa-snippets] "group query attention gqa" search snippets: GQA splits the query heads into
  G groups that share one K/V head; GQA-1 is MQA, GQA-H is MHA; SDPA with ``enable_gqa`` equals
  SDPA on K/V ``repeat_interleave``-d along the head axis.
* [zizhi §1] "大模型推理加速终极指南：xformers如何让Transformer性能飙升300%", section 1
  "分块注意力计算引擎": blockwise computation, split-K attention over the key axis.

Readings where the pages are silent (each one is a choice of this implementation):

* causal alignment when L_q != L_k is bottom-right: query row i of a segment sits at key
  position ``p_i = i + L_k - L_q`` (parity unpinned except for L_q = L_k and L_q = 1);
* ALiBi bias is ``-slope_h * |p_i - j|`` with segment-local positions, added after scaling; the
  slopes default to ``2^(-8(h+1)/H)`` over the H query heads (non-causal form: parity unpinned
  beyond its limits);
* lse is the natural log of the row's sum of exp(scaled, biased scores); a row with no
  admissible key has out = 0 and lse = -inf;
* the split-KV merge combines chunk results by their log-sum-exp (plain algebra of the softmax);
* the backward pass is the derivative of the forward definition with respect to q, k and v for a
  given output gradient (the pages time the forward and the backward of this attention,
  [yifor 五大] "效能對比", but print no formula); the ALiBi slopes and the masks are constants.

Everything is computed in float64 from the exact upcast of the fp16/bf16 inputs. The softmax is
the two-pass, max-subtracted textbook form over the whole row: there is no tiling and no online
rescaling here, so the oracle does not share the GPU path's algorithm.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import torch

__all__ = [
    "alibi_slopes",
    "segment_positions",
    "attention",
    "attention_rows",
    "attention_probs",
    "decode",
    "lse_merge",
    "split_attention_chunks",
    "attention_bruteforce",
    "attention_backward",
    "paged_gather",
    "e4m3_decode",
]

F64 = torch.float64


def alibi_slopes(n_heads: int) -> torch.Tensor:
    """Per-head ALiBi slopes ``m_h = 2^(-8 (h+1) / H)`` for h = 0..H-1, float64.

    [yifor 五大] item 3 gives ALiBi as a different linear penalty per head; the geometric slope
    sequence is the plain reading used throughout this project.
    """
    h = torch.arange(n_heads, dtype=F64)
    return torch.pow(torch.tensor(2.0, dtype=F64), -8.0 * (h + 1.0) / n_heads)


def segment_positions(l_q: int, l_k: int) -> torch.Tensor:
    """Key-axis position of each query row of one segment: ``p_i = i + L_k - L_q`` (int64).

    Bottom-right alignment: the last query row lines up with the last key. For L_q = L_k this is
    the ordinary ``p_i = i`` of the lower-triangular mask ([yifor 五大] item 5).
    """
    return torch.arange(l_q, dtype=torch.int64) + (l_k - l_q)


def _segment_scores(q_s, k_s, scale, causal, slope):
    """Scores of one segment and one query head, with the mask applied as -inf.

    q_s [L_q, D], k_s [L_k, D] float64. Steps as in [mqa-snippets]: ``scale * q k^T`` (the
    snippet divides by sqrt(d_k); the scale is an argument here), then the ALiBi term of
    [yifor 五大] item 3, then the masks of [yifor 五大] items 1 and 5.
    """
    l_q, l_k = q_s.shape[0], k_s.shape[0]
    s = scale * (q_s @ k_s.T)  # [L_q, L_k]
    p = segment_positions(l_q, l_k)
    j = torch.arange(l_k, dtype=torch.int64)
    if slope is not None:
        dist = (p[:, None] - j[None, :]).abs().to(F64)
        s = s - float(slope) * dist
    if causal:
        s = s.masked_fill(j[None, :] > p[:, None], float("-inf"))
    return s


def _softmax_rows(s):
    """Two-pass max-subtracted softmax of each row; returns (P, lse). Empty rows: P = 0, lse = -inf."""
    m = s.max(dim=-1, keepdim=True).values if s.shape[-1] > 0 else torch.full(
        s.shape[:-1] + (1,), float("-inf"), dtype=F64)
    finite = torch.isfinite(m)
    m0 = torch.where(finite, m, torch.zeros_like(m))
    e = torch.exp(s - m0)
    z = e.sum(dim=-1, keepdim=True)
    pr = torch.where(z > 0, e / torch.where(z > 0, z, torch.ones_like(z)), torch.zeros_like(e))
    lse = torch.where(z[..., 0] > 0, m0[..., 0] + torch.log(z[..., 0]),
                      torch.full_like(z[..., 0], float("-inf")))
    return pr, lse


def _check(q, k, v, cu_q, cu_k):
    assert q.dim() == 3 and k.dim() == 3 and v.dim() == 3, "packed layout [tokens, heads, D]"
    assert k.shape == v.shape and q.shape[2] == k.shape[2]
    hq, hkv = q.shape[1], k.shape[1]
    assert hq % hkv == 0, "query heads must be a multiple of key/value heads (GQA groups)"
    cu_q = [int(x) for x in cu_q]
    cu_k = [int(x) for x in cu_k]
    assert len(cu_q) == len(cu_k) and cu_q[0] == 0 and cu_k[0] == 0
    assert cu_q[-1] == q.shape[0] and cu_k[-1] == k.shape[0]
    return cu_q, cu_k, hq // hkv


def attention(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool,
              slopes: Optional[torch.Tensor] = None):
    """Packed varlen attention. Returns ``(out [T_q, Hq, D], lse [Hq, T_q])`` in float64.

    Definition ([7minutos §4], [yifor 五大] items 1-3 and 5, [gqa-snippets]): each segment is
    attended independently (block-diagonal mask); query head h uses key/value head ``h // R``
    with ``R = Hq / Hkv``; per row, ``out_i = sum_j softmax_j(s_ij) v_j`` over the admissible
    keys, ``lse_i = ln sum_j exp(s_ij)``.
    """
    cu_q, cu_k, r = _check(q, k, v, cu_seqlens_q, cu_seqlens_k)
    q64, k64, v64 = q.to(F64), k.to(F64), v.to(F64)
    t_q, hq, d = q64.shape
    out = torch.zeros((t_q, hq, d), dtype=F64)
    lse = torch.full((hq, t_q), float("-inf"), dtype=F64)
    for s in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
        if q1 == q0:
            continue
        for h in range(hq):
            g = h // r
            sc = _segment_scores(q64[q0:q1, h], k64[k0:k1, g], scale, causal,
                                 None if slopes is None else slopes[h])
            pr, ls = _softmax_rows(sc)
            out[q0:q1, h] = pr @ v64[k0:k1, g]
            lse[h, q0:q1] = ls
    return out, lse


def attention_rows(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool,
                   slopes: Optional[torch.Tensor], rows: Iterable[tuple]):
    """The same definition as :func:`attention`, evaluated only at the given (head, token) pairs.

    ``token`` is a packed (global) query index. Returns ``(out [n, D], lse [n])`` float64. Used
    for sampled checks of workloads too large for the full oracle.
    """
    cu_q, cu_k, r = _check(q, k, v, cu_seqlens_q, cu_seqlens_k)
    rows = list(rows)
    d = q.shape[2]
    out = torch.zeros((len(rows), d), dtype=F64)
    lse = torch.full((len(rows),), float("-inf"), dtype=F64)
    import bisect
    for n, (h, t) in enumerate(rows):
        s = bisect.bisect_right(cu_q, t) - 1
        q0, q1, k0, k1 = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
        i = t - q0
        g = h // r
        qi = q[t:t + 1, h].to(F64)
        ks = k[k0:k1, g].to(F64)
        sc = scale * (qi @ ks.T)[0]
        p_i = i + (k1 - k0) - (q1 - q0)
        j = torch.arange(k1 - k0, dtype=torch.int64)
        if slopes is not None:
            sc = sc - float(slopes[h]) * (p_i - j).abs().to(F64)
        if causal:
            sc = sc.masked_fill(j > p_i, float("-inf"))
        pr, ls = _softmax_rows(sc[None, :])
        out[n] = (pr @ v[k0:k1, g].to(F64))[0]
        lse[n] = ls[0]
    return out, lse


def attention_probs(q, k, v, cu_seqlens_q, cu_seqlens_k, scale, causal, slopes=None):
    """Exposes the softmax matrix P for tiny shapes: a list over segments of ``[Hq, L_q, L_k]``."""
    cu_q, cu_k, r = _check(q, k, v, cu_seqlens_q, cu_seqlens_k)
    q64, k64 = q.to(F64), k.to(F64)
    res = []
    for s in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
        per_head = []
        for h in range(q.shape[1]):
            sc = _segment_scores(q64[q0:q1, h], k64[k0:k1, h // r], scale, causal,
                                 None if slopes is None else slopes[h])
            per_head.append(_softmax_rows(sc)[0])
        res.append(torch.stack(per_head) if per_head else torch.zeros(0))
    return res


def decode(q, k, v, cu_seqlens_k, scale: float, slopes: Optional[torch.Tensor] = None):
    """Single-token decode: request b's one query (q[b], newest token) against its L_k keys.

    It is :func:`attention` with L_q = 1 per segment; the bottom-right position of that query is
    ``p = L_k - 1`` so a causal mask admits every key. Returns ``(out [B, Hq, D], lse [Hq, B])``.
    """
    b = q.shape[0]
    cu_q = list(range(b + 1))
    return attention(q, k, v, cu_q, cu_seqlens_k, scale, causal=True, slopes=slopes)


def lse_merge(lse_parts: torch.Tensor, out_parts: torch.Tensor):
    """Merge partial softmax results over disjoint key chunks by their log-sum-exp.

    ``lse_parts [n, ...]`` and ``out_parts [n, ..., D]`` hold, for chunk c, ``lse_c`` and the
    chunk-normalised ``O_c = sum_{j in c} exp(s_j - lse_c) v_j``. Then
    ``lse = ln sum_c exp(lse_c)`` and ``O = sum_c exp(lse_c - lse) O_c``: the softmax over the
    union of the chunks ([zizhi §1] split-K). Chunks with lse_c = -inf contribute nothing; if all
    are -inf the result is O = 0, lse = -inf.
    """
    lp = lse_parts.to(F64)
    m = lp.max(dim=0).values
    m0 = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
    w = torch.exp(lp - m0)  # [n, ...]
    z = w.sum(dim=0)
    lse = torch.where(z > 0, m0 + torch.log(torch.where(z > 0, z, torch.ones_like(z))),
                      torch.full_like(z, float("-inf")))
    wn = torch.where(z > 0, w / torch.where(z > 0, z, torch.ones_like(z)), torch.zeros_like(w))
    out = (wn[..., None] * out_parts.to(F64)).sum(dim=0)
    return out, lse


def split_attention_chunks(q_row, k_s, v_s, scale, chunk: int, bias=None):
    """Per-chunk (lse_c, O_c) of one query row over keys split into chunks of ``chunk`` keys.

    q_row [D], k_s/v_s [L, D], optional additive ``bias`` [L] (already scaled). Each chunk's
    result is the plain definition restricted to its keys; merging them with :func:`lse_merge`
    must give the unsplit row.
    """
    lses, outs = [], []
    q64 = q_row.to(F64)
    for c0 in range(0, k_s.shape[0], chunk):
        kc = k_s[c0:c0 + chunk].to(F64)
        vc = v_s[c0:c0 + chunk].to(F64)
        sc = scale * (kc @ q64)
        if bias is not None:
            sc = sc + bias[c0:c0 + chunk].to(F64)
        pr, ls = _softmax_rows(sc[None, :])
        lses.append(ls[0])
        outs.append((pr @ vc)[0])
    return torch.stack(lses), torch.stack(outs)


def attention_bruteforce(q, k, v, seqlens_q: Sequence[int], seqlens_k: Sequence[int],
                         scale: float, causal: bool, slopes: Optional[Sequence[float]] = None):
    """Pure-Python loops over an explicit additive mask matrix; tiny shapes only.

    Builds, over the packed token axes, ``mask[t, u] = 0`` if query token t and key token u are
    in the same segment (and, if causal, u's local index <= t's bottom-right position), else
    ``-inf`` ([7minutos §4] block-diagonal / block-diagonal-causal masks); adds the ALiBi term;
    then for each (token, head) takes ``sum_u exp(s - max) v_u / sum_u exp(s - max)`` with plain
    Python floats. Returns nested lists ``out[t][h][d]`` and ``lse[h][t]``.
    """
    tq, hq, d = q.shape
    tk, hkv = k.shape[0], k.shape[1]
    r = hq // hkv
    qf, kf, vf = q.to(F64).tolist(), k.to(F64).tolist(), v.to(F64).tolist()
    seg_q, pos_q, seg_k, pos_k = [], [], [], []
    for s, (lq, lk) in enumerate(zip(seqlens_q, seqlens_k)):
        for i in range(lq):
            seg_q.append(s)
            pos_q.append(i + lk - lq)
        for j in range(lk):
            seg_k.append(s)
            pos_k.append(j)
    neg_inf = float("-inf")
    mask = [[0.0 if (seg_q[t] == seg_k[u] and (not causal or pos_k[u] <= pos_q[t])) else neg_inf
             for u in range(tk)] for t in range(tq)]
    out = [[[0.0] * d for _ in range(hq)] for _ in range(tq)]
    lse = [[neg_inf] * tq for _ in range(hq)]
    for t in range(tq):
        for h in range(hq):
            g = h // r
            sc = []
            for u in range(tk):
                dot = 0.0
                for e in range(d):
                    dot += qf[t][h][e] * kf[u][g][e]
                val = scale * dot + mask[t][u]
                if slopes is not None and mask[t][u] == 0.0:
                    val -= slopes[h] * abs(pos_q[t] - pos_k[u])
                sc.append(val)
            mx = max(sc) if sc else neg_inf
            if mx == neg_inf:
                continue
            w = [math.exp(x - mx) for x in sc]
            z = sum(w)
            lse[h][t] = mx + math.log(z)
            for e in range(d):
                acc = 0.0
                for u in range(tk):
                    acc += w[u] * vf[u][g][e]
                out[t][h][e] = acc / z
    return out, lse


def attention_backward(q, k, v, dout, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool,
                       slopes: Optional[torch.Tensor] = None):
    """Gradients ``(dq, dk, dv)`` of ``L = sum(out * dout)`` for the :func:`attention` definition,
    in float64, with the shapes of q, k and v.

    The definition differentiated by hand, per segment and query head h (key/value head
    g = h // R), with ``P = softmax(S)`` the row softmax of the scaled, biased, masked scores:

    * ``dV_g += P^T dO``                       (out = P V)
    * ``dP = dO V^T``
    * ``dS = P * (dP - rowsum(dO * out))``      (softmax Jacobian: ``rowsum(P * dP) = rowsum(dO * out)``)
    * ``dQ = scale * dS K``,  ``dK_g += scale * dS^T Q``   (S = scale * Q K^T + bias)

    The heads of a group add into the same dK_g, dV_g (the key/value head is shared, [gqa-snippets]).
    Masked entries have P = 0 and contribute nothing; rows without an admissible key have zero
    gradients.
    """
    cu_q, cu_k, r = _check(q, k, v, cu_seqlens_q, cu_seqlens_k)
    assert dout.shape == q.shape
    q64, k64, v64, do64 = q.to(F64), k.to(F64), v.to(F64), dout.to(F64)
    dq = torch.zeros_like(q64)
    dk = torch.zeros_like(k64)
    dv = torch.zeros_like(v64)
    for s in range(len(cu_q) - 1):
        q0, q1, k0, k1 = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
        if q1 == q0 or k1 == k0:
            continue
        for h in range(q.shape[1]):
            g = h // r
            qs, ks, vs, dos = q64[q0:q1, h], k64[k0:k1, g], v64[k0:k1, g], do64[q0:q1, h]
            sc = _segment_scores(qs, ks, scale, causal, None if slopes is None else slopes[h])
            pr, _ = _softmax_rows(sc)
            out = pr @ vs
            dv[k0:k1, g] += pr.T @ dos
            dp = dos @ vs.T
            delta = (dos * out).sum(dim=-1, keepdim=True)
            ds = pr * (dp - delta)
            dq[q0:q1, h] = scale * (ds @ ks)
            dk[k0:k1, g] += scale * (ds.T @ qs)
    return dq, dk, dv


def paged_gather(cache: torch.Tensor, block_table, seqlens_k: Sequence[int]) -> torch.Tensor:
    """The packed ``[sum L_b, H, D]`` keys (or values) of a paged cache ``[num_blocks,
    block_size, H, D]``: request b's key t is ``cache[block_table[b][t // block_size],
    t % block_size]``.

    [7minutos §4] names vLLM-style engines as the users of packed variable-length batches; their
    K/V cache is paged through a per-request block table. The pages do not print that layout:
    this is the plain reading (a gather), used to state paged decode as packed decode.
    """
    bs = cache.shape[1]
    rows = []
    for b, length in enumerate(seqlens_k):
        for t in range(int(length)):
            rows.append(cache[int(block_table[b][t // bs]), t % bs])
    if not rows:
        return cache.new_zeros((0,) + tuple(cache.shape[2:]))
    return torch.stack(rows)


def e4m3_decode(codes: torch.Tensor) -> torch.Tensor:
    """Values of 8-bit E4M3 codes (uint8) in float64, from the format's definition: sign bit 7,
    exponent bits 6..3 with bias 7, mantissa bits 2..0; exponent field 0 is subnormal
    (m/8 * 2^-6); the all-ones exponent with mantissa 7 is NaN (no infinities); largest finite
    value 448. The FP8 forward's attention is this oracle's attention of the decoded values times
    the per-tensor descales ([zizhi §3] "混合精度计算流水线" lists FP8 among the supported
    precisions, with the critical parts of the computation kept in higher precision)."""
    c = codes.to(torch.int64)
    sign = torch.where((c >> 7) & 1 == 1, -1.0, 1.0).to(F64)
    e = (c >> 3) & 0xF
    m = (c & 7).to(F64)
    normal = torch.ldexp(1.0 + m / 8.0, (e - 7).to(torch.int64).to(torch.int32)).to(F64)
    sub = m / 8.0 * 2.0 ** -6
    val = torch.where(e == 0, sub, normal) * sign
    return torch.where((e == 15) & ((c & 7) == 7), torch.full_like(val, float("nan")), val)
