"""GPU parity of split-KV decode over a paged K/V cache (mea_decode_paged through the C ABI).

The cache is built from packed keys/values: each request's keys go to blocks taken in a shuffled
order; slots of a block past the end of its sequence and every unused block hold NaN, which the
kernel must never let into the result. The oracle is oracle.decode on the packed keys/values
recovered by oracle.paged_gather (pinned by a brute-force scatter). Same tolerance as every
decode test (bf16 8e-3 + 2e-2|ref|, fp16 2e-3 + 1e-2|ref|, lse 1e-3).
"""
import math

import pytest
import torch

import memory_efficient_attention_b200 as mea
import oracle
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv, randn, workload

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: (8e-3, 2e-2), torch.float16: (2e-3, 1e-2)}
LSE_TOL = 1e-3


def _paged(k, v, lens, bs, seed, extra_blocks=5):
    """Scatter packed k/v [sum L, H, D] into a shuffled block cache (NaN elsewhere)."""
    g = torch.Generator().manual_seed(seed)
    nblk = [-(-x // bs) for x in lens]
    num_blocks = sum(nblk) + extra_blocks
    perm = torch.randperm(num_blocks, generator=g)
    h, d = k.shape[1], k.shape[2]
    kc = torch.full((num_blocks, bs, h, d), float("nan"), dtype=k.dtype)
    vc = torch.full((num_blocks, bs, h, d), float("nan"), dtype=v.dtype)
    maxb = max(max(nblk), 1)
    # entries past a request's last block: out-of-range ids (never to be read)
    table = torch.full((len(lens), maxb), 1 << 30, dtype=torch.int32)
    nxt, off = 0, 0
    for b, length in enumerate(lens):
        for j in range(nblk[b]):
            blk = int(perm[nxt])
            nxt += 1
            table[b, j] = blk
            n = min(bs, length - j * bs)
            kc[blk, :n] = k[off + j * bs:off + j * bs + n]
            vc[blk, :n] = v[off + j * bs:off + j * bs + n]
        off += length
    return kc, vc, table


def _run(lens, hq, hkv, d, dtype, bs, alibi, scale, seed, split=0):
    _, k, v = make_qkv([1], lens, hq, hkv, d, dtype, seed)
    q = randn((len(lens), hq, d), seed + 1, dtype)
    kc, vc, table = _paged(k, v, lens, bs, seed + 2)
    slopes = alibi_slope_values(hq) if alibi else None
    cu = cu_seqlens(lens)
    out, lse = mea.decode_paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), cu.cuda(),
                                max(lens), alibi_slopes=None if slopes is None else slopes.cuda(),
                                scale=scale, split_keys=split)
    torch.cuda.synchronize()
    assert mea.device_error() == 0
    return (q, k, v, kc, vc, table, cu, slopes), out.cpu(), lse.cpu()


def _close(out, ref, lse, lref, dtype, what):
    atol, rtol = TOL[dtype]
    o = out.double()
    assert not torch.isnan(o).any(), f"{what}: NaN in output"
    bad = (o - ref).abs() > atol + rtol * ref.abs()
    assert not bad.any(), f"{what}: max err {float((o - ref).abs().max()):.3e}"
    fin = torch.isfinite(lref)
    assert torch.equal(torch.isfinite(lse), fin), f"{what}: -inf pattern of lse differs"
    assert float((lse.double()[fin] - lref[fin]).abs().max()) <= LSE_TOL, f"{what}: lse differs"


def _check(lens, hq, hkv, d, dtype, bs, alibi, scale, seed, split=0):
    (q, k, v, kc, vc, table, cu, slopes), out, lse = _run(lens, hq, hkv, d, dtype, bs, alibi,
                                                          scale, seed, split)
    kp = oracle.paged_gather(kc, table.tolist(), lens)
    vp = oracle.paged_gather(vc, table.tolist(), lens)
    assert torch.equal(kp, k) and torch.equal(vp, v)
    ref, lref = oracle.decode(q, kp, vp, cu.tolist(), scale,
                              None if slopes is None else slopes.double())
    _close(out, ref, lse, lref, dtype, f"lens {lens[:6]} bs {bs} H{hq}/{hkv} D{d} {dtype} "
                                       f"alibi={alibi} split={split}")


@pytest.mark.parametrize("bs", [16, 32, 64, 128, 256])
def test_paged_decode_block_sizes(bs):
    _check([1, 15, 16, 17, 64, 65, 300, 1000], 16, 2, 128, torch.bfloat16, bs, False,
           1 / math.sqrt(128), 1100 + bs)


@pytest.mark.parametrize("d", [40, 64, 96, 128, 256])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("alibi", [False, True])
def test_paged_decode_dtypes_dims_alibi(d, dtype, alibi):
    _check([33, 250, 129, 7], 8, 8, d, dtype, 16, alibi, 0.1, 1200)


@pytest.mark.parametrize("d", [64, 96, 256])
@pytest.mark.parametrize("bs", [32, 64, 128])
def test_paged_decode_dims_block_sizes(d, bs):
    # head dims 64 and 256 take one 5-D box per block (32 or 64 rows of every atom); 96 the
    # per-atom 4-D boxes
    _check([1, 31, 32, 33, 200, 700], 16, 2, d, torch.bfloat16, bs, True, 1 / math.sqrt(d),
           1300 + d + bs)


@pytest.mark.parametrize("split", [64, 128, 512])
def test_paged_decode_explicit_chunks(split):
    _check([2000, 70, 1, 513], 64, 8, 128, torch.bfloat16, 16, True, 0.088, 1300, split)


def test_paged_decode_matches_packed_decode():
    lens = [513, 64, 4000, 1, 2500, 700]
    (q, k, v, kc, vc, table, cu, slopes), out, lse = _run(lens, 64, 8, 128, torch.bfloat16, 32,
                                                          True, 0.09, 1400)
    o2, l2 = mea.decode_splitkv(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), max(lens),
                                alibi_slopes=slopes.cuda(), scale=0.09)
    torch.cuda.synchronize()
    _close(out, o2.cpu().double(), lse, l2.cpu().double(), torch.bfloat16, "paged vs packed")


def test_paged_decode_workload_full_size_sampled():
    """The 64-request decode workload (KV lengths U[512, 32768], 64/8 heads, D=128, bf16) from a
    paged cache of 16-slot blocks, through the CUDA path at full size; the oracle checks four
    requests (each request's output depends only on its own keys)."""
    w = workload(4)
    lens = w.seqlens_k
    (q, k, v, kc, vc, table, cu, slopes), out, lse = _run(lens, 64, 8, 128, torch.bfloat16, 16,
                                                          False, w.scale, w.seed)
    c = cu.tolist()
    for b in (0, 7, 31, 63):
        ref, lref = oracle.decode(q[b:b + 1], k[c[b]:c[b + 1]], v[c[b]:c[b + 1]],
                                  [0, c[b + 1] - c[b]], w.scale)
        _close(out[b:b + 1], ref, lse[:, b:b + 1], lref, torch.bfloat16, f"request {b}")
