"""CUDA graph capture of the hot path through the public binding.

Every entry point launches its kernels on the caller's stream, never synchronises the host and,
given its output and workspace buffers, allocates nothing, so one step of forward, backward,
split-KV decode (workspace and no-allocation forms) and paged decode can be captured once and
replayed. A replay runs the same kernels on the same buffers and none of them uses atomics, so it
must reproduce the eager calls bit for bit; after the inputs are overwritten in place, a replay
must follow the new inputs (the graph holds buffer addresses, not values).
"""
import math

import pytest
import torch

import memory_efficient_attention_b200 as mea
from mea_workloads import alibi_slope_values, cu_seqlens, make_qkv, randn

pytestmark = pytest.mark.gpu

LENS = [300, 77, 1000]
HQ, HKV, D = 8, 2, 128
BS = 16          # paged cache: keys per block


def _fill(seed, q, k, v, dout, qd):
    """Seeded values written in place into the step's input buffers."""
    q2, k2, v2 = make_qkv(LENS, LENS, HQ, HKV, D, torch.bfloat16, seed)
    q.copy_(q2)
    k.copy_(k2)
    v.copy_(v2)
    dout.copy_(randn(tuple(q.shape), seed + 3, torch.bfloat16, device="cuda"))
    qd.copy_(randn(tuple(qd.shape), seed + 4, torch.bfloat16, device="cuda"))


def _paged_layout(lens, seed):
    """Block table of a 16-slot cache holding the packed keys, blocks in a shuffled order."""
    g = torch.Generator().manual_seed(seed)
    nblk = [math.ceil(l / BS) for l in lens]
    total = sum(nblk)
    perm = torch.randperm(total, generator=g)
    table = torch.full((len(lens), max(nblk)), -1, dtype=torch.int32)
    i = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[i:i + n].to(torch.int32)
        i += n
    return table, total


def test_hot_path_replays_in_a_cuda_graph():
    tq = sum(LENS)
    dev = torch.device("cuda")
    q = torch.empty((tq, HQ, D), dtype=torch.bfloat16, device=dev)
    k = torch.empty((tq, HKV, D), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    dout = torch.empty_like(q)
    qd = torch.empty((len(LENS), HQ, D), dtype=torch.bfloat16, device=dev)
    cu = cu_seqlens(LENS).to(dev)
    slopes = alibi_slope_values(HQ).to(dev)
    mx = max(LENS)
    scale = 1.0 / math.sqrt(D)
    table_h, nblocks = _paged_layout(LENS, 5150)
    table = table_h.to(dev)
    k_cache = torch.empty((nblocks, BS, HKV, D), dtype=torch.bfloat16, device=dev)
    v_cache = torch.empty_like(k_cache)

    out = torch.empty_like(q)
    lse = torch.empty((HQ, tq), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bws = torch.empty(mea.backward_workspace_size(tq, HQ), dtype=torch.uint8, device=dev)
    od = torch.empty_like(qd)
    ld = torch.empty((HQ, len(LENS)), dtype=torch.float32, device=dev)
    dws = torch.empty(mea.decode_workspace_size(len(LENS), tq, HQ, HKV, D, 256),
                      dtype=torch.uint8, device=dev)
    odn = torch.empty_like(qd)
    op = torch.empty_like(qd)
    lp = torch.empty_like(ld)
    pws = torch.empty(mea.decode_workspace_size(len(LENS), nblocks * BS, HQ, HKV, D, 256),
                      dtype=torch.uint8, device=dev)
    outs = (out, lse, dq, dk, dv, od, ld, odn, op, lp)

    def scatter_cache():
        # the cache copy of the packed keys (outside the captured step: it is input data)
        c = cu.tolist()
        for b in range(len(LENS)):
            for j in range(math.ceil(LENS[b] / BS)):
                a, e = c[b] + j * BS, min(c[b] + (j + 1) * BS, c[b + 1])
                blk = int(table_h[b, j])
                k_cache[blk, :e - a] = k[a:e]
                v_cache[blk, :e - a] = v[a:e]

    def step():
        mea.attention_packed(q, k, v, cu, cu, mx, causal=True, alibi_slopes=slopes, scale=scale,
                             out=out, lse=lse)
        mea.attention_packed_backward(q, k, v, out, lse, dout, cu, cu, mx, mx, causal=True,
                                      alibi_slopes=slopes, scale=scale, workspace=bws,
                                      dq=dq, dk=dk, dv=dv)
        mea.decode_splitkv(qd, k, v, cu, mx, alibi_slopes=slopes, scale=scale, split_keys=256,
                           workspace=dws, out=od, lse=ld)
        mea.decode_splitkv_noalloc(qd, k, v, cu, mx, out=odn, alibi_slopes=slopes, scale=scale,
                                   split_keys=256)
        mea.decode_paged(qd, k_cache, v_cache, table, cu, mx, alibi_slopes=slopes, scale=scale,
                         workspace=pws, split_keys=256, out=op, lse=lp)

    _fill(5100, q, k, v, dout, qd)
    scatter_cache()
    step()                                   # eager (also sets the kernels' attributes)
    torch.cuda.synchronize()
    eager = [t.clone() for t in outs]

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in outs:                           # the replay must write every output
        t.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert mea.device_error() == 0
    for got, ref in zip(outs, eager):
        assert torch.equal(got, ref), "graph replay differs from the eager call"

    # new inputs in the same buffers: the replay follows them
    _fill(5200, q, k, v, dout, qd)
    scatter_cache()
    g.replay()
    torch.cuda.synchronize()
    replayed = [t.clone() for t in outs]
    assert not torch.equal(replayed[0], eager[0])
    step()
    torch.cuda.synchronize()
    assert mea.device_error() == 0
    for got, ref in zip(replayed, outs):
        assert torch.equal(got, ref), "replay on new inputs differs from the eager call"
    del g
