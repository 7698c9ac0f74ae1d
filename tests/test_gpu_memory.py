"""Peak memory: the forward and backward allocate nothing; memory is linear in the sequence.

The pages measure the peak memory of this attention against standard attention at long
sequences ("How to Build Memory-Efficient Transformers with xFormers…", section "效能對比"). Here:
one 16384- and one 32768-token segment (32 query / 8 KV heads, D=128, bf16, causal + ALiBi).
Neither call allocates device memory — through torch's allocator or otherwise (device free
memory is unchanged) — so the only memory besides inputs and outputs is the caller's backward
workspace of 2*(T+128)*Hq*4 + 4096 bytes. The score matrix a standard implementation materialises would be
T*T*Hq*4 bytes (34 GB at 32768 tokens).
"""
import pytest
import torch

import memory_efficient_attention_b200 as mea
from mea_workloads import alibi_slope_values

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("t", [16384, 32768])
def test_forward_and_backward_allocate_nothing(t):
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(t)
    q = torch.randn((t, 32, 128), generator=g, device=dev).bfloat16()
    k = torch.randn((t, 8, 128), generator=g, device=dev).bfloat16()
    v = torch.randn((t, 8, 128), generator=g, device=dev).bfloat16()
    dout = torch.randn((t, 32, 128), generator=g, device=dev).bfloat16()
    cu = torch.tensor([0, t], dtype=torch.int32, device=dev)
    sl = alibi_slope_values(32).to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((32, t), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = mea.backward_workspace_size(t, 32)
    assert ws_bytes == 2 * (t + 128) * 32 * 4 + 4096 + 256
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    # warm the library up once (per-kernel attributes, tensor-map encoder lookup)
    mea.attention_packed(q, k, v, cu, cu, t, causal=True, alibi_slopes=sl, out=out, lse=lse)
    mea.attention_packed_backward(q, k, v, out, lse, dout, cu, cu, t, t, causal=True,
                                  alibi_slopes=sl, workspace=ws, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    mea.attention_packed(q, k, v, cu, cu, t, causal=True, alibi_slopes=sl, out=out, lse=lse)
    mea.attention_packed_backward(q, k, v, out, lse, dout, cu, cu, t, t, causal=True,
                                  alibi_slopes=sl, workspace=ws, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.max_memory_allocated() == before
    assert free1 == free0
    assert mea.device_error() == 0
    assert torch.isfinite(out).all() and torch.isfinite(dq).all()
    assert torch.isfinite(dk).all() and torch.isfinite(dv).all()
