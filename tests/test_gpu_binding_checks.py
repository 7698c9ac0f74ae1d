"""The Python binding rejects caller-provided buffers that do not match before anything is
launched: the library writes through their pointers with sizes taken from the other arguments,
so a wrong shape, dtype, device or layout would otherwise write out of bounds."""
import pytest
import torch

import memory_efficient_attention_b200 as mea
from memory_efficient_attention_b200 import _lib

pytestmark = pytest.mark.gpu


def _inputs():
    q = torch.zeros((8, 4, 64), dtype=torch.float16, device="cuda")
    kv = torch.zeros((8, 2, 64), dtype=torch.float16, device="cuda")
    cu = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    return q, kv, cu


@pytest.mark.parametrize("kw,rc", [
    (dict(out=torch.zeros((8, 4, 32), dtype=torch.float16)), _lib.MEA_ERR_SHAPE),
    (dict(out="wrong_dtype"), _lib.MEA_ERR_SHAPE),
    (dict(out="strided"), _lib.MEA_ERR_SHAPE),
    (dict(lse="short"), _lib.MEA_ERR_SHAPE),
    (dict(cu="host"), _lib.MEA_ERR_DEVICE),
    (dict(k="host"), _lib.MEA_ERR_DEVICE),
])
def test_forward_rejects_mismatched_buffers(kw, rc):
    q, kv, cu = _inputs()
    out = lse = None
    k = kv
    cu_q = cu
    if "out" in kw:
        o = kw["out"]
        if o == "wrong_dtype":
            out = torch.zeros((8, 4, 64), dtype=torch.bfloat16, device="cuda")
        elif o == "strided":
            out = torch.zeros((4, 8, 64), dtype=torch.float16, device="cuda").transpose(0, 1)
        else:
            out = o.cuda()
    if kw.get("lse") == "short":
        lse = torch.zeros((4, 7), dtype=torch.float32, device="cuda")
    if kw.get("cu") == "host":
        cu_q = cu.cpu()
    if kw.get("k") == "host":
        k = kv.cpu()
    with pytest.raises(mea.MeaError) as e:
        mea.attention_packed(q, k, kv, cu_q, cu, 8, out=out, lse=lse)
    assert e.value.rc == rc
    assert mea.device_error() == 0


def test_decode_and_backward_reject_mismatched_buffers():
    q, kv, cu = _inputs()
    dq = torch.zeros((1, 4, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(mea.MeaError) as e:
        mea.decode_splitkv(dq, kv, kv, cu, 8, out=torch.zeros((1, 4, 32), dtype=torch.float16,
                                                               device="cuda"))
    assert e.value.rc == _lib.MEA_ERR_SHAPE
    out, lse = mea.attention_packed(q, kv, kv, cu, cu, 8)
    with pytest.raises(mea.MeaError) as e:
        mea.attention_packed_backward(q, kv, kv, out, lse, torch.zeros_like(q), cu, cu, 8, 8,
                                      dk=torch.zeros_like(q))
    assert e.value.rc == _lib.MEA_ERR_SHAPE
    torch.cuda.synchronize()
    assert mea.device_error() == 0
