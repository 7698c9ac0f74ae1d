"""Host-side checks of the C ABI: the library loads, exports every entry point include/mea.h
declares, and rejects bad arguments with the documented status before launching anything.
No GPU is needed: every call here fails argument validation before any CUDA call."""
import ctypes
import os
import re

import pytest

from memory_efficient_attention_b200 import _lib
from memory_efficient_attention_b200.build import build_library

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_library()
    return _lib.load()


def declared_entry_points():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(mea_\w+)\s*\(", text))
    return sorted(names)


def test_exports_every_declared_symbol(lib):
    declared = declared_entry_points()
    assert "mea_forward" in declared and "mea_decode_splitkv" in declared
    for name in declared:
        assert hasattr(lib, name), f"libmea.so does not export {name}"
    assert set(_lib.EXPORTS) <= set(declared)


def test_status_strings(lib):
    for rc in range(0, -13, -1):
        s = _lib.status_string(rc)
        assert s and "unknown" not in s
    assert "unknown" in _lib.status_string(-999)
    assert lib.mea_version().decode().startswith("mea")


A = 0x10000  # an aligned dummy address: never dereferenced, validation fails first


def fwd(lib, **kw):
    args = dict(q=A, k=A, v=A, out=A, lse=A, cu_q=A, cu_k=A, n_seqs=1, total_q=8, total_k=8,
                max_q=8, hq=8, hkv=2, d=64, scale=0.125, mask=0, slopes=None, dtype=1, stream=None)
    args.update(kw)
    return lib.mea_forward(args["q"], args["k"], args["v"], args["out"], args["lse"],
                           args["cu_q"], args["cu_k"], args["n_seqs"], args["total_q"],
                           args["total_k"], args["max_q"], args["hq"], args["hkv"], args["d"],
                           args["scale"], args["mask"], args["slopes"], args["dtype"],
                           args["stream"])


@pytest.mark.parametrize("kw,rc", [
    (dict(q=None), _lib.MEA_ERR_NULL),
    (dict(cu_k=None), _lib.MEA_ERR_NULL),
    (dict(n_seqs=0), _lib.MEA_ERR_SHAPE),
    (dict(total_q=-1), _lib.MEA_ERR_SHAPE),
    (dict(max_q=9), _lib.MEA_ERR_SHAPE),
    (dict(hq=6, hkv=4), _lib.MEA_ERR_HEADS),
    (dict(hkv=0), _lib.MEA_ERR_HEADS),
    (dict(d=100), _lib.MEA_ERR_HEAD_DIM),
    (dict(d=264), _lib.MEA_ERR_HEAD_DIM),
    (dict(d=0), _lib.MEA_ERR_HEAD_DIM),
    (dict(dtype=2), _lib.MEA_ERR_DTYPE),
    (dict(mask=2), _lib.MEA_ERR_MASK),
    (dict(scale=float("nan")), _lib.MEA_ERR_SCALE),
    (dict(scale=float("inf")), _lib.MEA_ERR_SCALE),
    (dict(q=A + 8), _lib.MEA_ERR_ALIGN),
    (dict(out=A + 2), _lib.MEA_ERR_ALIGN),
    (dict(lse=A + 2), _lib.MEA_ERR_ALIGN),
])
def test_forward_rejects(lib, kw, rc):
    assert fwd(lib, **kw) == rc


def dec(lib, **kw):
    args = dict(q=A, k=A, v=A, out=A, lse=A, cu_k=A, n_seqs=2, total_k=100, max_k=60, hq=64,
                hkv=8, d=128, scale=0.1, mask=1, slopes=None, dtype=1, ws=A, ws_bytes=1 << 30,
                split=0, stream=None)
    args.update(kw)
    return lib.mea_decode_splitkv(args["q"], args["k"], args["v"], args["out"], args["lse"],
                                  args["cu_k"], args["n_seqs"], args["total_k"], args["max_k"],
                                  args["hq"], args["hkv"], args["d"], args["scale"],
                                  args["mask"], args["slopes"], args["dtype"], args["ws"],
                                  args["ws_bytes"], args["split"], args["stream"])


@pytest.mark.parametrize("kw,rc", [
    (dict(k=None), _lib.MEA_ERR_NULL),
    (dict(n_seqs=0), _lib.MEA_ERR_SHAPE),
    (dict(max_k=101), _lib.MEA_ERR_SHAPE),
    (dict(split=100), _lib.MEA_ERR_SHAPE),
    (dict(hq=12, hkv=8), _lib.MEA_ERR_HEADS),
    (dict(d=36), _lib.MEA_ERR_HEAD_DIM),
    (dict(d=264), _lib.MEA_ERR_HEAD_DIM),
    (dict(dtype=-1), _lib.MEA_ERR_DTYPE),
    (dict(mask=3), _lib.MEA_ERR_MASK),
    (dict(v=A + 4), _lib.MEA_ERR_ALIGN),
])
def test_decode_rejects(lib, kw, rc):
    assert dec(lib, **kw) == rc


def test_decode_workspace_size(lib):
    # partials: (ceil(T_k / chunk) + n_seqs) slots x Hq x (D + 1) fp32, each region 256-aligned
    n = lib.mea_decode_workspace_size(4, 1000, 16, 4, 128, 256)
    slots = -(-1000 // 256) + 4
    o = slots * 16 * 128 * 4
    lse = slots * 16 * 4
    assert n == -(-o // 256) * 256 + -(-lse // 256) * 256
    assert lib.mea_decode_workspace_size(0, 10, 8, 8, 64, 0) == 0
    assert lib.mea_decode_workspace_size(1, 10, 8, 8, 64, 65) == 0
    assert lib.mea_decode_workspace_size(1, 10, 8, 3, 64, 64) == 0
    # too small a workspace is rejected before any launch
    need = lib.mea_decode_workspace_size(2, 100, 64, 8, 128, 64)
    assert dec(lib, ws_bytes=need - 1, split=64) == _lib.MEA_ERR_WORKSPACE
    assert dec(lib, ws=None, split=64) == _lib.MEA_ERR_WORKSPACE
    assert dec(lib, ws=A + 16, split=64) == _lib.MEA_ERR_WORKSPACE


@pytest.mark.parametrize("n_seqs,total_k,hq,hkv,chunk", [
    (64, 1107955, 64, 8, 2048),   # the 64-request decode workload: capped at 2048
    (8, 83113, 64, 8, 2048),      # its first 8 requests: still 2048
    (1, 32768, 64, 8, 2048),      # one long request: 128 items for 148 SMs is enough
    (1, 4096, 64, 8, 256),        # one short request: 2 * 4096 * 8 / 148 = 442 -> 256
    (1, 512, 64, 8, 128),         # the floor
    (2, 20000, 16, 16, 2048),     # MHA (one head per item): 16 items per chunk
])
def test_decode_automatic_chunk(lib, n_seqs, total_k, hq, hkv, chunk):
    # With split_keys = 0 the library takes the largest power of two from 128 to 2048 that keeps
    # about half a (chunk, head block) item per SM or more; head blocks are the largest divisor
    # of Hq/Hkv up to 16. On a host without a GPU the SM count defaults to 148. The workspace
    # size identifies the chunk it picked.
    assert lib.mea_decode_workspace_size(n_seqs, total_k, hq, hkv, 128, 0) == \
        lib.mea_decode_workspace_size(n_seqs, total_k, hq, hkv, 128, chunk)
    if chunk < 2048:
        assert lib.mea_decode_workspace_size(n_seqs, total_k, hq, hkv, 128, 0) != \
            lib.mea_decode_workspace_size(n_seqs, total_k, hq, hkv, 128, 2 * chunk)


def bwd(lib, **kw):
    args = dict(q=A, k=A, v=A, out=A, lse=A, dout=A, dq=A, dk=A, dv=A, cu_q=A, cu_k=A, n_seqs=2,
                total_q=100, total_k=120, max_q=60, max_k=70, hq=8, hkv=2, d=128, scale=0.1,
                mask=1, slopes=None, dtype=1, ws=A, ws_bytes=1 << 20, stream=None)
    args.update(kw)
    return lib.mea_backward(args["q"], args["k"], args["v"], args["out"], args["lse"],
                            args["dout"], args["dq"], args["dk"], args["dv"], args["cu_q"],
                            args["cu_k"], args["n_seqs"], args["total_q"], args["total_k"],
                            args["max_q"], args["max_k"], args["hq"], args["hkv"], args["d"],
                            args["scale"], args["mask"], args["slopes"], args["dtype"],
                            args["ws"], args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("kw,rc", [
    (dict(dout=None), _lib.MEA_ERR_NULL),
    (dict(lse=None), _lib.MEA_ERR_NULL),
    (dict(dk=None), _lib.MEA_ERR_NULL),
    (dict(n_seqs=0), _lib.MEA_ERR_SHAPE),
    (dict(n_seqs=70000), _lib.MEA_ERR_SHAPE),
    (dict(max_q=101), _lib.MEA_ERR_SHAPE),
    (dict(max_k=121), _lib.MEA_ERR_SHAPE),
    (dict(hq=6, hkv=4), _lib.MEA_ERR_HEADS),
    (dict(d=100), _lib.MEA_ERR_HEAD_DIM),
    (dict(d=256), _lib.MEA_ERR_HEAD_DIM),
    (dict(dtype=5), _lib.MEA_ERR_DTYPE),
    (dict(mask=-1), _lib.MEA_ERR_MASK),
    (dict(scale=float("nan")), _lib.MEA_ERR_SCALE),
    (dict(dq=A + 8), _lib.MEA_ERR_ALIGN),
    (dict(dout=A + 2), _lib.MEA_ERR_ALIGN),
    (dict(lse=A + 2), _lib.MEA_ERR_ALIGN),
    (dict(ws=None), _lib.MEA_ERR_WORKSPACE),
    (dict(ws=A + 4), _lib.MEA_ERR_WORKSPACE),
    (dict(ws_bytes=100 * 8 * 4 + 255), _lib.MEA_ERR_WORKSPACE),
])
def test_backward_rejects(lib, kw, rc):
    assert bwd(lib, **kw) == rc


def test_backward_workspace_size(lib):
    assert lib.mea_backward_workspace_size(100, 8) == 2 * (100 + 128) * 8 * 4 + 4096 + 256
    assert lib.mea_backward_workspace_size(0, 8) == 2 * 128 * 8 * 4 + 4096 + 256
    assert lib.mea_backward_workspace_size(-1, 8) == 0
    assert lib.mea_backward_workspace_size(10, 0) == 0


def paged(lib, **kw):
    args = dict(q=A, kc=A, vc=A, table=A, cu_k=A, out=A, lse=A, n_seqs=2, num_blocks=10, bs=16,
                max_blocks=5, total_k=160, max_k=70, hq=64, hkv=8, d=128, scale=0.1, mask=1,
                slopes=None, dtype=1, ws=A, ws_bytes=1 << 30, split=0, stream=None)
    args.update(kw)
    return lib.mea_decode_paged(args["q"], args["kc"], args["vc"], args["table"], args["cu_k"],
                                args["out"], args["lse"], args["n_seqs"], args["num_blocks"],
                                args["bs"], args["max_blocks"], args["total_k"], args["max_k"],
                                args["hq"], args["hkv"], args["d"], args["scale"], args["mask"],
                                args["slopes"], args["dtype"], args["ws"], args["ws_bytes"],
                                args["split"], args["stream"])


@pytest.mark.parametrize("kw,rc", [
    (dict(table=None), _lib.MEA_ERR_NULL),
    (dict(kc=None), _lib.MEA_ERR_NULL),
    (dict(bs=24), _lib.MEA_ERR_SHAPE),
    (dict(bs=8), _lib.MEA_ERR_SHAPE),
    (dict(bs=96), _lib.MEA_ERR_SHAPE),
    (dict(max_blocks=4), _lib.MEA_ERR_SHAPE),        # 4 x 16 < max_k = 70
    (dict(num_blocks=0), _lib.MEA_ERR_SHAPE),
    (dict(max_k=161), _lib.MEA_ERR_SHAPE),
    (dict(split=100), _lib.MEA_ERR_SHAPE),
    (dict(hq=12, hkv=8), _lib.MEA_ERR_HEADS),
    (dict(d=84), _lib.MEA_ERR_HEAD_DIM),
    (dict(d=512), _lib.MEA_ERR_HEAD_DIM),
    (dict(dtype=7), _lib.MEA_ERR_DTYPE),
    (dict(table=A + 2), _lib.MEA_ERR_ALIGN),
    (dict(vc=A + 8), _lib.MEA_ERR_ALIGN),
    (dict(ws=None), _lib.MEA_ERR_WORKSPACE),
    (dict(ws=A + 16), _lib.MEA_ERR_WORKSPACE),
])
def test_paged_decode_rejects(lib, kw, rc):
    assert paged(lib, **kw) == rc


def test_paged_decode_workspace_is_the_decode_workspace(lib):
    need = lib.mea_decode_workspace_size(2, 160, 64, 8, 128, 64)
    assert paged(lib, ws_bytes=need - 1, split=64) == _lib.MEA_ERR_WORKSPACE


def test_python_binding_fails_loudly_without_gpu():
    import torch
    import memory_efficient_attention_b200 as mea
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    q = torch.zeros((4, 2, 64), dtype=torch.float16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    with pytest.raises(mea.MeaError):
        mea.attention_packed(q, q, q, cu, cu, 4)


# ------------------------------------------------------------------ binding argument checks
def test_binding_buffer_checks():
    import torch
    import memory_efficient_attention_b200 as mea
    cpu = torch.device("cpu")
    good = torch.zeros((4, 2, 64), dtype=torch.float16)
    assert mea._check_buffer("out", good, (4, 2, 64), torch.float16, cpu) is good
    for bad, shape, dtype in [(good, (4, 2, 32), torch.float16),       # wrong shape
                              (good, (4, 2, 64), torch.bfloat16),      # wrong dtype
                              (good.transpose(0, 1), (2, 4, 64), torch.float16)]:  # not contiguous
        with pytest.raises(mea.MeaError) as e:
            mea._check_buffer("out", bad, shape, dtype, cpu)
        assert e.value.rc == _lib.MEA_ERR_SHAPE
    with pytest.raises(mea.MeaError) as e:  # a host tensor where a device one is needed
        mea._check_buffer("out", good, (4, 2, 64), torch.float16, torch.device("cuda", 0))
    assert e.value.rc == _lib.MEA_ERR_SHAPE


def test_binding_cu_seqlens_and_device_checks():
    import torch
    import memory_efficient_attention_b200 as mea
    dev = torch.device("cuda", 0)
    for bad in (torch.tensor([0, 4], dtype=torch.int64), torch.tensor([0, 4, 8], dtype=torch.int32)):
        with pytest.raises(mea.MeaError) as e:
            mea._check_cu("cu_seqlens_q", bad, 2, dev)
        assert e.value.rc == _lib.MEA_ERR_SHAPE
    with pytest.raises(mea.MeaError) as e:  # right shape, but host memory
        mea._check_cu("cu_seqlens_q", torch.tensor([0, 4], dtype=torch.int32), 2, dev)
    assert e.value.rc == _lib.MEA_ERR_DEVICE
    with pytest.raises(mea.MeaError) as e:
        mea._on_device(dev, k=torch.zeros(2))
    assert e.value.rc == _lib.MEA_ERR_DEVICE
    mea._on_device(dev, k=None)  # optional tensors are skipped
    with pytest.raises(mea.MeaError) as e:
        mea._check_workspace(torch.zeros(16, dtype=torch.uint8), dev)
    assert e.value.rc == _lib.MEA_ERR_WORKSPACE


def test_binding_decode_rejects_host_tensors_before_any_launch():
    import torch
    import memory_efficient_attention_b200 as mea
    q = torch.zeros((2, 8, 64), dtype=torch.float16)
    kv = torch.zeros((10, 2, 64), dtype=torch.float16)
    cu = torch.tensor([0, 4, 10], dtype=torch.int32)
    for call in (lambda: mea.decode_splitkv(q, kv, kv, cu, 6),
                 lambda: mea.decode_splitkv_noalloc(q, kv, kv, cu, 6, out=torch.empty_like(q))):
        with pytest.raises(mea.MeaError) as e:
            call()
        assert e.value.rc == _lib.MEA_ERR_DEVICE
    with pytest.raises(mea.MeaError) as e:  # k and v shapes disagree
        mea.decode_splitkv(q, kv, kv[:5], cu, 6)
    assert e.value.rc == _lib.MEA_ERR_SHAPE
