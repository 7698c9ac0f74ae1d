"""memory_efficient_attention_b200 — exact memory-efficient attention on B200 (sm_100a).

A thin PyTorch binding over libmea.so (C ABI in include/mea.h). PyTorch supplies device memory
and the current CUDA stream; every step of the computation runs in the library's kernels. There
is no CPU path: calling any op without a built library or without an sm_100 GPU raises.

Public API (names follow the pages' vocabulary):

* :func:`memory_efficient_attention` — ``(q, k, v, attn_bias=None, scale=None)`` on BMHK
  ``[B, M, H, K]`` or BMGHK ``[B, M, G, Hq, K]`` tensors, the call of the 7minutos page's packed
  and grouped examples; ``attn_bias`` is a :class:`BlockDiagonalMask`,
  :class:`BlockDiagonalCausalMask` or :class:`LowerTriangularMask`, optionally with ALiBi slopes.
* :func:`attention_packed` — the raw packed-varlen call ``[T, H, D]`` with ``cu_seqlens``;
  :func:`attention_packed_fp8` the same with e4m3 inputs; :func:`attention_packed_backward` its
  gradients.
* :func:`decode_splitkv` — one query token per request against a packed KV cache;
  :func:`decode_paged` against a block cache; :func:`decode_splitkv_noalloc` without a workspace.
* :func:`alibi_slopes` — ``2^(-8(h+1)/H)``.

Caller-provided outputs and workspaces must be contiguous tensors of exactly the documented
shape, dtype and device: the library writes through their pointers with sizes taken from the
other arguments, so a mismatch raises here instead.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence

import torch

from . import _lib
from ._lib import MeaError  # noqa: F401

__all__ = [
    "memory_efficient_attention", "attention_packed", "attention_packed_fp8",
    "attention_packed_backward", "backward_workspace_size", "decode_splitkv", "decode_paged",
    "decode_splitkv_noalloc", "decode_workspace_size", "wait_selftest", "alibi_slopes",
    "BlockDiagonalMask", "BlockDiagonalCausalMask", "LowerTriangularMask", "device_error",
    "set_wait_timeout_ns", "MeaError", "library_path",
]

library_path = _lib.LIB_PATH


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float16:
        return _lib.MEA_F16
    if t == torch.bfloat16:
        return _lib.MEA_BF16
    raise MeaError(_lib.MEA_ERR_DTYPE, f"dtype {t}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _on_device(device: torch.device, **tensors) -> None:
    """Each given tensor (None is skipped) must be a CUDA tensor on ``device``: the kernels
    dereference every pointer on that GPU."""
    for name, t in tensors.items():
        if t is not None and (not t.is_cuda or t.device != device):
            raise MeaError(_lib.MEA_ERR_DEVICE, f"{name} must be a CUDA tensor on {device}")


def _check_buffer(name: str, t: torch.Tensor, shape, dtype: torch.dtype,
                  device: torch.device) -> torch.Tensor:
    """A caller-provided output must match exactly (the library writes through its pointer)."""
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device \
            or not t.is_contiguous():
        raise MeaError(_lib.MEA_ERR_SHAPE,
                       f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} "
                       f"on {device}")
    return t


def _check_workspace(t: torch.Tensor, device: torch.device) -> int:
    """A caller-provided workspace: contiguous, on ``device``; returns its size in bytes (the
    library checks that it is large enough)."""
    if t.device != device or not t.is_contiguous():
        raise MeaError(_lib.MEA_ERR_WORKSPACE, f"workspace must be contiguous on {device}")
    return t.numel() * t.element_size()


def _check_cu(name: str, t: torch.Tensor, n: int, device: torch.device) -> torch.Tensor:
    """cu_seqlens: int32 ``[n]`` on ``device`` (made contiguous)."""
    if t.dtype != torch.int32 or t.dim() != 1 or t.numel() != n:
        raise MeaError(_lib.MEA_ERR_SHAPE, f"{name} must be int32 [{n}]")
    _on_device(device, **{name: t})
    return t.contiguous()


def alibi_slopes(n_heads: int, device=None) -> torch.Tensor:
    """fp32 ALiBi slopes ``2^(-8(h+1)/H)`` for h = 0..H-1."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / n_heads) for h in range(n_heads)],
                        dtype=torch.float32, device=device)


def _cu(seqlens: Sequence[int], device) -> torch.Tensor:
    c = [0]
    for s in seqlens:
        c.append(c[-1] + int(s))
    return torch.tensor(c, dtype=torch.int32, device=device)


def attention_packed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                     cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, max_seqlen_q: int,
                     causal: bool = False, alibi_slopes: Optional[torch.Tensor] = None,
                     scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, return_lse: bool = True):
    """Packed varlen attention: q ``[T_q, Hq, D]``, k/v ``[T_k, Hkv, D]``, cu_seqlens int32 on
    the same device. Returns ``(out [T_q, Hq, D], lse [Hq, T_q] fp32 or None)``."""
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3:
        raise MeaError(_lib.MEA_ERR_SHAPE, "packed tensors must be [tokens, heads, head_dim]")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise MeaError(_lib.MEA_ERR_DEVICE, "tensors must live on the GPU")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    tq, hq, d = q.shape
    tk, hkv, _ = k.shape
    if k.shape != v.shape or k.shape[2] != d or q.dtype != k.dtype or k.dtype != v.dtype:
        raise MeaError(_lib.MEA_ERR_SHAPE, "q/k/v shapes or dtypes disagree")
    _on_device(q.device, k=k, v=v)
    n_seqs = cu_seqlens_q.numel() - 1
    cu_seqlens_q = _check_cu("cu_seqlens_q", cu_seqlens_q, n_seqs + 1, q.device)
    cu_seqlens_k = _check_cu("cu_seqlens_k", cu_seqlens_k, n_seqs + 1, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_buffer("out", out, (tq, hq, d), q.dtype, q.device)
    if return_lse and lse is None:
        lse = torch.empty((hq, tq), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _check_buffer("lse", lse, (hq, tq), torch.float32, q.device)
    if alibi_slopes is not None:
        alibi_slopes = alibi_slopes.to(device=q.device, dtype=torch.float32).contiguous()
    rc = _lib.load().mea_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
        n_seqs, tq, tk, int(max_seqlen_q), hq, hkv, d, float(scale),
        _lib.MEA_MASK_CAUSAL if causal else _lib.MEA_MASK_NONE, _ptr(alibi_slopes),
        _dtype_code(q.dtype), _stream(q.device))
    _lib.check(rc, "mea_forward")
    return out, lse


def attention_packed_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, max_seqlen_q: int,
                         causal: bool = False, alibi_slopes: Optional[torch.Tensor] = None,
                         scale: Optional[float] = None, q_descale: float = 1.0,
                         k_descale: float = 1.0, v_descale: float = 1.0,
                         out_dtype: torch.dtype = torch.bfloat16,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """FP8 forward: q, k, v ``torch.float8_e4m3fn`` (D = 128) with per-tensor descales; returns
    ``(out [T_q, Hq, D] out_dtype, lse [Hq, T_q] fp32)``."""
    for t in (q, k, v):
        if not t.is_cuda or t.dtype != torch.float8_e4m3fn:
            raise MeaError(_lib.MEA_ERR_DTYPE, "q, k, v must be float8_e4m3fn on the GPU")
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or k.shape[2] != q.shape[2]:
        raise MeaError(_lib.MEA_ERR_SHAPE, "q [T_q, Hq, D], k/v [T_k, Hkv, D]")
    _on_device(q.device, k=k, v=v)
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    tq, hq, d = q.shape
    tk, hkv, _ = k.shape
    n_seqs = cu_seqlens_q.numel() - 1
    cu_seqlens_q = _check_cu("cu_seqlens_q", cu_seqlens_q, n_seqs + 1, q.device)
    cu_seqlens_k = _check_cu("cu_seqlens_k", cu_seqlens_k, n_seqs + 1, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((tq, hq, d), dtype=out_dtype, device=q.device)
    else:
        _check_buffer("out", out, (tq, hq, d), out.dtype, q.device)
    if lse is None:
        lse = torch.empty((hq, tq), dtype=torch.float32, device=q.device)
    else:
        _check_buffer("lse", lse, (hq, tq), torch.float32, q.device)
    if alibi_slopes is not None:
        alibi_slopes = alibi_slopes.to(device=q.device, dtype=torch.float32).contiguous()
    rc = _lib.load().mea_forward_fp8(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
        n_seqs, tq, tk, int(max_seqlen_q), hq, hkv, d, float(scale),
        _lib.MEA_MASK_CAUSAL if causal else _lib.MEA_MASK_NONE, _ptr(alibi_slopes),
        float(q_descale), float(k_descale), float(v_descale), _dtype_code(out.dtype),
        _stream(q.device))
    _lib.check(rc, "mea_forward_fp8")
    return out, lse


def backward_workspace_size(total_q: int, n_heads_q: int) -> int:
    return int(_lib.load().mea_backward_workspace_size(int(total_q), int(n_heads_q)))


def attention_packed_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              out: torch.Tensor, lse: torch.Tensor, dout: torch.Tensor,
                              cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                              max_seqlen_q: int, max_seqlen_k: int, causal: bool = False,
                              alibi_slopes: Optional[torch.Tensor] = None,
                              scale: Optional[float] = None,
                              workspace: Optional[torch.Tensor] = None,
                              dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                              dv: Optional[torch.Tensor] = None):
    """Gradients ``(dq, dk, dv)`` of ``sum(out * dout)`` for :func:`attention_packed` called with
    the same arguments; ``out`` and ``lse`` are that call's results. ``dq``/``dk``/``dv`` may be
    given as preallocated contiguous outputs."""
    for t in (q, k, v, out, dout):
        if not t.is_cuda:
            raise MeaError(_lib.MEA_ERR_DEVICE, "tensors must live on the GPU")
    _on_device(q.device, k=k, v=v, out=out, lse=lse, dout=dout)
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or k.shape[2] != q.shape[2] \
            or k.dtype != q.dtype or v.dtype != q.dtype:
        raise MeaError(_lib.MEA_ERR_SHAPE, "q [T_q, Hq, D], k/v [T_k, Hkv, D] of one dtype")
    q, k, v, out, dout = (t.contiguous() for t in (q, k, v, out, dout))
    lse = lse.contiguous()
    tq, hq, d = q.shape
    tk, hkv, _ = k.shape
    if dout.shape != q.shape or out.shape != q.shape or lse.shape != (hq, tq) \
            or lse.dtype != torch.float32 or dout.dtype != q.dtype or out.dtype != q.dtype:
        raise MeaError(_lib.MEA_ERR_SHAPE, "out/dout must match q; lse must be fp32 [Hq, T_q]")
    n_seqs = cu_seqlens_q.numel() - 1
    cu_seqlens_q = _check_cu("cu_seqlens_q", cu_seqlens_q, n_seqs + 1, q.device)
    cu_seqlens_k = _check_cu("cu_seqlens_k", cu_seqlens_k, n_seqs + 1, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if alibi_slopes is not None:
        alibi_slopes = alibi_slopes.to(device=q.device, dtype=torch.float32).contiguous()
    need = backward_workspace_size(tq, hq)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = _check_workspace(workspace, q.device)
    dq = torch.empty_like(q) if dq is None else _check_buffer("dq", dq, q.shape, q.dtype, q.device)
    dk = torch.empty_like(k) if dk is None else _check_buffer("dk", dk, k.shape, k.dtype, q.device)
    dv = torch.empty_like(v) if dv is None else _check_buffer("dv", dv, v.shape, v.dtype, q.device)
    rc = _lib.load().mea_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), n_seqs, tq, tk, int(max_seqlen_q),
        int(max_seqlen_k), hq, hkv, d, float(scale),
        _lib.MEA_MASK_CAUSAL if causal else _lib.MEA_MASK_NONE, _ptr(alibi_slopes),
        _dtype_code(q.dtype), _ptr(workspace), ws_bytes, _stream(q.device))
    _lib.check(rc, "mea_backward")
    return dq, dk, dv


def decode_workspace_size(n_seqs: int, total_k: int, n_heads_q: int, n_heads_kv: int,
                          head_dim: int, split_keys: int = 0) -> int:
    return int(_lib.load().mea_decode_workspace_size(n_seqs, total_k, n_heads_q, n_heads_kv,
                                                     head_dim, split_keys))


def decode_splitkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_k: torch.Tensor,
                   max_seqlen_k: int, alibi_slopes: Optional[torch.Tensor] = None,
                   scale: Optional[float] = None, split_keys: int = 0,
                   workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                   lse: Optional[torch.Tensor] = None, return_lse: bool = True):
    """Single-token decode: q ``[B, Hq, D]`` against packed k/v ``[T_k, Hkv, D]``.
    Returns ``(out [B, Hq, D], lse [Hq, B] or None)``."""
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or k.shape[2] != q.shape[2]:
        raise MeaError(_lib.MEA_ERR_SHAPE, "q [B, Hq, D], k/v [T_k, Hkv, D]")
    if not q.is_cuda:
        raise MeaError(_lib.MEA_ERR_DEVICE, "tensors must live on the GPU")
    _on_device(q.device, k=k, v=v)
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    b, hq, d = q.shape
    tk, hkv, _ = k.shape
    cu_seqlens_k = _check_cu("cu_seqlens_k", cu_seqlens_k, b + 1, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ws_bytes = decode_workspace_size(b, tk, hq, hkv, d, split_keys)
    if ws_bytes == 0:
        raise MeaError(_lib.MEA_ERR_SHAPE, "mea_decode_workspace_size")
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_buffer("out", out, (b, hq, d), q.dtype, q.device)
    if return_lse and lse is None:
        lse = torch.empty((hq, b), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _check_buffer("lse", lse, (hq, b), torch.float32, q.device)
    if alibi_slopes is not None:
        alibi_slopes = alibi_slopes.to(device=q.device, dtype=torch.float32).contiguous()
    rc = _lib.load().mea_decode_splitkv(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_k), b, tk,
        int(max_seqlen_k), hq, hkv, d, float(scale), _lib.MEA_MASK_CAUSAL, _ptr(alibi_slopes),
        _dtype_code(q.dtype), _ptr(workspace), _check_workspace(workspace, q.device),
        int(split_keys), _stream(q.device))
    _lib.check(rc, "mea_decode_splitkv")
    return out, lse


def decode_paged(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 block_table: torch.Tensor, cu_seqlens_k: torch.Tensor, max_seqlen_k: int,
                 alibi_slopes: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                 workspace: Optional[torch.Tensor] = None, split_keys: int = 0,
                 total_k_bound: Optional[int] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None):
    """Split-KV decode over a paged cache ``[num_blocks, block_size, Hkv, D]`` with an int32
    ``block_table [n_seqs, max_blocks]``. Returns ``(out [n_seqs, Hq, D], lse [Hq, n_seqs])``."""
    for t in (q, k_cache, v_cache, block_table, cu_seqlens_k):
        if not t.is_cuda:
            raise MeaError(_lib.MEA_ERR_DEVICE, "tensors must live on the GPU")
    q = q.contiguous()
    k_cache, v_cache = k_cache.contiguous(), v_cache.contiguous()
    block_table = block_table.contiguous()
    n, hq, d = q.shape
    nb, bs, hkv, _ = k_cache.shape
    if v_cache.shape != k_cache.shape or block_table.dtype != torch.int32 \
            or block_table.dim() != 2 or block_table.shape[0] != n or k_cache.shape[3] != d:
        raise MeaError(_lib.MEA_ERR_SHAPE, "cache / block table shapes disagree")
    _on_device(q.device, k_cache=k_cache, v_cache=v_cache, block_table=block_table)
    cu_seqlens_k = _check_cu("cu_seqlens_k", cu_seqlens_k, n + 1, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    total = int(total_k_bound) if total_k_bound is not None else nb * bs
    if workspace is None:
        workspace = torch.empty(decode_workspace_size(n, total, hq, hkv, d, split_keys),
                                dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_buffer("out", out, (n, hq, d), q.dtype, q.device)
    if lse is None:
        lse = torch.empty((hq, n), dtype=torch.float32, device=q.device)
    else:
        _check_buffer("lse", lse, (hq, n), torch.float32, q.device)
    if alibi_slopes is not None:
        alibi_slopes = alibi_slopes.to(device=q.device, dtype=torch.float32).contiguous()
    rc = _lib.load().mea_decode_paged(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(cu_seqlens_k), _ptr(out),
        _ptr(lse), n, nb, bs, block_table.shape[1], total, int(max_seqlen_k), hq, hkv, d,
        float(scale), _lib.MEA_MASK_CAUSAL, _ptr(alibi_slopes), _dtype_code(q.dtype),
        _ptr(workspace), _check_workspace(workspace, q.device), int(split_keys),
        _stream(q.device))
    _lib.check(rc, "mea_decode_paged")
    return out, lse


def decode_splitkv_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           cu_seqlens_k: torch.Tensor, max_seqlen_k: int, out: torch.Tensor,
                           lse: Optional[torch.Tensor] = None,
                           alibi_slopes: Optional[torch.Tensor] = None,
                           scale: Optional[float] = None, split_keys: int = 0):
    """:func:`decode_splitkv` for callers that cannot allocate device memory.

    The split-KV partials go to a fixed array inside the library instead of a workspace, so this
    call performs no device allocation of its own: the caller passes the output buffers (``out``
    ``[B, Hq, D]``, optional ``lse`` ``[Hq, B]`` fp32) along with the inputs. Calls that overlap on
    the GPU share that array and race; keep them ordered on one stream. Raises ``MeaError`` with
    ``MEA_ERR_SCRATCH_LIMIT`` when the partials cannot fit in the array.

    Nothing is copied or converted here either (a copy would allocate device memory): every
    tensor, ``cu_seqlens_k`` and ``alibi_slopes`` included, must already be contiguous, of the
    documented dtype and on q's GPU, otherwise ``MeaError`` is raised.
    """
    if q.dim() != 3 or k.dim() != 3 or k.shape != v.shape or k.shape[2] != q.shape[2]:
        raise MeaError(_lib.MEA_ERR_SHAPE, "q [B, Hq, D], k/v [T_k, Hkv, D]")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise MeaError(_lib.MEA_ERR_DTYPE, "q, k and v must share one dtype")
    if not q.is_cuda:
        raise MeaError(_lib.MEA_ERR_DEVICE, "tensors must live on the GPU")
    _on_device(q.device, k=k, v=v, cu_seqlens_k=cu_seqlens_k, alibi_slopes=alibi_slopes)
    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens_k", cu_seqlens_k),
                    ("alibi_slopes", alibi_slopes)):
        if t is not None and not t.is_contiguous():
            raise MeaError(_lib.MEA_ERR_SHAPE, f"{name} must be contiguous (no copy is made)")
    b, hq, d = q.shape
    tk, hkv, _ = k.shape
    _check_cu("cu_seqlens_k", cu_seqlens_k, b + 1, q.device)
    _check_buffer("out", out, (b, hq, d), q.dtype, q.device)
    if lse is not None:
        _check_buffer("lse", lse, (hq, b), torch.float32, q.device)
    if alibi_slopes is not None and (alibi_slopes.dtype != torch.float32
                                     or tuple(alibi_slopes.shape) != (hq,)):
        raise MeaError(_lib.MEA_ERR_SHAPE,
                       f"alibi_slopes must be a float32 [{hq}] tensor (no conversion is made)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = _lib.load().mea_decode_splitkv_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_k), b, tk,
        int(max_seqlen_k), hq, hkv, d, float(scale), _lib.MEA_MASK_CAUSAL, _ptr(alibi_slopes),
        _dtype_code(q.dtype), int(split_keys), _stream(q.device))
    _lib.check(rc, "mea_decode_splitkv_noalloc")
    return out, lse


# ------------------------------------------------------------------------------------------
# Attention-bias descriptors (host objects, like the masks of the 7minutos page, section 4).
# ------------------------------------------------------------------------------------------
class BlockDiagonalMask:
    """Packed segments that never attend to one another. ``q_seqlen[i]`` queries of segment i
    attend to its ``kv_seqlen[i]`` keys (bottom-right aligned when causal)."""
    causal = False

    def __init__(self, q_seqlen: Sequence[int], kv_seqlen: Optional[Sequence[int]] = None,
                 alibi_slopes: Optional[torch.Tensor] = None):
        self.q_seqlen = [int(x) for x in q_seqlen]
        self.kv_seqlen = [int(x) for x in (kv_seqlen if kv_seqlen is not None else q_seqlen)]
        if len(self.kv_seqlen) != len(self.q_seqlen):
            raise ValueError("q_seqlen and kv_seqlen must have the same length")
        self.alibi_slopes = alibi_slopes
        self._dev = {}

    @classmethod
    def from_seqlens(cls, q_seqlen: Sequence[int], kv_seqlen: Optional[Sequence[int]] = None,
                     alibi_slopes: Optional[torch.Tensor] = None):
        return cls(q_seqlen, kv_seqlen, alibi_slopes)

    def cu_seqlens(self, device):
        key = str(device)
        if key not in self._dev:
            self._dev[key] = (_cu(self.q_seqlen, device), _cu(self.kv_seqlen, device))
        return self._dev[key]

    def split(self, out: torch.Tensor) -> List[torch.Tensor]:
        """Splits a packed ``[1, T, ...]`` output back into per-segment ``[1, L_i, ...]`` views."""
        return list(torch.split(out, self.q_seqlen, dim=1))


class BlockDiagonalCausalMask(BlockDiagonalMask):
    """Block-diagonal plus the implicit lower-triangular (bottom-right) mask in each segment."""
    causal = True


class LowerTriangularMask:
    """Causal mask over each batch row of a BMHK / BMGHK call."""
    causal = True

    def __init__(self, alibi_slopes: Optional[torch.Tensor] = None):
        self.alibi_slopes = alibi_slopes


def memory_efficient_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                               attn_bias=None, scale: Optional[float] = None) -> torch.Tensor:
    """Exact attention on BMHK ``[B, M, H, K]`` or BMGHK ``[B, M, G, Hq, K]`` tensors;
    differentiable (the backward runs mea_backward) when an input requires grad.

    BMGHK: k/v are ``[B, Mk, G, 1, K]`` (one KV head per group, shared by the group's Hq query
    heads) and the output is ``[B, M, G, Hq, K]``. With a block-diagonal mask B must be 1 and the
    token axis is the packed concatenation of the mask's segments.
    """
    if q.dim() == 5:
        b, m, g, hq, kd = q.shape
        if k.dim() != 5 or k.shape[3] != 1 or v.shape != k.shape or k.shape[2] != g:
            raise MeaError(_lib.MEA_ERR_SHAPE, "BMGHK expects k/v [B, Mk, G, 1, K]")
        mk = k.shape[1]
        qp = q.reshape(b * m, g * hq, kd)
        kp = k.reshape(b * mk, g, kd)
        vp = v.reshape(b * mk, g, kd)
        out = _bmhk_packed(qp, kp, vp, b, m, mk, attn_bias, scale)
        return out.reshape(b, m, g, hq, kd)
    if q.dim() != 4:
        raise MeaError(_lib.MEA_ERR_SHAPE, "expected BMHK [B, M, H, K] or BMGHK [B, M, G, Hq, K]")
    b, m, h, kd = q.shape
    mk = k.shape[1]
    out = _bmhk_packed(q.reshape(b * m, h, kd), k.reshape(b * mk, k.shape[2], kd),
                       v.reshape(b * mk, v.shape[2], kd), b, m, mk, attn_bias, scale)
    return out.reshape(b, m, h, kd)


def _bmhk_packed(qp, kp, vp, b, m, mk, attn_bias, scale):
    slopes = getattr(attn_bias, "alibi_slopes", None)
    if isinstance(attn_bias, BlockDiagonalMask):
        if b != 1:
            raise MeaError(_lib.MEA_ERR_SHAPE, "block-diagonal masks need B == 1 (packed tokens)")
        if sum(attn_bias.q_seqlen) != m or sum(attn_bias.kv_seqlen) != mk:
            raise MeaError(_lib.MEA_ERR_SHAPE, "mask seqlens do not sum to the token count")
        cu_q, cu_k = attn_bias.cu_seqlens(qp.device)
        max_q = max(attn_bias.q_seqlen) if attn_bias.q_seqlen else 0
        causal = attn_bias.causal
    else:
        cu_q = torch.arange(0, (b + 1) * m, m, dtype=torch.int32, device=qp.device)
        cu_k = torch.arange(0, (b + 1) * mk, mk, dtype=torch.int32, device=qp.device)
        max_q = m
        causal = isinstance(attn_bias, LowerTriangularMask)
        if attn_bias is not None and not isinstance(attn_bias, LowerTriangularMask):
            raise MeaError(_lib.MEA_ERR_MASK, f"unsupported attn_bias {type(attn_bias).__name__}")
    max_k = max(attn_bias.kv_seqlen) if isinstance(attn_bias, BlockDiagonalMask) and \
        attn_bias.kv_seqlen else mk
    if torch.is_grad_enabled() and (qp.requires_grad or kp.requires_grad or vp.requires_grad):
        return _PackedAttention.apply(qp, kp, vp, cu_q, cu_k, max_q, max_k, causal, slopes, scale)
    out, _ = attention_packed(qp, kp, vp, cu_q, cu_k, max_q, causal=causal, alibi_slopes=slopes,
                              scale=scale, return_lse=False)
    return out


class _PackedAttention(torch.autograd.Function):
    """Packed attention with its gradients: forward through mea_forward (keeping out and lse),
    backward through mea_backward."""

    @staticmethod
    def forward(ctx, q, k, v, cu_q, cu_k, max_q, max_k, causal, slopes, scale):
        out, lse = attention_packed(q, k, v, cu_q, cu_k, max_q, causal=causal,
                                    alibi_slopes=slopes, scale=scale)
        ctx.save_for_backward(q, k, v, out, lse, cu_q, cu_k)
        ctx.args = (max_q, max_k, causal, slopes, scale)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse, cu_q, cu_k = ctx.saved_tensors
        max_q, max_k, causal, slopes, scale = ctx.args
        dq, dk, dv = attention_packed_backward(q, k, v, out, lse, dout.contiguous(), cu_q, cu_k,
                                               max_q, max_k, causal=causal, alibi_slopes=slopes,
                                               scale=scale)
        return dq, dk, dv, None, None, None, None, None, None, None


def device_error(clear: bool = True) -> int:
    """The device-side error word (non-zero if a kernel gave up on a bounded wait)."""
    import ctypes
    code = ctypes.c_int(0)
    _lib.check(_lib.load().mea_device_error(ctypes.byref(code), 1 if clear else 0),
               "mea_device_error")
    return code.value


def set_wait_timeout_ns(ns: int) -> None:
    _lib.load().mea_set_wait_timeout_ns(int(ns))


def wait_selftest(timeout_ns: int, arrive: bool, device=None) -> None:
    """Runs the library's bounded wait on a barrier that is (arrive=True) or is never
    (arrive=False) completed; in the second case the device error word afterwards holds
    MEA_SELFTEST_WAIT_CODE. Asynchronous on the device's current stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _lib.check(_lib.load().mea_wait_selftest(int(timeout_ns), 1 if arrive else 0, _stream(dev)),
               "mea_wait_selftest")
