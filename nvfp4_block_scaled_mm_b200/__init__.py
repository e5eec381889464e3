"""NVFP4 block-scaled GEMM with a fused BF16 LoRA correction on B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/nvfp4lora.h`` (``libnvfp4lora.so``, built
in-tree by :mod:`nvfp4_block_scaled_mm_b200.build`).  It only marshals arguments: every
step of the operation runs in the library's CUDA kernels.  PyTorch supplies device
memory, the current stream and the tensors' version counters (used for the stale-adapter
check).  There is no CPU fallback: the library is loaded on first use, and a missing
library raises ``RuntimeError`` there.

Two layers:

* ``nvfp4lora_mm``, ``nvfp4lora_prepare``, ``nvfp4lora_refold``,
  ``nvfp4lora_mm_prepared`` -- one-to-one with the C entry points (torch tensors in, the
  status mapped to exceptions);
* ``mm_nvfp4_lora``, ``prepare_nvfp4_lora_adapter``, ``PreparedNvFp4LoraAdapter``,
  ``StaleAdapterError`` -- the API of flashinfer.gemm.mm_nvfp4_lora and
  flashinfer.gemm.prepare_nvfp4_lora_adapter (signatures, Parameters, Returns, Notes);
  ``grouped_mm_nvfp4_lora`` (grouped_mm_bf16's grouped form), ``fp4_quantize``, and
  ``bgmv_moe_gemm2_lora_delta`` / ``fill_w_ptr`` (flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4lora.so")

__all__ = [
    "StaleAdapterError", "PreparedNvFp4LoraAdapter", "mm_nvfp4_lora", "prepare_nvfp4_lora_adapter",
    "nvfp4lora_mm", "nvfp4lora_prepare", "nvfp4lora_refold", "nvfp4lora_mm_prepared",
    "nvfp4lora_device_status", "nvfp4lora_quantize", "fp4_quantize", "library_path", "version",
    "nvfp4lora_grouped_mm", "grouped_mm_nvfp4_lora", "nvfp4lora_bgmv_moe_gemm2_lora_delta",
    "bgmv_moe_gemm2_lora_delta", "fill_w_ptr",
]

OK, INVALID_ARG, STALE, ALPHA_ZERO, UNSUPPORTED_ARCH, DEVICE_TIMEOUT, CUDA_ERR = range(7)


class StaleAdapterError(RuntimeError):
    """A prepared adapter's alpha, lora_b or lora_scale changed since its last (re)fold."""


class DeviceTimeoutError(RuntimeError):
    """A kernel's bounded wait ran out (reported by :func:`nvfp4lora_device_status`)."""


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m nvfp4_block_scaled_mm_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, U64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int32
    lib.nvfp4lora_mm.argtypes = [P, P, P, I64, P, I64, P, P, P, P, I64, P, P, I64, I64, I64, P]
    lib.nvfp4lora_mm.restype = ctypes.c_int
    lib.nvfp4lora_prepare.argtypes = [P, P, P, I64, I64, P, P, U64, P, P]
    lib.nvfp4lora_prepare.restype = ctypes.c_int
    lib.nvfp4lora_refold.argtypes = [P, P, P, P, I64, I64, U64, P]
    lib.nvfp4lora_refold.restype = ctypes.c_int
    lib.nvfp4lora_mm_prepared.argtypes = [P, P, P, I64, P, I64, P, P, P, P, P, U64, P, P, I64, I64, I64, P]
    lib.nvfp4lora_mm_prepared.restype = ctypes.c_int
    lib.nvfp4lora_device_status.argtypes = [P]
    lib.nvfp4lora_device_status.restype = ctypes.c_int
    lib.nvfp4lora_selftest_wait_timeout.argtypes = [I64, P]
    lib.nvfp4lora_selftest_wait_timeout.restype = ctypes.c_int
    lib.nvfp4lora_quantize.argtypes = [P, I64, I64, P, P, P, I64, P]
    lib.nvfp4lora_quantize.restype = ctypes.c_int
    lib.nvfp4lora_grouped_mm.argtypes = [P, P, P, I64, P, I64, P, I64, P, P, P, P, I64, P, P, I64, I64, I64, P]
    lib.nvfp4lora_grouped_mm.restype = ctypes.c_int
    lib.nvfp4lora_bgmv_moe_gemm2_lora_delta.argtypes = [P, I64, I64, P, P, I64, P, I64, P, P, P, I64, I64, I64, I64,
                                                        I64, ctypes.c_int32, ctypes.c_float, ctypes.c_int32, P, P]
    lib.nvfp4lora_bgmv_moe_gemm2_lora_delta.restype = ctypes.c_int
    lib.nvfp4lora_last_error.argtypes = []
    lib.nvfp4lora_last_error.restype = ctypes.c_char_p
    lib.nvfp4lora_version.argtypes = []
    lib.nvfp4lora_version.restype = ctypes.c_char_p
    del I32
    return lib


class _LazyLib:
    """Loads libnvfp4lora.so on first attribute access (raises if it was never built)."""

    _handle = None

    def __getattr__(self, name):
        if _LazyLib._handle is None:
            _LazyLib._handle = _load()
        return getattr(_LazyLib._handle, name)


_lib = _LazyLib()


def library_path() -> str:
    return LIB_PATH


def load_library():
    """Load the CUDA library now (it is otherwise loaded on first use)."""
    _lib.nvfp4lora_version  # noqa: B018
    return LIB_PATH


def version() -> str:
    return _lib.nvfp4lora_version().decode()


class _Adapter(ctypes.Structure):
    _fields_ = [("b_folded", ctypes.c_void_p), ("ratio", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("lora_b", ctypes.c_void_p), ("lora_scale", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("r", ctypes.c_int64), ("src_version", ctypes.c_uint64), ("device", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


def _check(status: int) -> None:
    if status == OK:
        return
    msg = _lib.nvfp4lora_last_error().decode()
    if status in (INVALID_ARG, ALPHA_ZERO):
        raise ValueError(msg)
    if status == STALE:
        raise StaleAdapterError(msg)
    if status == DEVICE_TIMEOUT:
        raise DeviceTimeoutError(msg)
    raise RuntimeError(msg)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _version_token(lora_b: torch.Tensor, lora_scale: torch.Tensor) -> int:
    return ((lora_b._version & 0xFFFFFFFF) << 32) | (lora_scale._version & 0xFFFFFFFF)


# --------------------------------------------------------------------------------------
# one-to-one C ABI wrappers
# --------------------------------------------------------------------------------------

def nvfp4lora_mm(a, b, a_sf, b_sf, alpha, d, lora_b, lora_scale, r, bias, out, M, N, K, stream=None):
    _check(_lib.nvfp4lora_mm(_ptr(a), _ptr(b), _ptr(a_sf), a_sf.numel(), _ptr(b_sf), b_sf.numel(),
                             _ptr(alpha), _ptr(d), _ptr(lora_b), _ptr(lora_scale), int(r), _ptr(bias),
                             _ptr(out), int(M), int(N), int(K), _stream(stream)))
    return out


def nvfp4lora_prepare(lora_b, lora_scale, alpha, N, r, b_folded, ratio, src_version, stream=None):
    adp = _Adapter()
    _check(_lib.nvfp4lora_prepare(_ptr(lora_b), _ptr(lora_scale), _ptr(alpha), int(N), int(r),
                                  _ptr(b_folded), _ptr(ratio), int(src_version), ctypes.byref(adp),
                                  _stream(stream)))
    return adp


def nvfp4lora_refold(adp, lora_b, lora_scale, alpha, N, r, src_version, stream=None):
    _check(_lib.nvfp4lora_refold(ctypes.byref(adp), _ptr(lora_b), _ptr(lora_scale), _ptr(alpha),
                                 int(N), int(r), int(src_version), _stream(stream)))
    return adp


def nvfp4lora_mm_prepared(a, b, a_sf, b_sf, alpha, d, adp, cur_lora_b, cur_lora_scale, cur_version,
                          bias, out, M, N, K, stream=None):
    _check(_lib.nvfp4lora_mm_prepared(_ptr(a), _ptr(b), _ptr(a_sf), a_sf.numel(), _ptr(b_sf),
                                      b_sf.numel(), _ptr(alpha), _ptr(d), ctypes.byref(adp),
                                      _ptr(cur_lora_b), _ptr(cur_lora_scale), int(cur_version),
                                      _ptr(bias), _ptr(out), int(M), int(N), int(K), _stream(stream)))
    return out


def nvfp4lora_grouped_mm(a, b, a_sf, b_sf, m_indptr, num_experts, alpha, d, lora_b, lora_scale, r, bias, out,
                         rows, N, K, stream=None):
    _check(_lib.nvfp4lora_grouped_mm(_ptr(a), _ptr(b), _ptr(a_sf), a_sf.numel(), _ptr(b_sf), b_sf.numel(),
                                     _ptr(m_indptr), int(num_experts), _ptr(alpha), _ptr(d), _ptr(lora_b),
                                     _ptr(lora_scale), int(r), _ptr(bias), _ptr(out), int(rows), int(N), int(K),
                                     _stream(stream)))
    return out


def nvfp4lora_bgmv_moe_gemm2_lora_delta(act, padded_rows, I, perm, w_ptr_a, lora_stride_a, w_ptr_b, lora_stride_b,
                                        topk_ids, topk_weights, lora_ids, num_tokens, top_k, num_experts, rank,
                                        hidden_size, lora_dtype, scale, out_dtype, out, stream=None):
    _check(_lib.nvfp4lora_bgmv_moe_gemm2_lora_delta(
        _ptr(act), int(padded_rows), int(I), _ptr(perm), _ptr(w_ptr_a), int(lora_stride_a), _ptr(w_ptr_b),
        int(lora_stride_b), _ptr(topk_ids), _ptr(topk_weights), _ptr(lora_ids), int(num_tokens), int(top_k),
        int(num_experts), int(rank), int(hidden_size), int(lora_dtype), float(scale), int(out_dtype), _ptr(out),
        _stream(stream)))
    return out


def nvfp4lora_device_status(stream=None) -> None:
    """Synchronise the stream; raise DeviceTimeoutError if a kernel's wait ran out, ValueError if a
    table read on the device (a grouped call's m_indptr, a LoRA delta's routing) broke its rules."""
    _check(_lib.nvfp4lora_device_status(_stream(stream)))


def nvfp4lora_quantize(x, rows, K, global_scale, codes, scales, stream=None):
    _check(_lib.nvfp4lora_quantize(_ptr(x), int(rows), int(K), _ptr(global_scale), _ptr(codes), _ptr(scales),
                                   scales.numel(), _stream(stream)))
    return codes, scales


def nvfp4lora_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test: a wait that nothing completes runs out after
    limit_ns; the next nvfp4lora_device_status raises DeviceTimeoutError."""
    _check(_lib.nvfp4lora_selftest_wait_timeout(int(limit_ns), _stream(stream)))


# --------------------------------------------------------------------------------------
# the pages' API
# --------------------------------------------------------------------------------------

def _need(t, name, dtype, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")


def _same_device(anchor_name: str, anchor: torch.Tensor, **others) -> None:
    """Every tensor given must live on the anchor tensor's device: the kernels run on that device
    and read every operand by address there, so an operand on another GPU would be read through
    a foreign address.  ValueError names the first tensor that differs (None entries are
    skipped)."""
    for name, t in others.items():
        if t is not None and t.device != anchor.device:
            raise ValueError(f"{name} is on {t.device} but {anchor_name} is on {anchor.device}: "
                             "every tensor of a call must be on the same device")


class PreparedNvFp4LoraAdapter:
    """A folded adapter (prepare_nvfp4_lora_adapter, Returns): ``b_folded`` bf16 [N, r], the
    device ``ratio`` scalar, the alpha tensor it belongs to, and the pins of its sources."""

    def __init__(self, c_adapter: _Adapter, b_folded, ratio, alpha, lora_b, lora_scale):
        self._c = c_adapter
        self.b_folded = b_folded
        self.ratio = ratio
        self.alpha = alpha
        self.lora_b = lora_b
        self.lora_scale = lora_scale

    @property
    def N(self) -> int:
        return int(self._c.N)

    @property
    def r(self) -> int:
        return int(self._c.r)


def _check_fold_inputs(lora_b, lora_scale, alpha):
    _need(lora_b, "lora_b", torch.bfloat16, 2)
    _need(lora_scale, "lora_scale", torch.float32)
    _need(alpha, "alpha", torch.float32)
    if lora_scale.numel() != 1:
        raise ValueError("lora_scale must be a one-element fp32 tensor")
    if alpha.numel() < 1:
        raise ValueError("alpha must hold at least one element")


def prepare_nvfp4_lora_adapter(lora_b: torch.Tensor, lora_scale: torch.Tensor, alpha: torch.Tensor, *,
                               out: Optional[PreparedNvFp4LoraAdapter] = None) -> PreparedNvFp4LoraAdapter:
    """Fold ``b_folded = bf16(lora_b * (lora_scale / alpha[0]))``.

    ``out=None``: the eager form (one host read of (lora_scale, alpha); alpha == 0 or a
    non-finite ratio raises ValueError).  ``out=adapter``: in-place refold on the device,
    no host read, graph-capturable; alpha must be the adapter's own alpha tensor.
    """
    _check_fold_inputs(lora_b, lora_scale, alpha)
    _same_device("lora_b", lora_b, lora_scale=lora_scale, alpha=alpha,
                 b_folded=None if out is None else out.b_folded, ratio=None if out is None else out.ratio)
    N, r = lora_b.shape
    stream = torch.cuda.current_stream(lora_b.device)
    if out is None:
        with torch.cuda.device(lora_b.device):
            b_folded = torch.empty_like(lora_b)
            ratio = torch.empty(1, dtype=torch.float32, device=lora_b.device)
            c = nvfp4lora_prepare(lora_b, lora_scale, alpha, N, r, b_folded, ratio,
                                  _version_token(lora_b, lora_scale), stream)
        return PreparedNvFp4LoraAdapter(c, b_folded, ratio, alpha, lora_b, lora_scale)
    if not isinstance(out, PreparedNvFp4LoraAdapter):
        raise ValueError("out must be a PreparedNvFp4LoraAdapter")
    with torch.cuda.device(lora_b.device):
        nvfp4lora_refold(out._c, lora_b, lora_scale, alpha, N, r, _version_token(lora_b, lora_scale), stream)
    out.lora_b = lora_b
    out.lora_scale = lora_scale
    return out


def mm_nvfp4_lora(a: torch.Tensor, b: torch.Tensor, a_sf: torch.Tensor, b_sf: torch.Tensor,
                  alpha: torch.Tensor, d: Optional[torch.Tensor] = None,
                  lora_b: Optional[torch.Tensor] = None, lora_scale: Optional[torch.Tensor] = None, *,
                  lora_adapter: Optional[PreparedNvFp4LoraAdapter] = None,
                  bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                  out_dtype: torch.dtype = torch.bfloat16, backend: str = "cake",
                  enable_pdl: Optional[bool] = None) -> torch.Tensor:
    """``out = alpha * (dequant(a) @ dequant(b)^T) + lora_scale * (d @ lora_b^T) [+ bias]``.

    Raw path: ``d``, ``lora_b``, ``lora_scale``; ``lora_scale=None`` is the adapter-off
    call even if d / lora_b are given.  Prepared path: ``lora_adapter=`` plus ``d``.

    The call returns once the kernel is enqueued.  A kernel whose bounded wait gives up (a
    stalled pipeline) returns early and leaves ``out`` partly unwritten, so ``out`` is defined
    only once a later :func:`nvfp4lora_device_status` on the stream has returned without
    raising ``DeviceTimeoutError``.
    """
    if out_dtype != torch.bfloat16:
        raise ValueError("out_dtype: only torch.bfloat16 is supported")
    if backend not in ("cake", "auto"):
        raise ValueError("backend must be 'cake' or 'auto'")
    if enable_pdl not in (None, True):
        raise ValueError("enable_pdl must be None or True")
    if lora_adapter is not None and (lora_b is not None or lora_scale is not None):
        raise ValueError("pass either the raw adapter (lora_b, lora_scale) or lora_adapter, not both")
    _need(a, "a", torch.uint8, 2)
    _need(b, "b", torch.uint8, 2)
    _need(a_sf, "a_sf", torch.uint8)
    _need(b_sf, "b_sf", torch.uint8)
    _need(alpha, "alpha", torch.float32)
    M, K = a.shape[0], a.shape[1] * 2
    N = b.shape[0]
    if b.shape[1] * 2 != K:
        raise ValueError(f"a is [M, K/2] = {tuple(a.shape)} but b is {tuple(b.shape)}: K differs")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
        if bias.shape[0] != N:
            raise ValueError(f"bias must be [N] = [{N}]")
    _same_device("a", a, b=b, a_sf=a_sf, b_sf=b_sf, alpha=alpha, d=d, lora_b=lora_b, lora_scale=lora_scale,
                 bias=bias, out=out,
                 b_folded=None if lora_adapter is None else lora_adapter.b_folded,
                 ratio=None if lora_adapter is None else lora_adapter.ratio)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    else:
        _need(out, "out", torch.bfloat16, 2)
        if tuple(out.shape) != (M, N):
            raise ValueError(f"out must be [M, N] = [{M}, {N}]")
    stream = torch.cuda.current_stream(a.device)
    with torch.cuda.device(a.device):
        if lora_adapter is not None:
            if d is None:
                raise ValueError("the prepared path still requires d")
            _need(d, "d", torch.bfloat16, 2)
            if tuple(d.shape) != (M, lora_adapter.r):
                raise ValueError(f"d must be [M, r] = [{M}, {lora_adapter.r}]")
            src = lora_adapter
            nvfp4lora_mm_prepared(a, b, a_sf, b_sf, alpha, d, src._c, src.lora_b, src.lora_scale,
                                  _version_token(src.lora_b, src.lora_scale), bias, out, M, N, K, stream)
            return out
        if lora_scale is None:
            nvfp4lora_mm(a, b, a_sf, b_sf, alpha, None, None, None, 0, bias, out, M, N, K, stream)
            return out
        _need(lora_scale, "lora_scale", torch.float32)
        if lora_scale.numel() != 1:
            raise ValueError("lora_scale must be a one-element fp32 tensor")
        if d is None or lora_b is None:
            raise ValueError("the raw path needs d and lora_b with lora_scale")
        _need(d, "d", torch.bfloat16, 2)
        _need(lora_b, "lora_b", torch.bfloat16, 2)
        r = d.shape[1]
        if d.shape[0] != M or tuple(lora_b.shape) != (N, r):
            raise ValueError(f"d must be [M, r] and lora_b [N, r]; got {tuple(d.shape)}, {tuple(lora_b.shape)}")
        nvfp4lora_mm(a, b, a_sf, b_sf, alpha, d, lora_b, lora_scale, r, bias, out, M, N, K, stream)
        return out


def grouped_mm_nvfp4_lora(a: torch.Tensor, b: torch.Tensor, a_sf: torch.Tensor, b_sf: torch.Tensor,
                          m_indptr: torch.Tensor, alpha: torch.Tensor, d: Optional[torch.Tensor] = None,
                          lora_b: Optional[torch.Tensor] = None, lora_scale: Optional[torch.Tensor] = None, *,
                          bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Grouped (expert-partitioned) form, flashinfer.grouped_mm.grouped_mm_bf16's formula applied to
    :func:`mm_nvfp4_lora`: for each expert e with rows ``s, t = m_indptr[e], m_indptr[e+1]``,
    ``out[s:t] = alpha[e] * (dequant(a[s:t]) @ dequant(b[e])^T) + lora_scale * (d[s:t] @ lora_b[e]^T)
    [+ bias[e]]``.

    a: uint8 [rows, K/2] with a_sf over all rows; b: uint8 [E, N, K/2] with b_sf holding E
    consecutive 128x4 buffers; m_indptr: int32 [E + 1] on the device, 0, non-decreasing multiples
    of 128, at most rows (each expert's rows fill whole 128-row scale blocks); alpha: fp32 [E];
    d: bf16 [rows, r]; lora_b: bf16 [E, N, r]; lora_scale: fp32 [1] or None; bias: bf16 [E, N].
    Rows from m_indptr[E] on are left untouched.  m_indptr is checked on the device: a table that
    breaks its rules computes nothing, and :func:`nvfp4lora_device_status` raises ValueError.
    """
    _need(a, "a", torch.uint8, 2)
    _need(b, "b", torch.uint8, 3)
    _need(a_sf, "a_sf", torch.uint8)
    _need(b_sf, "b_sf", torch.uint8)
    _need(m_indptr, "m_indptr", torch.int32, 1)
    _need(alpha, "alpha", torch.float32, 1)
    rows, K = a.shape[0], a.shape[1] * 2
    E, N = b.shape[0], b.shape[1]
    if b.shape[2] * 2 != K:
        raise ValueError(f"a is [rows, K/2] = {tuple(a.shape)} but b is {tuple(b.shape)}: K differs")
    if m_indptr.shape[0] != E + 1 or alpha.shape[0] != E:
        raise ValueError(f"m_indptr must be [E + 1] = [{E + 1}] and alpha [E] = [{E}]")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 2)
        if tuple(bias.shape) != (E, N):
            raise ValueError(f"bias must be [E, N] = [{E}, {N}]")
    r = 0
    if lora_scale is not None:
        _need(lora_scale, "lora_scale", torch.float32)
        if lora_scale.numel() != 1:
            raise ValueError("lora_scale must be a one-element fp32 tensor")
        if d is None or lora_b is None:
            raise ValueError("the LoRA term needs d and lora_b with lora_scale")
        _need(d, "d", torch.bfloat16, 2)
        _need(lora_b, "lora_b", torch.bfloat16, 3)
        r = d.shape[1]
        if d.shape[0] != rows or tuple(lora_b.shape) != (E, N, r):
            raise ValueError(f"d must be [rows, r] and lora_b [E, N, r]; got {tuple(d.shape)}, {tuple(lora_b.shape)}")
    if out is None:
        out = torch.empty((rows, N), dtype=torch.bfloat16, device=a.device)
    else:
        _need(out, "out", torch.bfloat16, 2)
        if tuple(out.shape) != (rows, N):
            raise ValueError(f"out must be [rows, N] = [{rows}, {N}]")
    _same_device("a", a, b=b, a_sf=a_sf, b_sf=b_sf, m_indptr=m_indptr, alpha=alpha, d=d, lora_b=lora_b,
                 lora_scale=lora_scale, bias=bias, out=out)
    with torch.cuda.device(a.device):
        nvfp4lora_grouped_mm(a, b, a_sf, b_sf, m_indptr, E, alpha, d if lora_scale is not None else None,
                             lora_b if lora_scale is not None else None, lora_scale, r, bias, out, rows, N, K,
                             torch.cuda.current_stream(a.device))
    return out


_DTYPE_CODES = {torch.bfloat16: 0, torch.float16: 1}


def fill_w_ptr(banks) -> torch.Tensor:
    """The int64 ``[1, num_experts]`` table of bank addresses that
    :func:`bgmv_moe_gemm2_lora_delta` takes as ``w_ptr_a`` / ``w_ptr_b``: entry e is the device
    address of ``banks[e]`` (one contiguous bf16 or fp16 CUDA tensor per expert, holding that
    expert's adapters ``lora_stride`` elements apart).  The table does not keep the banks alive."""
    banks = list(banks)
    if not banks:
        raise ValueError("fill_w_ptr needs at least one bank")
    dev = banks[0].device
    for i, t in enumerate(banks):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"bank {i} must be a contiguous CUDA tensor")
        if t.dtype not in _DTYPE_CODES:
            raise ValueError(f"bank {i} must be bf16 or fp16, got {t.dtype}")
        if t.device != dev:
            raise ValueError(f"bank {i} is on {t.device} but bank 0 is on {dev}")
    return torch.tensor([[t.data_ptr() for t in banks]], dtype=torch.int64, device=dev)


def bgmv_moe_gemm2_lora_delta(gemm1_activation_output: torch.Tensor, expanded_idx_to_permuted_idx: torch.Tensor,
                              w_ptr_a: torch.Tensor, lora_stride_a: int, w_ptr_b: torch.Tensor,
                              lora_stride_b: int, topk_ids: torch.Tensor, topk_weights: torch.Tensor,
                              lora_ids: torch.Tensor, rank: int, hidden_size: int, *,
                              lora_dtype: torch.dtype = torch.bfloat16, scale: float = 1.0,
                              out_dtype: torch.dtype = torch.bfloat16,
                              out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """FC2 (down projection) LoRA delta of a routed MoE, flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta:
    ``delta[t] = scale * sum_j topk_weights[t, j] * (B_down[l, e] @ (A_down[l, e] @ act[p]))`` with
    ``l = lora_ids[t]`` (negative: a zero row), ``e = topk_ids[t, j]`` and
    ``p = expanded_idx_to_permuted_idx[t * top_k + j]`` (negative: inactive slot).  Returns
    ``[T, hidden_size]`` in out_dtype, to be added to the MoE output.

    gemm1_activation_output: lora_dtype ``[padded_rows, I]`` (I % 8 == 0); the index, id and weight
    tensors are int32 / int32 / fp32 as shaped on the page; ``w_ptr_a`` / ``w_ptr_b``: int64
    ``[1, num_experts]`` bank-address tables (:func:`fill_w_ptr`), A_down[l, e] being the
    ``[rank, I]`` row-major block ``l * lora_stride_a`` elements into expert e's A bank and
    B_down[l, e] the ``[H, rank]`` block ``l * lora_stride_b`` elements into its B bank.  The banks
    must live on the activation's device; adapter ids must exist in them.  Routing entries are
    read on the device: one out of range is skipped and :func:`nvfp4lora_device_status` raises
    ValueError."""
    act = gemm1_activation_output
    if lora_dtype not in _DTYPE_CODES or out_dtype not in _DTYPE_CODES:
        raise ValueError("lora_dtype and out_dtype must be torch.bfloat16 or torch.float16")
    _need(act, "gemm1_activation_output", lora_dtype, 2)
    _need(expanded_idx_to_permuted_idx, "expanded_idx_to_permuted_idx", torch.int32)
    _need(w_ptr_a, "w_ptr_a", torch.int64)
    _need(w_ptr_b, "w_ptr_b", torch.int64)
    _need(topk_ids, "topk_ids", torch.int32, 2)
    _need(topk_weights, "topk_weights", torch.float32, 2)
    _need(lora_ids, "lora_ids", torch.int32, 1)
    T, top_k = topk_ids.shape
    E = w_ptr_a.numel()
    if w_ptr_b.numel() != E:
        raise ValueError(f"w_ptr_a has {E} entries but w_ptr_b has {w_ptr_b.numel()}")
    if tuple(topk_weights.shape) != (T, top_k) or lora_ids.shape[0] != T:
        raise ValueError(f"topk_weights must be [T, top_k] = [{T}, {top_k}] and lora_ids [T]")
    if expanded_idx_to_permuted_idx.numel() != T * top_k:
        raise ValueError(f"expanded_idx_to_permuted_idx must hold T * top_k = {T * top_k} entries")
    H = int(hidden_size)
    if out is None:
        out = torch.empty((T, H), dtype=out_dtype, device=act.device)
    else:
        _need(out, "out", out_dtype, 2)
        if tuple(out.shape) != (T, H):
            raise ValueError(f"out must be [T, hidden_size] = [{T}, {H}]")
    _same_device("gemm1_activation_output", act, expanded_idx_to_permuted_idx=expanded_idx_to_permuted_idx,
                 w_ptr_a=w_ptr_a, w_ptr_b=w_ptr_b, topk_ids=topk_ids, topk_weights=topk_weights, lora_ids=lora_ids,
                 out=out)
    with torch.cuda.device(act.device):
        nvfp4lora_bgmv_moe_gemm2_lora_delta(act, act.shape[0], act.shape[1], expanded_idx_to_permuted_idx, w_ptr_a,
                                            lora_stride_a, w_ptr_b, lora_stride_b, topk_ids, topk_weights, lora_ids,
                                            T, top_k, E, rank, H, _DTYPE_CODES[lora_dtype], scale,
                                            _DTYPE_CODES[out_dtype], out, torch.cuda.current_stream(act.device))
    return out


def fp4_quantize(x: torch.Tensor, global_scale: torch.Tensor, *, codes: Optional[torch.Tensor] = None,
                 scales: Optional[torch.Tensor] = None):
    """Quantize bf16 ``x [rows, K]`` into the operand format of :func:`mm_nvfp4_lora`: E2M1
    ``codes uint8 [rows, K/2]`` and UE4M3 ``scales`` (16 K-elements each, 128x4 swizzled, rows
    padded to 128), with the per-tensor ``global_scale`` (fp32, one element, on the device) folded
    in: ``value(code) * value(scale) / global_scale`` approximates x.  Rule (per 16-block, fp32):
    ``scale = e4m3(amax * gs / 6)``, ``code = e2m1(x * gs / value(scale))``, round to nearest
    even, saturating."""
    _need(x, "x", torch.bfloat16, 2)
    _need(global_scale, "global_scale", torch.float32)
    if global_scale.numel() != 1:
        raise ValueError("global_scale must be a one-element fp32 tensor")
    _same_device("x", x, global_scale=global_scale, codes=codes, scales=scales)
    rows, K = x.shape
    if K % 64 != 0:
        raise ValueError(f"K = {K}: a multiple of 64 is required")
    nbytes = (rows + 127) // 128 * 128 * (K // 16)
    if codes is None:
        codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    else:
        _need(codes, "codes", torch.uint8, 2)
        if tuple(codes.shape) != (rows, K // 2):
            raise ValueError(f"codes must be [rows, K/2] = [{rows}, {K // 2}]")
    if scales is None:
        scales = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    else:
        _need(scales, "scales", torch.uint8)
    with torch.cuda.device(x.device):
        nvfp4lora_quantize(x, rows, K, global_scale, codes, scales, torch.cuda.current_stream(x.device))
    return codes, scales
