"""CPU oracle for the NVFP4 block-scaled GEMM with a fused BF16 LoRA correction.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The product path (the CUDA library and its Python binding) never imports, links or
calls anything here, and this module imports nothing from the product.

It restates, slowly and in float64, what the pages define:

* ``flashinfer.gemm.mm_nvfp4_lora`` -- opening formula
  ``out = alpha * (dequant(a) @ dequant(b)^T) + lora_scale * (d @ lora_b^T) [+ bias]``,
  the paragraph after it (operands consumed as ``mm_fp4`` does: E2M1 codes packed two
  per byte, UE4M3 scales over 16 K-elements in the 128x4 swizzled layout; correction
  in fp32 in the same kernel; one rounding to bf16), the "Raw path" and "Prepared path"
  bullets, and the Parameters entries for a, b, a_sf, b_sf, alpha, d, lora_b,
  lora_scale and bias.
* ``flashinfer.gemm.prepare_nvfp4_lora_adapter`` -- summary paragraph (the fold:
  ``ratio = div.rn.f32(lora_scale, alpha[0])``,
  ``b_folded[i] = bf16_rne(fp32(lora_b[i]) * ratio)``).
* the quantizer the mm_nvfp4_lora page names as the producer of a / a_sf (``fp4_quantize``),
  by the reading given at :func:`quantize_nvfp4`.
* ``flashinfer.grouped_mm.grouped_mm_bf16`` -- the grouped (expert-partitioned) form, by the
  reading given at :func:`grouped_mm`.
* ``flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta`` -- opening formula and Parameters: the
  routed-MoE FC2 LoRA delta, by the readings given at :func:`bgmv_moe_lora_delta`.

Readings taken where the pages are silent:

* nibble order: element ``2j`` of a row is the LOW nibble of byte ``j``.  The GEMM
  result does not depend on it (both nibbles of a byte sit in the same 16-block and
  A and B use the same convention), only generators do;
* the 128x4 swizzle is the block-scale layout of the tensor-core scale copy:
  ``offset(r, c) = ((r // 128) * (C // 4) + c // 4) * 512 + (r % 32) * 16
  + ((r % 128) // 32) * 4 + (c % 4)`` with ``C = K // 16`` scale columns;
* UE4M3 byte ``0x7F`` is NaN; a byte with bit 7 set is not a UE4M3 value and is
  rejected;
* the output rounding goes from the float64 value straight to bf16 (round to nearest,
  ties to even, subnormals kept, overflow to infinity) -- one rounding, no float32 step;
* raw epilogue ``alpha*base + s*L (+ bias)``; prepared ``alpha*(base + L_folded)
  (+ bias)`` (bias is not multiplied by alpha); adapter-off ``alpha*base (+ bias)``;
* NaN produced by the fold is stored as 0x7FC0, PyTorch's bf16 NaN.

Parity of the base product: with the configs' scale range every product
``e2m1 * e2m1 * ue4m3 * ue4m3`` is a multiple of 2**-12 below 576 in magnitude, so
partial sums over K <= 8192 need at most 35 significant bits and the float64 matmul
below is exact whatever order the library sums in.
"""

from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------------------
# Element formats (mm_nvfp4_lora page, paragraph after the formula and Parameters: a, b,
# a_sf, b_sf).  The pages name the formats; their value sets are fixed by the formats.
# --------------------------------------------------------------------------------------

#: E2M1 value of each 4-bit code (bit 3 sign, bits 2..1 exponent with bias 1, bit 0
#: mantissa).  Written out as the 16-entry table.
E2M1_TABLE = np.array(
    [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
     -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0],
    dtype=np.float64,
)

SF_VEC = 16          # K-elements covered by one UE4M3 scale
SF_ATOM_ROWS = 128   # rows of one swizzle atom
SF_ATOM_COLS = 4     # scale columns of one swizzle atom
SF_ATOM_BYTES = SF_ATOM_ROWS * SF_ATOM_COLS


def decode_e2m1(packed: np.ndarray) -> np.ndarray:
    """Unpack ``uint8 [R, K/2]`` into float64 ``[R, K]``; element 2j = low nibble of byte j."""
    packed = np.asarray(packed, dtype=np.uint8)
    lo = E2M1_TABLE[packed & 0x0F]
    hi = E2M1_TABLE[packed >> 4]
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.float64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def decode_ue4m3(x: np.ndarray) -> np.ndarray:
    """UE4M3 bytes -> float64: 4 exponent bits (bias 7), 3 mantissa bits, no sign.

    ``e == 0`` is subnormal (``m * 2**-9``); ``0x7F`` is NaN; max finite ``0x7E`` = 448.
    """
    x = np.asarray(x, dtype=np.uint8)
    if np.any(x & 0x80):
        raise ValueError("UE4M3 byte with bit 7 set: not an unsigned E4M3 value")
    e = (x >> 3).astype(np.int64) & 0xF
    m = (x & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64))
    sub = m * 2.0 ** -9
    val = np.where(e == 0, sub, normal)
    return np.where(x == 0x7F, np.nan, val)


# --------------------------------------------------------------------------------------
# 128x4 swizzled scale layout (mm_nvfp4_lora page, Parameters: a_sf / b_sf: "128x4
# swizzled layout (rows padded to 128); larger contiguous backing buffers are accepted")
# --------------------------------------------------------------------------------------

def padded_rows(rows: int) -> int:
    return -(-rows // SF_ATOM_ROWS) * SF_ATOM_ROWS


def sf_buffer_bytes(rows: int, k: int) -> int:
    """Minimum byte size of a swizzled scale buffer for ``rows`` rows and K = ``k``."""
    return padded_rows(rows) * (k // SF_VEC)


def sf_offset(r, c, k: int):
    """Byte offset of logical scale ``(row r, scale column c)`` for K = ``k``."""
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    col_atoms = (k // SF_VEC) // SF_ATOM_COLS
    return (((r // 128) * col_atoms + c // 4) * SF_ATOM_BYTES
            + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4))


def unswizzle_scales(buf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Logical ``uint8 [rows, k/16]`` scale matrix read out of a swizzled buffer."""
    buf = np.asarray(buf, dtype=np.uint8).reshape(-1)
    need = sf_buffer_bytes(rows, k)
    if buf.size < need:
        raise ValueError(f"scale buffer has {buf.size} bytes, needs {need}")
    rr, cc = np.meshgrid(np.arange(rows), np.arange(k // SF_VEC), indexing="ij")
    return buf[sf_offset(rr, cc, k)]


def swizzle_scales(logical: np.ndarray, k: int, pad_value: int = 0) -> np.ndarray:
    """Inverse of :func:`unswizzle_scales`: place ``[rows, k/16]`` into a padded buffer."""
    logical = np.asarray(logical, dtype=np.uint8)
    rows = logical.shape[0]
    buf = np.full(sf_buffer_bytes(rows, k), pad_value, dtype=np.uint8)
    rr, cc = np.meshgrid(np.arange(rows), np.arange(k // SF_VEC), indexing="ij")
    buf[sf_offset(rr, cc, k)] = logical
    return buf


def dequant(codes: np.ndarray, sf_buf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """``dequant(x)`` of the opening formula: E2M1 value times its block's UE4M3 scale."""
    vals = decode_e2m1(np.asarray(codes, dtype=np.uint8).reshape(rows, k // 2))
    scales = decode_ue4m3(unswizzle_scales(sf_buf, rows, k))
    return vals * np.repeat(scales, SF_VEC, axis=1)


# --------------------------------------------------------------------------------------
# bf16 helpers (the output dtype; d, lora_b, bias, b_folded are bf16 bit patterns)
# --------------------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_rne(y: np.ndarray) -> np.ndarray:
    """Round float64 straight to bf16 bits: nearest, ties to even, one rounding.

    bf16 keeps 8 significant bits and float32's exponent range (normal down to 2**-126,
    subnormal quantum 2**-133).  The quantum of |y| in [2**(E-1), 2**E) is
    ``2**(max(E, -125) - 8)``; dividing by a power of two is exact, ``rint`` rounds
    half to even, and a result of 2**128 or more is infinity.
    """
    y = np.asarray(y, dtype=np.float64)
    out = np.zeros(y.shape, dtype=np.uint16)
    sign = np.signbit(y)
    mag = np.abs(y)
    finite = np.isfinite(y)
    nz = finite & (mag > 0)
    _, exp = np.frexp(np.where(nz, mag, 1.0))          # mag = f * 2**exp, f in [0.5, 1)
    q_exp = np.maximum(exp, -125) - 8
    q = np.exp2(q_exp.astype(np.float64))
    rounded = np.rint(np.where(nz, mag, 0.0) / q) * q
    overflow = nz & (rounded >= 2.0 ** 128)
    fin_bits = (np.where(overflow, 0.0, rounded).astype(np.float32).view(np.uint32) >> 16)
    out[:] = fin_bits.astype(np.uint16)
    out[overflow] = 0x7F80
    out[np.isinf(y)] = 0x7F80
    out = np.where(sign, out | 0x8000, out).astype(np.uint16)
    out[np.isnan(y)] = 0x7FC0
    return out


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, nearest-even, NaN -> 0x7FC0 (PyTorch's bf16 NaN)."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = (rounded & 0xFFFF).astype(np.uint16)
    out[np.isnan(x)] = 0x7FC0
    return out


# --------------------------------------------------------------------------------------
# The operation (mm_nvfp4_lora page)
# --------------------------------------------------------------------------------------

def base_product(a, b, a_sf, b_sf, M: int, N: int, K: int) -> np.ndarray:
    """``dequant(a) @ dequant(b)^T`` in float64 (opening formula); a library matmul."""
    return dequant(a, a_sf, M, K) @ dequant(b, b_sf, N, K).T


def base_element(a, b, a_sf, b_sf, M: int, N: int, K: int, m: int, n: int) -> float:
    """One element of the base product, summed block by block in float64."""
    a_row = decode_e2m1(np.asarray(a, dtype=np.uint8).reshape(M, K // 2)[m])
    b_row = decode_e2m1(np.asarray(b, dtype=np.uint8).reshape(N, K // 2)[n])
    cols = np.arange(K // SF_VEC)
    sa = decode_ue4m3(np.asarray(a_sf, dtype=np.uint8).reshape(-1)[sf_offset(m, cols, K)])
    sb = decode_ue4m3(np.asarray(b_sf, dtype=np.uint8).reshape(-1)[sf_offset(n, cols, K)])
    total = 0.0
    for blk in range(K // SF_VEC):
        sl = slice(blk * SF_VEC, (blk + 1) * SF_VEC)
        total += float(np.dot(a_row[sl], b_row[sl])) * float(sa[blk]) * float(sb[blk])
    return total


def dequant_rows(codes, sf_buf, K: int, rows) -> np.ndarray:
    """``dequant`` of selected rows only (for sampled checks at full sizes)."""
    rows = np.asarray(rows, dtype=np.int64)
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1, K // 2)
    vals = decode_e2m1(codes[rows])
    cols = np.arange(K // SF_VEC)
    offs = sf_offset(rows[:, None], cols[None, :], K)
    scales = decode_ue4m3(np.asarray(sf_buf, dtype=np.uint8).reshape(-1)[offs])
    return vals * np.repeat(scales, SF_VEC, axis=1)


def base_product_rows_cols(a, b, a_sf, b_sf, K: int, rows, cols) -> np.ndarray:
    """The base product restricted to ``rows`` x ``cols`` (same definition, fewer outputs)."""
    return dequant_rows(a, a_sf, K, rows) @ dequant_rows(b, b_sf, K, cols).T


def _pick(idx, count: int) -> np.ndarray:
    """The selected output rows (or columns): all of them when ``idx`` is None."""
    return np.arange(count) if idx is None else np.asarray(idx, dtype=np.int64)


def lora_term(d_bits, lb_bits, M: int, N: int, r: int, rows=None, cols=None) -> np.ndarray:
    """``d @ lora_b^T`` in float64 (bf16 x bf16 products are exact in float64), restricted to
    the output ``rows`` x ``cols`` when given."""
    d = bf16_bits_to_f64(np.asarray(d_bits).reshape(M, r))[_pick(rows, M)]
    lb = bf16_bits_to_f64(np.asarray(lb_bits).reshape(N, r))[_pick(cols, N)]
    return d @ lb.T


def _bias_row(bias_bits, N: int, cols=None):
    if bias_bits is None:
        return 0.0
    return bf16_bits_to_f64(np.asarray(bias_bits).reshape(N))[_pick(cols, N)][None, :]


def _base(a, b, a_sf, b_sf, M: int, N: int, K: int, rows, cols) -> np.ndarray:
    if rows is None and cols is None:
        return base_product(a, b, a_sf, b_sf, M, N, K)
    return base_product_rows_cols(a, b, a_sf, b_sf, K, _pick(rows, M), _pick(cols, N))


# The three call forms below take optional ``rows`` / ``cols`` (index arrays): the same
# definition evaluated on the selected outputs only, for sampled checks at full sizes.  A
# caller-supplied ``base`` must already cover exactly those outputs.

def mm_raw(a, b, a_sf, b_sf, alpha: float, d_bits, lb_bits, lora_scale, bias_bits,
           M: int, N: int, K: int, r: int, base: np.ndarray | None = None,
           rows=None, cols=None) -> np.ndarray:
    """Raw path ("Raw path" bullet): ``alpha*base + s*(d @ lora_b^T) [+ bias]``, float64.

    ``lora_scale`` None or equal to zero is the zero-adapter call (Parameters:
    lora_scale): the LoRA term is not evaluated at all.
    """
    if base is None:
        base = _base(a, b, a_sf, b_sf, M, N, K, rows, cols)
    y = np.float64(alpha) * base
    if lora_scale is not None and float(lora_scale) != 0.0:
        y = y + np.float64(lora_scale) * lora_term(d_bits, lb_bits, M, N, r, rows, cols)
    return y + _bias_row(bias_bits, N, cols)


def mm_prepared(a, b, a_sf, b_sf, alpha: float, d_bits, b_folded_bits, ratio, bias_bits,
                M: int, N: int, K: int, r: int, base: np.ndarray | None = None,
                rows=None, cols=None) -> np.ndarray:
    """Prepared path ("Prepared path" bullet): base first, LoRA with ``b_folded`` into the
    same accumulator, alpha applied once: ``alpha*(base + d @ b_folded^T) [+ bias]``.

    ``ratio`` is the fold's ``lora_scale / alpha``; a zero ratio is the zero adapter
    (Parameters: lora_adapter -- a zero lora_scale gives the adapter-off output).
    """
    if base is None:
        base = _base(a, b, a_sf, b_sf, M, N, K, rows, cols)
    acc = base
    if float(ratio) != 0.0:
        acc = acc + lora_term(d_bits, b_folded_bits, M, N, r, rows, cols)
    return np.float64(alpha) * acc + _bias_row(bias_bits, N, cols)


def mm_off(a, b, a_sf, b_sf, alpha: float, bias_bits, M: int, N: int, K: int,
           base: np.ndarray | None = None, rows=None, cols=None) -> np.ndarray:
    """Adapter-off call (neither form): ``alpha*base [+ bias]``."""
    if base is None:
        base = _base(a, b, a_sf, b_sf, M, N, K, rows, cols)
    return np.float64(alpha) * base + _bias_row(bias_bits, N, cols)


# --------------------------------------------------------------------------------------
# Grouped (expert-partitioned) form: flashinfer.grouped_mm.grouped_mm_bf16's formula
# (out[start:end] = a[start:end] x b[e]^T for each expert e, start, end = m_indptr[e],
# m_indptr[e+1]) applied to this operation.  Reading taken: every m_indptr[e] is a multiple of
# 128 (each expert's token rows fill whole 128-row blocks of the 128x4 scale layout, padding rows
# included), alpha is per expert ([E]), lora_b ([E, N, r]) and bias ([E, N]) are per expert, d
# and lora_scale are shared.
# --------------------------------------------------------------------------------------

def check_grouped_indptr(m_indptr, rows: int) -> np.ndarray:
    """The reading's rules: int, starts at 0, non-decreasing, multiples of 128, ends <= rows."""
    ind = np.asarray(m_indptr, dtype=np.int64).reshape(-1)
    if ind.size < 2 or ind[0] != 0 or np.any(np.diff(ind) < 0) or np.any(ind % 128 != 0) or ind[-1] > rows:
        raise ValueError("m_indptr must start at 0, be non-decreasing, hold multiples of 128 and end <= rows")
    return ind


def grouped_mm(a, b, a_sf, b_sf, m_indptr, alpha, d_bits, lb_bits, lora_scale, bias_bits,
               rows: int, N: int, K: int, r: int) -> np.ndarray:
    """float64 values of the rows [0, m_indptr[E]) of the grouped call; expert e's segment is the
    raw-path call form (``mm_raw``; lora_scale None or 0 is adapter-off) on a[s:t] and b[e].

    a: [rows, K/2]; a_sf: the 128x4 layout of all rows (so a segment's scales are its 128-row
    blocks); b: [E, N, K/2]; b_sf: [E] consecutive scale buffers of ceil(N/128)*128*K/16 bytes;
    alpha: [E]; d: [rows, r]; lora_b: [E, N, r]; bias: [E, N] or None."""
    ind = check_grouped_indptr(m_indptr, rows)
    E = ind.size - 1
    a = np.asarray(a, dtype=np.uint8).reshape(rows, K // 2)
    a_sf = np.asarray(a_sf, dtype=np.uint8).reshape(-1)
    b = np.asarray(b, dtype=np.uint8).reshape(E, N, K // 2)
    sfb_bytes = sf_buffer_bytes(N, K)
    b_sf = np.asarray(b_sf, dtype=np.uint8).reshape(-1)
    alpha = np.asarray(alpha, dtype=np.float64).reshape(E)
    lb = None if lb_bits is None else np.asarray(lb_bits).reshape(E, N, r)
    d = None if d_bits is None else np.asarray(d_bits).reshape(rows, r)
    bias = None if bias_bits is None else np.asarray(bias_bits).reshape(E, N)
    out = np.zeros((int(ind[-1]), N), dtype=np.float64)
    row_sf = K // SF_VEC                        # scale bytes per row (whole 128-row blocks)
    for e in range(E):
        s, t = int(ind[e]), int(ind[e + 1])
        if t == s:
            continue
        out[s:t] = mm_raw(a[s:t], b[e], a_sf[s * row_sf:t * row_sf], b_sf[e * sfb_bytes:(e + 1) * sfb_bytes],
                          float(alpha[e]), None if d is None else d[s:t], None if lb is None else lb[e],
                          lora_scale, None if bias is None else bias[e], t - s, N, K, r)
    return out


def round_output(y: np.ndarray) -> np.ndarray:
    """The single rounding of the fp32 result to bf16, taken here from float64."""
    return f64_to_bf16_rne(y)


# --------------------------------------------------------------------------------------
# The fold (prepare_nvfp4_lora_adapter page, summary paragraph)
# --------------------------------------------------------------------------------------

def fold_ratio(lora_scale: float, alpha: float) -> np.float32:
    """``div.rn.f32(fp32(lora_scale), fp32(alpha[0]))``: one IEEE binary32 division."""
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        return np.float32(lora_scale) / np.float32(alpha)


def fold(lb_bits, lora_scale: float, alpha: float):
    """Return ``(ratio, b_folded_bits)``: ``b_folded[i] = bf16_rne(fp32(lora_b[i]) * ratio)``.

    The product is one binary32 multiply; the rounding is nearest-even with NaN stored
    as 0x7FC0.
    """
    ratio = fold_ratio(lora_scale, alpha)
    lb32 = bf16_bits_to_f64(lb_bits).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        prod = lb32 * ratio
    return ratio, f32_to_bf16_rne(prod.astype(np.float32))


def eager_prepare_check(lora_scale: float, alpha: float) -> None:
    """The eager prepare's checks (prepare_nvfp4_lora_adapter page, Parameters: alpha and
    Returns): alpha == 0 is refused and the ratio must be finite; ValueError otherwise."""
    if np.float32(alpha) == 0.0:
        raise ValueError("alpha == 0: lora_scale / alpha is undefined")
    if not np.isfinite(fold_ratio(lora_scale, alpha)):
        raise ValueError("lora_scale / alpha is not finite")


# --------------------------------------------------------------------------------------
# The quantizer that produces a and a_sf (mm_nvfp4_lora page: the paragraph after the formula
# says the operands come "in the 128x4 swizzled layout produced by fp4_quantize()"; Parameters:
# alpha is "alpha_base / (a_global_scale * b_global_scale)", so dequant(codes, scales) carries
# a per-tensor global scale).  The pages name the quantizer but not its rule.  The reading
# taken, each step in float32 as the kernel computes it:
#   per 16-element block along K:  amax = max |x|                (x: bf16, exact in float32)
#   sf    = E4M3(rne, saturate to 448)( (amax * gs) / 6 )         (6 = largest E2M1 value)
#   inv   = gs / value(sf)               (sf == 0: every code of the block is +0)
#   code  = E2M1(rne, saturate to 6)( x * inv ),  sign kept, -0 for negatives rounding to 0
# so that value(code) * value(sf) / gs ~= x; scale rows past the last row are 0.
# --------------------------------------------------------------------------------------

#: the 127 finite non-negative E4M3 values, by code 0x00..0x7E
_E4M3_VALUES = decode_ue4m3(np.arange(0x7F, dtype=np.uint8))


def _round_to_table(v: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of the increasing table `values` to each v >= 0; a tie goes
    to the even index (the code whose last bit is 0); v above the last entry saturates."""
    v = np.asarray(v, dtype=np.float64)
    hi = np.searchsorted(values, v, side="left")          # first entry >= v
    hi = np.minimum(hi, len(values) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = v - values[lo]
    d_hi = values[hi] - v
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(v >= values[-1], len(values) - 1, idx)
    return idx


def e4m3_rne_satfinite(v: np.ndarray) -> np.ndarray:
    """float32 v >= 0 -> E4M3 code (round to nearest, ties to even, saturating at 448)."""
    v = np.asarray(v, dtype=np.float32)
    if np.any(~np.isfinite(v)) or np.any(v < 0):
        raise ValueError("scale input must be finite and non-negative")
    return _round_to_table(v.astype(np.float64), _E4M3_VALUES).astype(np.uint8)


def e2m1_rne_satfinite(q: np.ndarray) -> np.ndarray:
    """float32 q -> 4-bit E2M1 code: magnitude rounded to nearest (ties to even code), saturating
    at 6; bit 3 holds the sign (so a negative q that rounds to 0 gives -0, code 8)."""
    q = np.asarray(q, dtype=np.float32)
    if np.any(~np.isfinite(q)):
        raise ValueError("non-finite value to quantize")
    mag = _round_to_table(np.abs(q).astype(np.float64), E2M1_TABLE[:8]).astype(np.uint8)
    sign = np.signbit(q).astype(np.uint8) << 3
    return mag | sign


def quantize_nvfp4(x_bits: np.ndarray, global_scale: float):
    """bf16 bit patterns ``[R, K]`` -> (codes ``uint8 [R, K/2]``, swizzled scales of
    ``sf_buffer_bytes(R, K)`` bytes), by the reading above.  K must be a multiple of 64."""
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    rows, k = x_bits.shape
    if k % 64 != 0:
        raise ValueError("K must be a multiple of 64")
    gs = np.float32(global_scale)
    if not np.isfinite(gs) or gs <= 0:
        raise ValueError("global_scale must be positive and finite")
    x = (x_bits.astype(np.uint32) << 16).view(np.float32)            # exact bf16 -> fp32
    if np.any(~np.isfinite(x)):
        raise ValueError("non-finite input")
    blocks = x.reshape(rows, k // SF_VEC, SF_VEC)
    amax = np.max(np.abs(blocks), axis=2)                                # float32, exact
    sval = np.float32(amax * gs) / np.float32(6.0)                       # two float32 roundings
    sf = e4m3_rne_satfinite(sval)                                        # [rows, k/16] codes
    sfv = _E4M3_VALUES[sf].astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(sfv > 0, gs / np.where(sfv > 0, sfv, np.float32(1)), np.float32(0))
    q = (blocks * inv.astype(np.float32)[..., None]).astype(np.float32)  # float32 product
    codes = e2m1_rne_satfinite(q)
    codes = np.where((sfv > 0)[..., None], codes, np.uint8(0)).reshape(rows, k)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, swizzle_scales(sf, k, pad_value=0)


# --------------------------------------------------------------------------------------
# The routed-MoE FC2 LoRA delta (flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta page: the
# opening formula and Parameters).  For token t with adapter l = lora_ids[t] and routed slots j
# (expert e = topk_ids[t, j], combine weight w = topk_weights[t, j], activation row
# p = expanded_idx_to_permuted_idx[t * top_k + j]):
#     delta[t] = scale * sum_j w * ( B_down[l, e] @ ( A_down[l, e] @ act[p] ) )
# Readings taken where the page is silent:
#   * A_down[l, e] is the [rank, I] row-major block that starts l * lora_stride_a elements into
#     expert e's A bank (A_down @ act maps I -> rank); B_down[l, e] is the [H, rank] row-major
#     block l * lora_stride_b elements into expert e's B bank (B_down @ v maps rank -> H);
#   * the activation and both banks hold lora_dtype values (bf16 or fp16);
#   * a token whose lora id is negative gets an all-zero delta; a slot whose permuted index is
#     negative contributes nothing;
#   * scale is taken as a float32 value; the delta is formed in float64 here (its error far below
#     a float32 accumulation's) and rounded once to out_dtype (nearest, ties to even).
# --------------------------------------------------------------------------------------

def f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def f64_to_f16_rne(y: np.ndarray) -> np.ndarray:
    """Round float64 straight to binary16 bits: nearest, ties to even, one rounding.

    binary16 keeps 11 significant bits, normals down to 2**-14, subnormal quantum 2**-24 and a
    largest finite value of 65504.  The quantum of |y| in [2**(E-1), 2**E) is
    ``2**(max(E, -13) - 11)``; a rounded magnitude of 2**16 or more is infinity."""
    y = np.asarray(y, dtype=np.float64)
    sign = np.signbit(y)
    mag = np.abs(y)
    nz = np.isfinite(y) & (mag > 0)
    _, exp = np.frexp(np.where(nz, mag, 1.0))
    q = np.exp2((np.maximum(exp, -13) - 11).astype(np.float64))
    rounded = np.rint(np.where(nz, mag, 0.0) / q) * q
    overflow = nz & (rounded >= 2.0 ** 16)
    out = np.where(overflow, 0.0, rounded).astype(np.float16).view(np.uint16).copy()
    out[overflow | np.isinf(y)] = 0x7C00
    out = np.where(sign, out | 0x8000, out).astype(np.uint16)
    out[np.isnan(y)] = 0x7E00
    return out


def lora_values(bits, lora_dtype: str) -> np.ndarray:
    """bf16 or fp16 bit patterns -> float64."""
    if lora_dtype == "bf16":
        return bf16_bits_to_f64(bits)
    if lora_dtype == "fp16":
        return f16_bits_to_f64(bits)
    raise ValueError("lora_dtype must be 'bf16' or 'fp16'")


def round_to(y: np.ndarray, out_dtype: str) -> np.ndarray:
    """The single rounding of the delta to out_dtype (bf16 or fp16 bits)."""
    if out_dtype == "bf16":
        return f64_to_bf16_rne(y)
    if out_dtype == "fp16":
        return f64_to_f16_rne(y)
    raise ValueError("out_dtype must be 'bf16' or 'fp16'")


def bgmv_moe_lora_delta(act_bits, perm, a_banks, lora_stride_a: int, b_banks, lora_stride_b: int,
                        topk_ids, topk_weights, lora_ids, rank: int, hidden_size: int, scale: float,
                        lora_dtype: str = "bf16", tokens=None) -> np.ndarray:
    """float64 delta rows [len(tokens) or T, H] before the output rounding.

    act_bits: [padded_rows, I] bit patterns; perm: [T * top_k]; a_banks / b_banks: one flat bit
    array per expert (the memory each pointer-table entry points at); topk_ids, topk_weights:
    [T, top_k]; lora_ids: [T].  ``tokens`` selects the rows to evaluate (all when None)."""
    act = lora_values(act_bits, lora_dtype)
    rows, I = act.shape
    ids = np.asarray(topk_ids, dtype=np.int64)
    T, top_k = ids.shape
    w = np.asarray(topk_weights, dtype=np.float32).astype(np.float64)
    perm = np.asarray(perm, dtype=np.int64).reshape(T * top_k)
    lids = np.asarray(lora_ids, dtype=np.int64).reshape(T)
    s = float(np.float32(scale))
    H = int(hidden_size)
    sel = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64).reshape(-1)
    out = np.zeros((sel.size, H), dtype=np.float64)
    for i, t in enumerate(sel):
        l = int(lids[t])
        if l < 0:
            continue
        acc = np.zeros(H, dtype=np.float64)
        for j in range(top_k):
            p = int(perm[t * top_k + j])
            if p < 0:
                continue
            if p >= rows:
                raise ValueError("permuted index past the activation rows")
            e = int(ids[t, j])
            a0 = l * int(lora_stride_a)
            b0 = l * int(lora_stride_b)
            A = lora_values(np.asarray(a_banks[e]).reshape(-1)[a0:a0 + rank * I], lora_dtype).reshape(rank, I)
            B = lora_values(np.asarray(b_banks[e]).reshape(-1)[b0:b0 + H * rank], lora_dtype).reshape(H, rank)
            v = A @ act[p]                      # [rank]
            acc += w[t, j] * (B @ v)            # [H]
        out[i] = s * acc
    return out


# --------------------------------------------------------------------------------------
# Acceptance measures
# --------------------------------------------------------------------------------------

def tolerance(y_ref: np.ndarray) -> np.ndarray:
    """Per-element bound ``2**-7*|ref| + 2**-10*max|ref|`` on ``|gpu - ref|``."""
    y_ref = np.asarray(y_ref, dtype=np.float64)
    return 2.0 ** -7 * np.abs(y_ref) + 2.0 ** -10 * np.max(np.abs(y_ref))


def sqnr_db(y_ref: np.ndarray, y_test: np.ndarray) -> float:
    """``10*log10(sum(ref**2) / sum((test - ref)**2))``; infinite when they agree."""
    y_ref = np.asarray(y_ref, dtype=np.float64)
    err = np.sum((np.asarray(y_test, dtype=np.float64) - y_ref) ** 2)
    sig = np.sum(y_ref ** 2)
    if err == 0.0:
        return float("inf")
    return float(10.0 * np.log10(sig / err))
