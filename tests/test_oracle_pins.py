"""Pins of the CPU oracle against what the formats, the pages and mathematics fix.

None of these re-types the oracle's formulas: each expected value comes from a
different route (a library decoder, a closed form written from the format
definition, a brute-force loop, a second formulation of the layout, or an invariant),
chosen so that a dropped term, a wrong sign or index, a swapped nibble or a
transposed operand in the oracle fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------------------
# independent decoders used only by the tests
# ---------------------------------------------------------------------------------------

def e2m1_closed_form(code: int) -> float:
    """E2M1 from its bit fields: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return s * 0.5 * m
    return s * (2.0 ** (e - 1)) * (1.0 + 0.5 * m)


def ue4m3_library(byte_values) -> np.ndarray:
    """UE4M3 through PyTorch's float8_e4m3fn decoder (bit 7 = sign = 0)."""
    t = torch.tensor(np.asarray(byte_values, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.float().numpy().astype(np.float64)


def swizzle_by_permute(logical: np.ndarray, k: int) -> np.ndarray:
    """128x4 layout as a reshape/permute of the padded logical matrix:
    [R/128, 4, 32, C/4, 4] -> [R/128, C/4, 32, 4, 4]."""
    rows, c = logical.shape
    rp = -(-rows // 128) * 128
    pad = torch.zeros((rp, c), dtype=torch.uint8)
    pad[:rows] = torch.from_numpy(logical)
    v = pad.view(rp // 128, 4, 32, c // 4, 4).permute(0, 3, 2, 1, 4).contiguous()
    return v.view(-1).numpy()


def brute_base(a, b, a_sf_logical, b_sf_logical, M, N, K):
    """Pure-Python triple loop with the closed-form decoders above."""
    out = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for kk in range(K):
                ab = int(a[m, kk // 2]); bb = int(b[n, kk // 2])
                ca = (ab >> 4) if kk % 2 else (ab & 15)
                cb = (bb >> 4) if kk % 2 else (bb & 15)
                sa = ue4m3_library([a_sf_logical[m, kk // 16]])[0]
                sb = ue4m3_library([b_sf_logical[n, kk // 16]])[0]
                acc += e2m1_closed_form(ca) * e2m1_closed_form(cb) * sa * sb
            out[m, n] = acc
    return out


# ---------------------------------------------------------------------------------------
# formats
# ---------------------------------------------------------------------------------------

def test_e2m1_table_matches_bit_fields():
    for code in range(16):
        got = O.E2M1_TABLE[code]
        want = e2m1_closed_form(code)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), code
    # negation symmetry: flipping the sign bit negates
    for code in range(8):
        assert O.E2M1_TABLE[code ^ 8] == -O.E2M1_TABLE[code]


def test_e2m1_nibble_order_low_first():
    packed = np.array([[0x71, 0x0F]], dtype=np.uint8)   # codes 1,7 then 15,0
    vals = O.decode_e2m1(packed)
    assert vals.tolist() == [[0.5, 6.0, -6.0, 0.0]]


def test_ue4m3_all_bytes_vs_torch_float8():
    x = np.arange(128, dtype=np.uint8)
    got = O.decode_ue4m3(x)
    want = ue4m3_library(x)
    assert np.isnan(got[0x7F]) and np.isnan(want[0x7F])
    np.testing.assert_array_equal(got[:0x7F], want[:0x7F])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0
    assert np.all(np.diff(got[:0x7F]) > 0)                     # strictly monotone


def test_ue4m3_rejects_sign_bit():
    with pytest.raises(ValueError):
        O.decode_ue4m3(np.array([0x80], dtype=np.uint8))


def test_config_scale_range_is_positive_e4m3_in_quarter_to_four():
    codes = np.arange(0x28, 0x49, dtype=np.uint8)
    vals = O.decode_ue4m3(codes)
    assert len(codes) == 33 and vals[0] == 0.25 and vals[-1] == 4.0
    allv = ue4m3_library(np.arange(0x7F, dtype=np.uint8))
    inrange = allv[(allv >= 0.25) & (allv <= 4.0)]
    np.testing.assert_array_equal(np.sort(inrange), vals)


# ---------------------------------------------------------------------------------------
# 128x4 swizzle
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,k", [(1, 64), (128, 256), (200, 512), (300, 128)])
def test_swizzle_is_a_bijection_and_matches_permute(rows, k):
    rp = -(-rows // 128) * 128
    c = k // 16
    rr, cc = np.meshgrid(np.arange(rp), np.arange(c), indexing="ij")
    offs = O.sf_offset(rr, cc, k).ravel()
    assert sorted(offs.tolist()) == list(range(rp * c))
    rng = np.random.default_rng(rows + k)
    logical = rng.integers(0, 127, size=(rows, c), dtype=np.uint8)
    buf = O.swizzle_scales(logical, k)
    np.testing.assert_array_equal(buf, swizzle_by_permute(logical, k))
    np.testing.assert_array_equal(O.unswizzle_scales(buf, rows, k), logical)


def test_unswizzle_accepts_larger_buffer_and_rejects_short():
    logical = np.full((5, 4), 0x38, dtype=np.uint8)
    buf = O.swizzle_scales(logical, 64)
    big = np.concatenate([buf, np.full(999, 0x7F, dtype=np.uint8)])
    np.testing.assert_array_equal(O.unswizzle_scales(big, 5, 64), logical)
    with pytest.raises(ValueError):
        O.unswizzle_scales(buf[:-1], 5, 64)


# ---------------------------------------------------------------------------------------
# base product
# ---------------------------------------------------------------------------------------

def test_single_block_all_byte_pairs():
    """Every (a byte, b byte) pair in one 16-block: sa*sb*(lo*lo + hi*hi)."""
    K = 64
    M = N = 256
    a = np.zeros((M, K // 2), dtype=np.uint8); a[:, 0] = np.arange(256)
    b = np.zeros((N, K // 2), dtype=np.uint8); b[:, 0] = np.arange(256)
    rng = np.random.default_rng(7)
    sa = rng.integers(0x28, 0x49, size=(M, K // 16), dtype=np.uint8)
    sb = rng.integers(0x28, 0x49, size=(N, K // 16), dtype=np.uint8)
    got = O.base_product(a, b, O.swizzle_scales(sa, K), O.swizzle_scales(sb, K), M, N, K)
    lo = np.array([e2m1_closed_form(i & 15) for i in range(256)])
    hi = np.array([e2m1_closed_form(i >> 4) for i in range(256)])
    want = (np.outer(lo, lo) + np.outer(hi, hi)) * np.outer(ue4m3_library(sa[:, 0]),
                                                            ue4m3_library(sb[:, 0]))
    np.testing.assert_array_equal(got, want)


def test_brute_force_small_random():
    M, N, K = 3, 5, 128
    rng = np.random.default_rng(11)
    a = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    b = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = rng.integers(0x01, 0x7F, size=(M, K // 16), dtype=np.uint8)   # full finite range
    sb = rng.integers(0x01, 0x7F, size=(N, K // 16), dtype=np.uint8)
    want = brute_base(a, b, sa, sb, M, N, K)
    got = O.base_product(a, b, swizzle_by_permute(sa, K), swizzle_by_permute(sb, K), M, N, K)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=0)
    for m in range(M):
        for n in range(N):
            e = O.base_element(a, b, swizzle_by_permute(sa, K), swizzle_by_permute(sb, K),
                               M, N, K, m, n)
            assert abs(e - want[m, n]) <= 1e-13 * max(1.0, abs(want[m, n]))


def test_all_ones_gives_k():
    M, N, K = 130, 7, 512
    a = np.full((M, K // 2), 0x22, dtype=np.uint8)       # both nibbles 1.0
    b = np.full((N, K // 2), 0x22, dtype=np.uint8)
    sa = np.full(O.sf_buffer_bytes(M, K), 0x38, dtype=np.uint8)   # 1.0
    sb = np.full(O.sf_buffer_bytes(N, K), 0x38, dtype=np.uint8)
    got = O.base_product(a, b, sa, sb, M, N, K)
    assert np.all(got == K)


@pytest.mark.parametrize("k_idx", [0, 1, 15, 16, 17, 63, 64, 65, 127, 191, 255])
def test_one_hot_lands_on_one_output(k_idx):
    M, N, K = 40, 140, 256
    m0, n0 = 37, 133
    a = np.zeros((M, K // 2), dtype=np.uint8)
    b = np.zeros((N, K // 2), dtype=np.uint8)
    a[m0, k_idx // 2] = (0x5 << 4) if k_idx % 2 else 0x5     # 3.0
    b[n0, k_idx // 2] = (0xB << 4) if k_idx % 2 else 0xB     # -1.5
    sa_l = np.full((M, K // 16), 0x38, dtype=np.uint8)
    sb_l = np.full((N, K // 16), 0x38, dtype=np.uint8)
    sa_l[m0, k_idx // 16] = 0x40          # 2.0
    sb_l[n0, k_idx // 16] = 0x29          # 0.28125
    got = O.base_product(a, b, swizzle_by_permute(sa_l, K), swizzle_by_permute(sb_l, K),
                         M, N, K)
    want = np.zeros((M, N)); want[m0, n0] = 3.0 * -1.5 * 2.0 * 0.28125
    np.testing.assert_array_equal(got, want)


def test_golden_hand_computed_case():
    with open(os.path.join(GOLDEN, "hand_case.json")) as f:
        g = json.load(f)
    M, N, K, r = g["M"], g["N"], g["K"], g["r"]
    a = np.array(g["a"], dtype=np.uint8).reshape(M, K // 2)
    b = np.array(g["b"], dtype=np.uint8).reshape(N, K // 2)
    sa = O.swizzle_scales(np.array(g["a_sf_logical"], dtype=np.uint8).reshape(M, K // 16), K)
    sb = O.swizzle_scales(np.array(g["b_sf_logical"], dtype=np.uint8).reshape(N, K // 16), K)
    d = np.array(g["d_bits"], dtype=np.uint16)
    lb = np.array(g["lora_b_bits"], dtype=np.uint16)
    bias = np.array(g["bias_bits"], dtype=np.uint16)
    y = O.mm_raw(a, b, sa, sb, g["alpha"], d, lb, g["lora_scale"], bias, M, N, K, r)
    np.testing.assert_array_equal(y.ravel(), np.array(g["expected_y"]))
    np.testing.assert_array_equal(O.round_output(y).ravel(),
                                  np.array(g["expected_out_bits"], dtype=np.uint16))


# ---------------------------------------------------------------------------------------
# rounding
# ---------------------------------------------------------------------------------------

def test_f64_to_bf16_matches_torch_on_float32_values():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    x32 = bits.view(np.float32)
    x32 = x32[~np.isnan(x32)]
    got = O.f64_to_bf16_rne(x32.astype(np.float64))
    want = torch.from_numpy(x32.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)
    got32 = O.f32_to_bf16_rne(x32)
    np.testing.assert_array_equal(got32, want)


def test_f64_to_bf16_single_rounding_cases():
    one = 1.0
    cases = [
        (one + 2.0 ** -8, 0x3F80),                    # tie -> even (down)
        (one + 2.0 ** -8 + 2.0 ** -40, 0x3F81),       # just above the tie: up (f32 route says down)
        (one + 3 * 2.0 ** -8, 0x3F82),                # tie -> even (up)
        (-(one + 2.0 ** -8 + 2.0 ** -40), 0xBF81),
        ((2 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),       # tie at the top -> even = infinity
        ((2 - 2.0 ** -8 - 2.0 ** -30) * 2.0 ** 127, 0x7F7F),
        (2.0 ** -133, 0x0001),                        # smallest subnormal
        (2.0 ** -134, 0x0000),                        # tie -> even (zero)
        (1.5 * 2.0 ** -134, 0x0001),
        (2.0 ** -126, 0x0080),                        # smallest normal
        (0.0, 0x0000),
        (-0.0, 0x8000),
        (float("inf"), 0x7F80),
        (float("-inf"), 0xFF80),
        (1e300, 0x7F80),
    ]
    ys = np.array([c[0] for c in cases])
    got = O.f64_to_bf16_rne(ys)
    assert [int(v) for v in got] == [c[1] for c in cases]
    assert int(O.f64_to_bf16_rne(np.array([float("nan")]))[0]) == 0x7FC0


# ---------------------------------------------------------------------------------------
# fold
# ---------------------------------------------------------------------------------------

FOLD_PAIRS = [(0.25, 2.0 ** -10), (2.0, 2.0 ** -9), (0.5, 3.0), (1.7, -0.013), (0.0, 2.0 ** -9),
              (-0.0, 1.0), (3.999, 1e-30), (1e-30, 3.0), (7.0, 1e-38)]


@pytest.mark.parametrize("s,alpha", FOLD_PAIRS)
def test_fold_matches_torch_mul_exhaustive(s, alpha):
    lb_bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ratio, got = O.fold(lb_bits, s, alpha)
    st = torch.tensor([s], dtype=torch.float32)
    at = torch.tensor([alpha], dtype=torch.float32)
    rt = (st / at[0])
    assert np.float32(rt.item()) == ratio or (np.isnan(ratio) and math.isnan(rt.item()))
    lb = torch.from_numpy(lb_bits.view(np.int16).copy()).view(torch.bfloat16)
    want = (lb * rt[0]).view(torch.int16).numpy().view(np.uint16)
    gotf = (got.astype(np.uint32) << 16).view(np.float32)
    wantf = (want.astype(np.uint32) << 16).view(np.float32)
    nan_g, nan_w = np.isnan(gotf), np.isnan(wantf)
    np.testing.assert_array_equal(nan_g, nan_w)
    np.testing.assert_array_equal(got[~nan_g], want[~nan_w])
    assert np.all(got[nan_g] == 0x7FC0)


def test_fold_exact_when_ratio_is_power_of_two():
    rng = np.random.default_rng(5)
    lb = (torch.from_numpy(rng.standard_normal(4096).astype(np.float32)) * 0.02).to(torch.bfloat16)
    bits = lb.view(torch.int16).numpy().view(np.uint16)
    ratio, folded = O.fold(bits, 0.25, 2.0 ** -10)
    assert ratio == np.float32(256.0)
    np.testing.assert_array_equal(O.bf16_bits_to_f64(folded), O.bf16_bits_to_f64(bits) * 256.0)


def test_eager_checks():
    with pytest.raises(ValueError):
        O.eager_prepare_check(1.0, 0.0)
    with pytest.raises(ValueError):
        O.eager_prepare_check(1.0, -0.0)
    with pytest.raises(ValueError):
        O.eager_prepare_check(3e38, 1e-10)       # ratio overflows
    with pytest.raises(ValueError):
        O.eager_prepare_check(float("nan"), 1.0)
    O.eager_prepare_check(0.0, 1.0)               # the zero adapter is allowed


# ---------------------------------------------------------------------------------------
# epilogue algebra and invariants
# ---------------------------------------------------------------------------------------

def _small_problem(seed, M=33, N=70, K=256, r=16, bias=True):
    from workloads import make_problem
    p = make_problem(M, N, K, r, seed, alpha=2.0 ** -6, lora_scale=1.5, bias=bias)
    npy = dict(a=p.a.numpy(), b=p.b.numpy(), a_sf=p.a_sf.numpy(), b_sf=p.b_sf.numpy(),
               d=p.d.view(torch.int16).numpy().view(np.uint16),
               lb=p.lora_b.view(torch.int16).numpy().view(np.uint16),
               bias=None if p.bias is None else p.bias.view(torch.int16).numpy().view(np.uint16))
    return p, npy


def test_zero_adapter_is_bitwise_adapter_off_even_with_nonfinite_d():
    p, x = _small_problem(21)
    d = x["d"].copy(); d[0, 0] = 0x7F80; d[1, 3] = 0x7FC1       # inf, NaN
    off = O.mm_off(x["a"], x["b"], x["a_sf"], x["b_sf"], p.alpha, x["bias"], p.M, p.N, p.K)
    for s in (0.0, -0.0, None):
        raw = O.mm_raw(x["a"], x["b"], x["a_sf"], x["b_sf"], p.alpha, d, x["lb"], s, x["bias"],
                       p.M, p.N, p.K, p.r)
        np.testing.assert_array_equal(raw.view(np.uint64), off.view(np.uint64))
    prep = O.mm_prepared(x["a"], x["b"], x["a_sf"], x["b_sf"], p.alpha, d, x["lb"], 0.0,
                         x["bias"], p.M, p.N, p.K, p.r)
    np.testing.assert_array_equal(prep.view(np.uint64), off.view(np.uint64))


def test_raw_minus_off_is_the_lora_term_closed_form():
    """alpha = 0 isolates s * (d @ lora_b^T) + bias, checked by an explicit loop."""
    p, x = _small_problem(22, M=5, N=9, r=24)
    y = O.mm_raw(x["a"], x["b"], x["a_sf"], x["b_sf"], 0.0, x["d"], x["lb"], 1.5, x["bias"],
                 p.M, p.N, p.K, p.r)
    d = p.d.double().numpy(); lb = p.lora_b.double().numpy(); bias = p.bias.double().numpy()
    for m in range(p.M):
        for n in range(p.N):
            want = 1.5 * sum(d[m, j] * lb[n, j] for j in range(p.r)) + bias[n]
            assert abs(y[m, n] - want) <= 1e-14 * max(1.0, abs(want))


def test_raw_vs_prepared_agree_within_fold_rounding():
    p, x = _small_problem(23, M=64, N=96, r=32)
    for s, alpha in [(1.5, 2.0 ** -6), (0.3, 0.0071)]:
        ratio, bf = O.fold(x["lb"], s, alpha)
        y_raw = O.mm_raw(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], x["lb"], s,
                         x["bias"], p.M, p.N, p.K, p.r)
        y_prep = O.mm_prepared(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], bf, ratio,
                               x["bias"], p.M, p.N, p.K, p.r)
        d = np.abs(O.bf16_bits_to_f64(x["d"])); lb = np.abs(O.bf16_bits_to_f64(x["lb"]))
        bound = abs(s) * (d @ lb.T) * (2.0 ** -9 + 2.0 ** -22) + 1e-12 * np.abs(y_raw)
        assert np.all(np.abs(y_raw - y_prep) <= bound)
        assert np.any(y_raw != y_prep) or s == 1.5   # the fold does change something


def test_raw_vs_prepared_equal_when_fold_is_exact():
    p, x = _small_problem(24, M=32, N=48, r=64, bias=False)
    s, alpha = 0.25, 2.0 ** -10          # ratio 256, exact
    ratio, bf = O.fold(x["lb"], s, alpha)
    y_raw = O.mm_raw(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], x["lb"], s, None,
                     p.M, p.N, p.K, p.r)
    y_prep = O.mm_prepared(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], bf, ratio, None,
                           p.M, p.N, p.K, p.r)
    np.testing.assert_allclose(y_prep, y_raw, rtol=1e-15, atol=1e-300)


def test_sampled_call_forms_equal_the_full_forms_on_their_outputs():
    """The rows / cols forms (used at full sizes) give exactly the selected block of the full
    call forms, for unsorted, repeated and edge indices, with the brute-force loop as the anchor
    of one element."""
    p, x = _small_problem(25, M=40, N=72, K=512, r=24)
    rows = np.array([39, 0, 17, 17, 5])
    cols = np.array([71, 3, 0, 64, 64, 33])
    sel = np.ix_(rows, cols)
    s, alpha = 1.5, p.alpha
    ratio, bf = O.fold(x["lb"], s, alpha)
    full = {
        "raw": O.mm_raw(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], x["lb"], s, x["bias"],
                        p.M, p.N, p.K, p.r),
        "prepared": O.mm_prepared(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], bf, ratio, x["bias"],
                                  p.M, p.N, p.K, p.r),
        "off": O.mm_off(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["bias"], p.M, p.N, p.K),
    }
    part = {
        "raw": O.mm_raw(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], x["lb"], s, x["bias"],
                        p.M, p.N, p.K, p.r, rows=rows, cols=cols),
        "prepared": O.mm_prepared(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["d"], bf, ratio, x["bias"],
                                  p.M, p.N, p.K, p.r, rows=rows, cols=cols),
        "off": O.mm_off(x["a"], x["b"], x["a_sf"], x["b_sf"], alpha, x["bias"], p.M, p.N, p.K,
                        rows=rows, cols=cols),
    }
    for k in full:
        assert part[k].shape == (len(rows), len(cols)), k
        np.testing.assert_allclose(part[k], full[k][sel], rtol=1e-14, atol=0, err_msg=k)
    # one element of the raw form against the block-by-block sum written out here
    m, n = 39, 71
    a_log = O.unswizzle_scales(x["a_sf"], p.M, p.K); b_log = O.unswizzle_scales(x["b_sf"], p.N, p.K)
    base = brute_base(x["a"][m:m + 1], x["b"][n:n + 1], a_log[m:m + 1], b_log[n:n + 1], 1, 1, p.K)[0, 0]
    dl = p.d.double().numpy()[m] @ p.lora_b.double().numpy()[n]
    want = alpha * base + s * dl + p.bias.double().numpy()[n]
    assert abs(part["raw"][0, 0] - want) <= 1e-12 * max(1.0, abs(want))


def _grouped_inputs(seg, N, K, r, seed, bias=True):
    rng = np.random.default_rng(seed)
    ind = np.concatenate([[0], np.cumsum(seg)]).astype(np.int64)
    rows = int(ind[-1]) + 128                  # rows past the last segment are padding
    E = len(seg)
    a = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    b = rng.integers(0, 256, (E, N, K // 2), dtype=np.uint8)
    a_sf = rng.integers(0x01, 0x7F, O.sf_buffer_bytes(rows, K), dtype=np.uint8)
    b_sf = rng.integers(0x01, 0x7F, E * O.sf_buffer_bytes(N, K), dtype=np.uint8)
    alpha = rng.uniform(-1, 1, E)
    d = O.f32_to_bf16_rne(rng.standard_normal((rows, r)).astype(np.float32))
    lb = O.f32_to_bf16_rne((0.02 * rng.standard_normal((E, N, r))).astype(np.float32))
    bias = O.f32_to_bf16_rne((0.1 * rng.standard_normal((E, N))).astype(np.float32)) if bias else None
    return ind, rows, a, b, a_sf, b_sf, alpha, d, lb, bias


def test_grouped_form_against_a_brute_force_loop():
    """Tiny grouped call (an empty expert included) against a per-row, per-element loop with the
    closed-form decoders: expert of each row from m_indptr, its own b, scales, alpha, lora_b, bias."""
    N, K, r = 3, 64, 8
    ind, rows, a, b, a_sf, b_sf, alpha, d, lb, bias = _grouped_inputs([128, 0, 256], N, K, r, 31)
    s = 0.75
    y = O.grouped_mm(a, b, a_sf, b_sf, ind, alpha, d, lb, s, bias, rows, N, K, r)
    a_log = O.unswizzle_scales(a_sf, rows, K)
    dd = O.bf16_bits_to_f64(d); ll = O.bf16_bits_to_f64(lb); bb = O.bf16_bits_to_f64(bias)
    rng = np.random.default_rng(5)
    for m in list(rng.choice(int(ind[-1]), 40, replace=False)) + [0, 127, 128, 383]:
        e = int(np.searchsorted(ind, m, side="right") - 1)
        b_log = O.unswizzle_scales(b_sf[e * O.sf_buffer_bytes(N, K):(e + 1) * O.sf_buffer_bytes(N, K)], N, K)
        for n in range(N):
            base = brute_base(a[m:m + 1], b[e, n:n + 1], a_log[m:m + 1], b_log[n:n + 1], 1, 1, K)[0, 0]
            want = alpha[e] * base + s * float(dd[m] @ ll[e, n]) + bb[e, n]
            assert abs(y[m, n] - want) <= 1e-12 * max(1.0, abs(want)), (m, n)


def test_grouped_single_expert_is_the_plain_call_and_rules_are_checked():
    N, K, r = 40, 128, 16
    ind, rows, a, b, a_sf, b_sf, alpha, d, lb, bias = _grouped_inputs([256], N, K, r, 32, bias=False)
    y = O.grouped_mm(a, b, a_sf, b_sf, ind, alpha, d, lb, None, None, rows, N, K, r)
    want = O.mm_off(a[:256], b[0], a_sf[:O.sf_buffer_bytes(256, K)], b_sf, alpha[0], None, 256, N, K)
    np.testing.assert_array_equal(y, want)
    for bad in ([0, 100], [128, 256], [0, 256, 128], [0, rows + 128], [0]):
        with pytest.raises(ValueError):
            O.check_grouped_indptr(bad, rows)


def test_measures():
    y = np.array([1.0, -2.0, 4.0])
    assert O.sqnr_db(y, y) == float("inf")
    assert abs(O.sqnr_db(y, y + np.array([0.0, 0.0, 0.21])) - 10 * np.log10(21 / 0.0441)) < 1e-9
    np.testing.assert_array_equal(O.tolerance(y), 2.0 ** -7 * np.abs(y) + 2.0 ** -10 * 4.0)


# ---------------------------------------------------------------------------------------
# the quantizer (the reading of fp4_quantize: per-16-block amax, UE4M3 scale, E2M1 codes)
# ---------------------------------------------------------------------------------------

def _e2m1_nearest_even_brute(q: float) -> int:
    """Brute force over the 8 magnitudes: nearest, ties to the even code, saturate at 6."""
    mag = abs(q)
    best, best_d = 0, None
    for code in range(8):
        d = abs(e2m1_closed_form(code) - mag)
        if best_d is None or d < best_d or (d == best_d and code % 2 == 0):
            best, best_d = code, d
    if mag >= 6.0:
        best = 7
    return best | (8 if math.copysign(1.0, q) < 0 else 0)


def test_e2m1_rounding_matches_brute_force():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0]
    vals = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 6.5, 9.0, 1e30, 0.1, 0.2499, 0.2501, 2.9, 4.99, 5.01]
    qs = []
    for v in mids + vals:
        qs += [v, -v, np.nextafter(np.float32(v), np.float32(0)), np.nextafter(np.float32(v), np.float32(1e38))]
    qs = np.array(qs, dtype=np.float32)
    got = O.e2m1_rne_satfinite(qs)
    want = np.array([_e2m1_nearest_even_brute(float(q)) for q in qs], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)
    # the ties, written out from the format: 0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2,
    # 2.5 -> 2, 3.5 -> 4, 5 -> 4; a negative value that rounds to 0 keeps its sign (-0 = code 8)
    np.testing.assert_array_equal(O.e2m1_rne_satfinite(np.array(mids[:7], dtype=np.float32)),
                                  np.array([0, 2, 2, 4, 4, 6, 6], dtype=np.uint8))
    assert O.e2m1_rne_satfinite(np.array([-0.2], dtype=np.float32))[0] == 8


def test_e4m3_rounding_matches_torch_float8_in_range():
    vals = O.decode_ue4m3(np.arange(0x7F, dtype=np.uint8))
    mids = (vals[1:] + vals[:-1]) / 2
    rng = np.random.default_rng(4)
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                        rng.uniform(0, 448, 4000), np.exp2(rng.uniform(-12, 8.8, 4000))])
    x = x[x <= 448].astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(O.e4m3_rne_satfinite(x), want)


def test_e4m3_saturation_and_underflow():
    x = np.array([448.0, 449.0, 464.0, 465.0, 1e20, 0.0, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -9], dtype=np.float32)
    np.testing.assert_array_equal(O.e4m3_rne_satfinite(x),
                                  np.array([0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0, 0, 2, 1], dtype=np.uint8))


def _bf16_bits(x64: np.ndarray) -> np.ndarray:
    x32 = np.asarray(x64, dtype=np.float32)
    bits = x32.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (bits >> 16).astype(np.uint16)


def _round_bf16_bits(x64: np.ndarray) -> np.ndarray:
    """Round to bf16 through PyTorch (a route independent of the oracle)."""
    t = torch.from_numpy(np.asarray(x64, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("rows,k", [(1, 64), (130, 256), (256, 512)])
def test_quantize_round_trip_exact(rows, k):
    """x built as code * scale / gs with one |6| code per block (so the block's amax fixes the
    scale exactly) quantizes back to the same codes and scale bytes."""
    rng = np.random.default_rng(rows + k)
    nb = k // 16
    codes = rng.integers(0, 16, size=(rows, k)).astype(np.uint8)
    codes[:, ::16] = np.where(rng.random((rows, nb)) < 0.5, 7, 15)       # a +-6 in every block
    sf = rng.integers(0x20, 0x60, size=(rows, nb)).astype(np.uint8)      # 2**-3 .. 2**4
    gs = 2.0 ** 5
    vals = np.array([e2m1_closed_form(c) for c in range(16)])[codes]
    x = vals * np.repeat(ue4m3_library(sf.ravel()).reshape(rows, nb), 16, axis=1) / gs
    packed, sf_buf = O.quantize_nvfp4(_bf16_bits(x), gs)
    codes_back = np.empty((rows, k), dtype=np.uint8)
    codes_back[:, 0::2] = packed & 0x0F
    codes_back[:, 1::2] = packed >> 4
    np.testing.assert_array_equal(O.unswizzle_scales(sf_buf, rows, k), sf)
    # codes 0 (+0) and 8 (-0) come back as they went in: the sign of a zero survives
    np.testing.assert_array_equal(codes_back, codes)


def test_quantize_zero_block_saturation_and_padding():
    rows, k = 3, 64
    x = np.zeros((rows, k), dtype=np.float64)
    x[1, :16] = 1.0e4              # amax * gs / 6 far above 448: scale saturates, codes saturate
    x[1, 5] = -3.0e4
    x[2, 16:32] = np.linspace(-1, 1, 16)
    packed, sf_buf = O.quantize_nvfp4(_round_bf16_bits(x), 1.0)
    sf = O.unswizzle_scales(sf_buf, rows, k)
    assert sf[0].tolist() == [0, 0, 0, 0] and packed[0].tolist() == [0] * 32
    assert sf[1, 0] == 0x7E
    lo, hi = packed[1, :8] & 0x0F, packed[1, :8] >> 4
    blk = np.empty(16, dtype=np.uint8)
    blk[0::2], blk[1::2] = lo, hi
    assert blk[5] == 15 and np.all(np.delete(blk, 5) == 7)        # -6 and +6 (saturated)
    # scale bytes of the padded rows 3..127 are 0
    full = np.frombuffer(sf_buf.tobytes(), dtype=np.uint8)
    mask = np.ones(full.size, dtype=bool)
    rr, cc = np.meshgrid(np.arange(rows), np.arange(k // 16), indexing="ij")
    mask[O.sf_offset(rr, cc, k)] = False
    assert np.all(full[mask] == 0)


def test_quantize_error_bound_random():
    """dequant(quant(x)) / gs stays within amax/6 * (1 + 2**-3) of x in every block."""
    rng = np.random.default_rng(9)
    rows, k = 64, 256
    x = rng.standard_normal((rows, k)) * np.exp2(rng.integers(-6, 6, size=(rows, 1)))
    xb = _round_bf16_bits(x)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    amax = np.abs(xf).max()
    gs = 448.0 * 6.0 / amax
    packed, sf_buf = O.quantize_nvfp4(xb, gs)
    back = O.dequant(packed, sf_buf, rows, k) / np.float32(gs)
    blk_amax = np.repeat(np.abs(xf).reshape(rows, k // 16, 16).max(axis=2), 16, axis=1)
    assert np.all(np.abs(back - xf) <= blk_amax / 6.0 * (1 + 2.0 ** -3))


# ---------------------------------------------------------------------------------------
# the routed-MoE FC2 LoRA delta (flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta page)
# ---------------------------------------------------------------------------------------

def _half_closed_form(bits: int, dtype: str) -> float:
    """bf16 / binary16 from the bit fields (bf16: 8 exponent bits, bias 127, 7 mantissa bits;
    binary16: 5 exponent bits, bias 15, 10 mantissa bits); finite values only."""
    eb, mb = (8, 7) if dtype == "bf16" else (5, 10)
    bias = (1 << (eb - 1)) - 1
    s = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> mb) & ((1 << eb) - 1)
    m = bits & ((1 << mb) - 1)
    assert e != (1 << eb) - 1
    if e == 0:
        return s * m * 2.0 ** (1 - bias - mb)
    return s * (1.0 + m * 2.0 ** -mb) * 2.0 ** (e - bias)


def _bits_of(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bgmv_args(p, dtype: str):
    return dict(act_bits=_bits_of(p.act), perm=p.perm.numpy(), a_banks=[_bits_of(x) for x in p.a_banks],
                lora_stride_a=p.stride_a, b_banks=[_bits_of(x) for x in p.b_banks], lora_stride_b=p.stride_b,
                topk_ids=p.topk_ids.numpy(), topk_weights=p.topk_weights.numpy(), lora_ids=p.lora_ids.numpy(),
                rank=p.rank, hidden_size=p.H, scale=p.scale, lora_dtype=dtype)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_bgmv_delta_against_a_brute_force_loop(dtype):
    """Per element, in pure Python with the bit-field decoders: the page's sum over slots of
    w * sum_k B[h, k] * sum_i A[k, i] * act[p, i], times scale; adapters addressed by stride
    (with NaN padding between blocks, so a wrong offset shows), skipped tokens and slots."""
    import workloads as W
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    p = W.make_bgmv_problem(6, 3, 4, 3, 16, 8, 8, seed=11, lora_dtype=tdt, scale=1.5, p_no_lora=0.2,
                            p_inactive=0.2, stride_pad=8, seg_align=4)
    p.topk_weights[2, 1] = -0.75                     # a negative combine weight
    args = _bgmv_args(p, dtype)
    got = O.bgmv_moe_lora_delta(**args)
    act, ab, bb = args["act_bits"], args["a_banks"], args["b_banks"]
    want = np.zeros((p.T, p.H))
    for t in range(p.T):
        l = int(p.lora_ids[t])
        if l < 0:
            continue
        for h in range(p.H):
            acc = 0.0
            for j in range(p.top_k):
                row = int(p.perm[t * p.top_k + j])
                if row < 0:
                    continue
                e = int(p.topk_ids[t, j])
                u = 0.0
                for k in range(p.rank):
                    v = 0.0
                    for i in range(p.I):
                        av = _half_closed_form(int(ab[e][l * p.stride_a + k * p.I + i]), dtype)
                        v += av * _half_closed_form(int(act[row, i]), dtype)
                    u += _half_closed_form(int(bb[e][l * p.stride_b + h * p.rank + k]), dtype) * v
                acc += float(p.topk_weights[t, j]) * u
            want[t, h] = float(np.float32(p.scale)) * acc
    assert (p.lora_ids < 0).any() and (p.perm < 0).any()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)
    rows = [1, 4]
    np.testing.assert_array_equal(O.bgmv_moe_lora_delta(**args, tokens=rows), got[rows])


def test_bgmv_single_route_is_two_library_matmuls():
    """One token, one slot, weight 1, scale 1: B @ (A @ x) through PyTorch's float64 matmul."""
    rng = np.random.default_rng(3)
    I, H, r = 64, 48, 16
    A = rng.standard_normal((r, I)); B = rng.standard_normal((H, r)); x = rng.standard_normal(I)
    to_bits = lambda v: _bits_of(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16))
    Ab, Bb, xb = to_bits(A), to_bits(B), to_bits(x)
    dec = lambda b: torch.tensor(b.astype(np.int16)).view(torch.bfloat16).double()
    want = (dec(Bb).reshape(H, r) @ (dec(Ab).reshape(r, I) @ dec(xb))).numpy()
    got = O.bgmv_moe_lora_delta(xb.reshape(1, I), [0], [Ab.reshape(-1)], r * I, [Bb.reshape(-1)], H * r,
                                [[0]], [[1.0]], [0], r, H, 1.0)
    np.testing.assert_allclose(got[0], want, rtol=1e-13, atol=1e-13)


def test_bgmv_one_hot_fixes_adapter_expert_and_orientation():
    """A single 1 at A[l*, e*][k0, i0] and B[l*, e*][h0, k0]: only out[t, h0] = scale * w * act[p, i0]
    is non-zero, so a transposed A or B, a wrong adapter or expert offset, or a wrong activation
    row moves or loses it."""
    I, H, r, E, L = 32, 24, 8, 3, 4
    l0, e0, k0, i0, h0 = 2, 1, 5, 17, 19
    a_banks = [np.zeros(L * r * I, dtype=np.uint16) for _ in range(E)]
    b_banks = [np.zeros(L * H * r, dtype=np.uint16) for _ in range(E)]
    one = 0x3F80                                       # bf16 1.0
    a_banks[e0][l0 * r * I + k0 * I + i0] = one
    b_banks[e0][l0 * H * r + h0 * r + k0] = one
    act = np.zeros((4, I), dtype=np.uint16)
    act[3, i0] = 0x4040                                # 3.0
    act[2, i0] = 0x4100                                # 8.0 (a row no slot of token 1 uses)
    got = O.bgmv_moe_lora_delta(act, [2, 0, 3, 1], a_banks, r * I, b_banks, H * r,
                                [[0, 2], [1, 0]], [[0.5, 0.5], [0.25, 0.75]], [l0, l0], r, H, 2.0)
    want = np.zeros((2, H))
    want[1, h0] = 2.0 * 0.25 * 3.0
    np.testing.assert_array_equal(got, want)


def test_bgmv_invariants_slot_order_inactive_slots_and_no_adapter():
    import workloads as W
    p = W.make_bgmv_problem(8, 3, 5, 2, 32, 16, 8, seed=5, p_no_lora=0.25, p_inactive=0.0, seg_align=8)
    args = _bgmv_args(p, "bf16")
    base = O.bgmv_moe_lora_delta(**args)
    # the slots of a token may come in any order
    order = [2, 0, 1]
    args2 = dict(args, topk_ids=p.topk_ids.numpy()[:, order], topk_weights=p.topk_weights.numpy()[:, order],
                 perm=p.perm.numpy().reshape(p.T, 3)[:, order].reshape(-1))
    np.testing.assert_allclose(O.bgmv_moe_lora_delta(**args2), base, rtol=1e-12, atol=1e-15)
    # an inactive slot equals a problem without that slot
    perm3 = p.perm.numpy().copy().reshape(p.T, 3)
    perm3[:, 2] = -1
    args3 = dict(args, perm=perm3.reshape(-1))
    args4 = dict(args, topk_ids=p.topk_ids.numpy()[:, :2], topk_weights=p.topk_weights.numpy()[:, :2],
                 perm=p.perm.numpy().reshape(p.T, 3)[:, :2].reshape(-1))
    np.testing.assert_allclose(O.bgmv_moe_lora_delta(**args3), O.bgmv_moe_lora_delta(**args4), rtol=1e-12)
    # no adapter: zero row; linear in scale
    assert np.all(base[p.lora_ids.numpy() < 0] == 0) and (p.lora_ids < 0).any()
    np.testing.assert_allclose(O.bgmv_moe_lora_delta(**dict(args, scale=2 * p.scale)), 2 * base, rtol=1e-15)


def test_f16_rounding_against_numpy_and_hand_cases():
    rng = np.random.default_rng(2)
    y = np.concatenate([rng.standard_normal(20000) * np.exp2(rng.integers(-30, 17, 20000)),
                        [1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -25, 3 * 2.0 ** -26, 65519.99, 65520.0,
                         -65520.0, 2.0 ** -24 * 0.5, 0.0, -0.0]])
    got = O.f64_to_f16_rne(y)
    with np.errstate(over="ignore"):
        want = y.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(got, want)
    assert got[-10] == 0x3C00 and got[-9] == 0x3C02          # ties to even at 1
    assert got[-6] == 0x7BFF and got[-5] == 0x7C00 and got[-4] == 0xFC00
    assert got[-3] == 0x0000 and got[-1] == 0x8000             # half the smallest subnormal -> 0


def test_bgmv_generator_routing_layout():
    """The LoRA-delta input generator lays the routed slots out as the recipe states: each token's
    experts distinct, weights positive and summing to 1, every active slot's row inside its expert's
    segment, segments ordered by expert and padded to the alignment, stride padding NaN."""
    import workloads as W
    p = W.make_bgmv_problem(40, 4, 6, 3, 64, 32, 8, seed=13, stride_pad=8, seg_align=16, p_inactive=0.1)
    ids = p.topk_ids.numpy()
    assert all(len(set(row)) == p.top_k for row in ids)
    w = p.topk_weights.numpy()
    assert np.all(w > 0) and np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    perm = p.perm.numpy().reshape(p.T, p.top_k)
    rows_of = {e: [] for e in range(p.num_experts)}
    for t in range(p.T):
        for j in range(p.top_k):
            if perm[t, j] >= 0:
                rows_of[int(ids[t, j])].append(int(perm[t, j]))
    used = [r for e in rows_of for r in rows_of[e]]
    assert len(used) == len(set(used)), "two slots share an activation row"
    start = 0
    for e in range(p.num_experts):
        n = int((ids == e).sum())
        seg = -(-n // 16) * 16
        assert all(start <= r < start + seg for r in rows_of[e])
        start += seg
    assert p.act.shape[0] >= start
    bank = p.a_banks[0].float().numpy().reshape(p.num_adapters, p.stride_a)
    assert np.all(np.isnan(bank[:, p.rank * p.I:])) and not np.any(np.isnan(bank[:, :p.rank * p.I]))
