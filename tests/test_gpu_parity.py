"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element.

Floating-point outputs: |gpu - y| <= 2^-7*|y| + 2^-10*max|y| and SQNR >= 50 dB, with y the
oracle's float64 value.  Bitwise: the fold (eager and in-place), the zero adapter against
adapter-off, and the exact regime (unit scales, short K, power-of-two alpha).
"""

import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_block_scaled_mm_b200 as L
from workloads import CONFIGS, make_problem, config_problem
from gpu_util import Dev, bits, check_close, host_arrays, to_f64

pytestmark = pytest.mark.gpu


def run_raw(x: Dev, lora_scale=None, bias=True, out=None):
    out = x.new_out() if out is None else out
    L.nvfp4lora_mm(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, x.lora_b, lora_scale, x.r,
                   x.bias if bias else None, out, x.M, x.N, x.K)
    return out


def run_off(x: Dev, bias=True, out=None):
    out = x.new_out() if out is None else out
    L.nvfp4lora_mm(x.a, x.b, x.a_sf, x.b_sf, x.alpha, None, None, None, 0,
                   x.bias if bias else None, out, x.M, x.N, x.K)
    return out


def prepare(x: Dev, lora_b=None, lora_scale=None):
    lb = x.lora_b if lora_b is None else lora_b
    s = x.lora_scale if lora_scale is None else lora_scale
    return L.prepare_nvfp4_lora_adapter(lb, s, x.alpha)


def run_prepared(x: Dev, adp, bias=True, out=None):
    return L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp,
                           bias=x.bias if bias else None, out=out)


def oracle_raw(p, h, s, bias=True):
    return O.mm_raw(h["a"], h["b"], h["a_sf"], h["b_sf"], p.alpha, h["d"], h["lb"], s,
                    h["bias"] if bias else None, p.M, p.N, p.K, p.r)


def finish():
    L.nvfp4lora_device_status()


# ---------------------------------------------------------------------------------------
# fold
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("s,alpha", [(0.25, 2.0 ** -10), (2.0, 2.0 ** -9), (1.7, -0.013), (0.0, 0.5),
                                     (3.999, 1e-30), (7.0, 1e-38), (1.0, 0.0), (0.0, 0.0)])
def test_fold_bitwise_all_bf16_patterns(s, alpha):
    """Eager fold (finite ratio) and in-place refold (any ratio) are bitwise the oracle's fold
    over all 65536 bf16 patterns; a non-finite ratio is refused by the eager form only."""
    lb_bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    lb = torch.from_numpy(lb_bits.view(np.int16).copy()).view(torch.bfloat16).reshape(512, 128).cuda()
    st = torch.tensor([s], dtype=torch.float32, device="cuda")
    at = torch.tensor([alpha], dtype=torch.float32, device="cuda")
    ratio, want = O.fold(lb_bits, s, alpha)
    if np.isfinite(ratio):
        adp = L.prepare_nvfp4_lora_adapter(lb, st, at)
        finish()
        assert adp.ratio.cpu().numpy()[0].view(np.uint32) == np.float32(ratio).view(np.uint32)
        np.testing.assert_array_equal(bits(adp.b_folded).ravel(), want)
    else:
        with pytest.raises(ValueError):
            L.prepare_nvfp4_lora_adapter(lb, st, at)
        adp = L.prepare_nvfp4_lora_adapter(lb, torch.tensor([1.0], device="cuda"), at if alpha != 0 else
                                           torch.tensor([1.0], device="cuda"))
        at = adp.alpha
        at.fill_(alpha)
    # in-place refold into the same adapter is bitwise the eager form
    adp.b_folded.fill_(1.0)
    adp.ratio.fill_(-5.0)
    L.prepare_nvfp4_lora_adapter(lb, st, at, out=adp)
    finish()
    np.testing.assert_array_equal(bits(adp.b_folded).ravel(), want)
    got = adp.ratio.cpu().numpy()[0]
    assert got.view(np.uint32) == np.float32(ratio).view(np.uint32) or (np.isnan(got) and np.isnan(ratio))


def test_eager_prepare_refuses_alpha_zero_and_nonfinite_ratio():
    lb = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        L.prepare_nvfp4_lora_adapter(lb, torch.tensor([1.0], device="cuda"), torch.tensor([0.0], device="cuda"))
    with pytest.raises(ValueError):
        L.prepare_nvfp4_lora_adapter(lb, torch.tensor([3e38], device="cuda"), torch.tensor([1e-10], device="cuda"))


# ---------------------------------------------------------------------------------------
# layout pins on the GPU: one-hot codes and scales
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("k_idx", [0, 1, 15, 16, 63, 64, 200, 255, 256, 511, 767])
def test_one_hot_code_and_scale_position(k_idx):
    M, N, K = 150, 260, 768
    m0, n0 = 141, 259
    a = torch.zeros(M, K // 2, dtype=torch.uint8)
    b = torch.zeros(N, K // 2, dtype=torch.uint8)
    a[m0, k_idx // 2] = (0x5 << 4) if k_idx % 2 else 0x5      # 3.0
    b[n0, k_idx // 2] = (0xB << 4) if k_idx % 2 else 0xB      # -1.5
    a_sf_l = np.full((M, K // 16), 0x38, dtype=np.uint8)
    b_sf_l = np.full((N, K // 16), 0x38, dtype=np.uint8)
    a_sf_l[m0, k_idx // 16] = 0x40                            # 2.0
    b_sf_l[n0, k_idx // 16] = 0x29                            # 0.28125
    a_sf = torch.from_numpy(O.swizzle_scales(a_sf_l, K))
    b_sf = torch.from_numpy(O.swizzle_scales(b_sf_l, K))
    alpha = torch.tensor([1.0], device="cuda")
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    L.nvfp4lora_mm(a.cuda(), b.cuda(), a_sf.cuda(), b_sf.cuda(), alpha, None, None, None, 0, None, out, M, N, K)
    finish()
    got = to_f64(out)
    want = np.zeros((M, N)); want[m0, n0] = 3.0 * -1.5 * 2.0 * 0.28125
    np.testing.assert_array_equal(got, want)


def test_every_scale_position_distinct():
    """Each A row gets one code per 16-block and a distinct scale per block; B is all-ones
    with unit scales, so out[m, n] = sum_blk code * sa[m, blk] identifies misplaced scales."""
    M, N, K = 256, 16, 1024
    rng = np.random.default_rng(99)
    a = np.zeros((M, K // 2), dtype=np.uint8)
    a[:, ::8] = 0x02                                   # element 16*blk = 1.0, others 0
    b = np.full((N, K // 2), 0x22, dtype=np.uint8)     # all 1.0
    sa = rng.integers(0x28, 0x49, size=(M, K // 16), dtype=np.uint8)
    sb = np.full((N, K // 16), 0x38, dtype=np.uint8)
    a_sf = O.swizzle_scales(sa, K)
    b_sf = O.swizzle_scales(sb, K)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    alpha = torch.tensor([1.0], device="cuda")
    L.nvfp4lora_mm(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), torch.from_numpy(a_sf).cuda(),
                   torch.from_numpy(b_sf).cuda(), alpha, None, None, None, 0, None, out, M, N, K)
    finish()
    y = O.mm_off(a, b, a_sf, b_sf, 1.0, None, M, N, K)
    np.testing.assert_array_equal(to_f64(out), O.bf16_bits_to_f64(O.round_output(y)))


# ---------------------------------------------------------------------------------------
# exact regime: bitwise against the oracle's rounded value
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (300, 200, 1024), (7, 1000, 512)])
def test_exact_regime_bitwise(M, N, K):
    g = torch.Generator().manual_seed(M * 7 + N)
    a = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8)
    b = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    a_sf = torch.full((O.sf_buffer_bytes(M, K),), 0x38, dtype=torch.uint8)
    b_sf = torch.full((O.sf_buffer_bytes(N, K),), 0x38, dtype=torch.uint8)
    alpha = 2.0 ** -4
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    L.nvfp4lora_mm(a.cuda(), b.cuda(), a_sf.cuda(), b_sf.cuda(), torch.tensor([alpha], device="cuda"),
                   None, None, None, 0, None, out, M, N, K)
    finish()
    y = O.mm_off(a.numpy(), b.numpy(), a_sf.numpy(), b_sf.numpy(), alpha, None, M, N, K)
    np.testing.assert_array_equal(bits(out), O.round_output(y))


# ---------------------------------------------------------------------------------------
# tolerance parity over shapes with several tiles and ragged tails
# ---------------------------------------------------------------------------------------

# M <= 32 runs the decode kernel (split-K cluster sizes 1, 2, 4, 8 below); 33..127 the single-SM
# tiled kernel; larger M (where the wave count allows) the SM-pair kernel
SHAPES = [(1, 8, 256, 8), (16, 4096, 256, 64), (200, 300, 512, 16), (130, 1000, 768, 72),
          (257, 129, 1024, 128), (384, 384, 2048, 32), (128, 256, 256, 16), (5, 100, 256, 24),
          (3, 256, 2048, 16), (32, 1000, 1024, 128), (20, 9000, 512, 8), (16, 4096, 4096, 64),
          (33, 520, 512, 40), (600, 520, 512, 24), (513, 256, 256, 8), (64, 300, 512, 16),
          (100, 1000, 768, 72), (127, 520, 1024, 8), (200, 600, 512, 8), (256, 1000, 768, 24),
          (256, 520, 512, 40),
          # a single output column and three (outputs of 2 and 6 bytes per row: the plain-store path)
          (1, 1, 256, 8), (40, 3, 512, 8), (130, 1, 256, 16)]


@pytest.mark.parametrize("M,N,K,r", SHAPES)
@pytest.mark.parametrize("bias", [False, True])
def test_raw_parity(M, N, K, r, bias):
    p = make_problem(M, N, K, r, seed=M + N + K + r, alpha=2.0 ** -6, lora_scale=1.25, bias=bias)
    x = Dev(p)
    out = run_raw(x, x.lora_scale, bias)
    finish()
    check_close(out, oracle_raw(p, host_arrays(p), p.lora_scale, bias), what=f"raw {M}x{N}x{K} r{r}")


@pytest.mark.parametrize("M,N,K,r", SHAPES)
def test_prepared_parity(M, N, K, r):
    p = make_problem(M, N, K, r, seed=3 * M + N + r, alpha=0.0137, lora_scale=0.61, bias=True)
    x = Dev(p)
    adp = prepare(x)
    out = run_prepared(x, adp)
    finish()
    h = host_arrays(p)
    ratio, bf = O.fold(h["lb"], p.lora_scale, p.alpha)
    np.testing.assert_array_equal(bits(adp.b_folded).ravel(), bf.ravel())
    y = O.mm_prepared(h["a"], h["b"], h["a_sf"], h["b_sf"], p.alpha, h["d"], bf, ratio, h["bias"],
                      M, N, K, r)
    check_close(out, y, what=f"prepared {M}x{N}x{K} r{r}")


@pytest.mark.parametrize("M,N,K", [(1, 8, 256), (200, 300, 512), (257, 129, 1024)])
def test_off_parity(M, N, K):
    p = make_problem(M, N, K, 8, seed=M * N + K, alpha=0.5, lora_scale=None, bias=True)
    x = Dev(p)
    out = run_off(x)
    finish()
    h = host_arrays(p)
    check_close(out, O.mm_off(h["a"], h["b"], h["a_sf"], h["b_sf"], p.alpha, h["bias"], M, N, K), what="off")


# ---------------------------------------------------------------------------------------
# the whole finite UE4M3 range (subnormal scales 0x01..0x07 up to 448 = 0x7E) on every kernel and
# every path (flashinfer.gemm.mm_nvfp4_lora: the paragraph after the formula and Parameters: a_sf,
# b_sf -- UE4M3 block scales of 16 along K)
# ---------------------------------------------------------------------------------------

# (kernel the shape dispatches to, M, N, K, r): M <= 16 decode with 16 token columns, 17..32 decode
# with 32, 33..127 the single-SM tiled kernel, 256 rows here the SM-pair kernel (r >= 32 keeps the
# raw path on it); N = 520 leaves a ragged last tile on each
RANGE_SHAPES = [("decode16", 16, 520, 1024, 40), ("decode32", 20, 520, 512, 40),
                ("single_sm", 64, 520, 1024, 40), ("sm_pair", 256, 520, 1024, 40)]
SCALE_RANGES = [("full", (0x01, 0x7E), (0x01, 0x7E)),
                ("a_subnormal", (0x01, 0x07), (0x01, 0x7E)),
                ("a_large_b_subnormal", (0x70, 0x7E), (0x01, 0x07))]


@pytest.mark.parametrize("kernel,M,N,K,r", RANGE_SHAPES)
@pytest.mark.parametrize("name,ra,rb", SCALE_RANGES)
def test_full_ue4m3_scale_range_every_kernel_and_path(kernel, M, N, K, r, name, ra, rb):
    """Scale bytes drawn over whole UE4M3 sub-ranges; alpha is the power of two that brings the
    base product to unit RMS, so the LoRA term stays comparable and both are checked."""
    p = make_problem(M, N, K, r, seed=M * 31 + K + ra[0], alpha=1.0, lora_scale=1.25, bias=True,
                     a_sf_range=ra, b_sf_range=rb)
    h = host_arrays(p)
    base = O.base_product(h["a"], h["b"], h["a_sf"], h["b_sf"], M, N, K)
    alpha = float(2.0 ** -np.round(np.log2(np.sqrt(np.mean(base ** 2)))))
    x = Dev(p)
    x.alpha.fill_(alpha)
    off = run_off(x)
    raw = run_raw(x, x.lora_scale)
    adp = prepare(x)
    prep = run_prepared(x, adp)
    finish()
    ratio, bf = O.fold(h["lb"], p.lora_scale, alpha)
    what = f"{kernel} {name}"
    check_close(off, O.mm_off(h["a"], h["b"], h["a_sf"], h["b_sf"], alpha, h["bias"], M, N, K, base=base),
                what=what + " off")
    check_close(raw, O.mm_raw(h["a"], h["b"], h["a_sf"], h["b_sf"], alpha, h["d"], h["lb"], p.lora_scale,
                              h["bias"], M, N, K, r, base=base), what=what + " raw")
    check_close(prep, O.mm_prepared(h["a"], h["b"], h["a_sf"], h["b_sf"], alpha, h["d"], bf, ratio, h["bias"],
                                    M, N, K, r, base=base), what=what + " prepared")


def test_lora_isolation_alpha_zero():
    """alpha = 0 (the LoRA-only raw call) leaves bf16(s * d @ lora_b^T + bias)."""
    p = make_problem(200, 300, 512, 40, seed=5, alpha=0.0, lora_scale=3.0, bias=True)
    x = Dev(p)
    out = run_raw(x, x.lora_scale)
    finish()
    check_close(out, oracle_raw(p, host_arrays(p), 3.0), what="lora only")


def test_prepared_zero_codes_isolates_folded_term():
    p = make_problem(130, 260, 512, 64, seed=6, alpha=0.25, lora_scale=0.8, bias=False)
    p.a.zero_()
    x = Dev(p)
    adp = prepare(x)
    out = run_prepared(x, adp, bias=False)
    finish()
    h = host_arrays(p)
    ratio, bf = O.fold(h["lb"], 0.8, 0.25)
    y = O.mm_prepared(h["a"], h["b"], h["a_sf"], h["b_sf"], 0.25, h["d"], bf, ratio, None, p.M, p.N, p.K, p.r)
    check_close(out, y, what="prepared folded term only")


# ---------------------------------------------------------------------------------------
# zero adapter: bitwise equal to adapter-off
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K,r", [(200, 300, 512, 16), (16, 4096, 1024, 64)])
def test_zero_adapter_bitwise(M, N, K, r):
    p = make_problem(M, N, K, r, seed=77, alpha=2.0 ** -9, lora_scale=2.0, bias=True)
    x = Dev(p)
    x.d[0, 0] = float("inf")
    x.d[min(1, M - 1), 1] = float("nan")
    off = run_off(x)
    for s in (0.0, -0.0):
        out = run_raw(x, torch.tensor([s], device="cuda"))
        finish()
        assert torch.equal(out.view(torch.int16), off.view(torch.int16)), f"s={s}"
    adp = L.prepare_nvfp4_lora_adapter(x.lora_b, torch.tensor([0.0], device="cuda"), x.alpha)
    out = run_prepared(x, adp)
    finish()
    assert torch.equal(out.view(torch.int16), off.view(torch.int16))


# ---------------------------------------------------------------------------------------
# padding rows of the scale buffers never reach rows < M or columns < N
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N", [(16, 200), (20, 136), (70, 200), (200, 300)],
                         ids=["decode16", "decode32", "single_sm", "sm_pair"])
def test_nan_poisoned_scale_padding(M, N):
    K, r = 512, 16
    p = make_problem(M, N, K, r, seed=8, alpha=2.0 ** -6, lora_scale=1.0, bias=True)
    for buf, rows in ((p.a_sf, M), (p.b_sf, N)):
        rp = -(-rows // 128) * 128
        rr, cc = np.meshgrid(np.arange(rows, rp), np.arange(K // 16), indexing="ij")
        buf.numpy()[O.sf_offset(rr, cc, K).ravel()] = 0x7F
    x = Dev(p)
    out = run_raw(x, x.lora_scale)
    finish()
    assert torch.isfinite(out.float()).all()
    check_close(out, oracle_raw(p, host_arrays(p), 1.0), what="poisoned padding")


def test_output_guard_bytes_untouched():
    p = make_problem(130, 70, 256, 8, seed=9, alpha=2.0 ** -6, lora_scale=1.0, bias=False)
    x = Dev(p)
    total = p.M * p.N
    buf = torch.full((total + 2 * 64,), 12345, dtype=torch.int16, device="cuda")
    out = buf[64:64 + total].view(torch.bfloat16).view(p.M, p.N)
    run_raw(x, x.lora_scale, bias=False, out=out)
    finish()
    assert (buf[:64] == 12345).all() and (buf[64 + total:] == 12345).all()
    check_close(out, oracle_raw(p, host_arrays(p), 1.0, bias=False), what="guarded")


def test_repeat_runs_bitwise_deterministic():
    p = make_problem(384, 384, 2048, 32, seed=10, alpha=2.0 ** -6, lora_scale=1.0, bias=True)
    x = Dev(p)
    o1 = run_raw(x, x.lora_scale)
    o2 = run_raw(x, x.lora_scale)
    finish()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


# ---------------------------------------------------------------------------------------
# the stated workloads
# ---------------------------------------------------------------------------------------

def test_cfg0_full():
    p = config_problem("cfg0")
    x = Dev(p)
    out = run_raw(x, x.lora_scale, bias=False)
    finish()
    check_close(out, oracle_raw(p, host_arrays(p), p.lora_scale, bias=False), what="cfg0")


def test_cfg1_decode_full():
    p = config_problem("cfg1")
    x = Dev(p)
    out = run_raw(x, x.lora_scale)
    finish()
    check_close(out, oracle_raw(p, host_arrays(p), p.lora_scale), what="cfg1")


def test_cfg2_prefill_full_and_zero_adapter():
    p = config_problem("cfg2")
    x = Dev(p)
    out = run_raw(x, x.lora_scale)
    off = run_off(x)
    zero = run_raw(x, torch.tensor([0.0], device="cuda"))
    finish()
    assert torch.equal(zero.view(torch.int16), off.view(torch.int16))
    h = host_arrays(p)
    base = O.base_product(h["a"], h["b"], h["a_sf"], h["b_sf"], p.M, p.N, p.K)
    y = O.mm_raw(h["a"], h["b"], h["a_sf"], h["b_sf"], p.alpha, h["d"], h["lb"], p.lora_scale, h["bias"],
                 p.M, p.N, p.K, p.r, base=base)
    check_close(out, y, what="cfg2")


@pytest.mark.slow
def test_cfg3_sampled_prepared_and_raw():
    """Full-size launch; the oracle checks 48 random rows x 512 random columns plus the four
    corner 128 x 128 tiles."""
    c = CONFIGS["cfg3"]
    p = config_problem("cfg3")
    x = Dev(p)
    adp = prepare(x)
    out = run_prepared(x, adp)
    out_raw = run_raw(x, x.lora_scale)
    finish()
    h = host_arrays(p)
    ratio, bf = O.fold(h["lb"], p.lora_scale, p.alpha)
    np.testing.assert_array_equal(bits(adp.b_folded).ravel(), bf.ravel())
    rng = np.random.default_rng(33)
    rows = np.unique(np.concatenate([rng.choice(p.M, 48, replace=False), np.arange(128),
                                     np.arange(p.M - 128, p.M)]))
    cols = np.unique(np.concatenate([rng.choice(p.N, 512, replace=False), np.arange(128),
                                     np.arange(p.N - 128, p.N)]))
    base = O.base_product_rows_cols(h["a"], h["b"], h["a_sf"], h["b_sf"], p.K, rows, cols)
    y_prep = O.mm_prepared(h["a"], h["b"], h["a_sf"], h["b_sf"], c["alpha"], h["d"], bf, ratio, None,
                           p.M, p.N, p.K, p.r, base=base, rows=rows, cols=cols)
    y_raw = O.mm_raw(h["a"], h["b"], h["a_sf"], h["b_sf"], c["alpha"], h["d"], h["lb"], c["lora_scale"], None,
                     p.M, p.N, p.K, p.r, base=base, rows=rows, cols=cols)
    ri = torch.from_numpy(rows).cuda()
    ci = torch.from_numpy(cols).cuda()
    check_close(out[ri][:, ci], y_prep, what="cfg3 prepared")
    check_close(out_raw[ri][:, ci], y_raw, what="cfg3 raw")


@pytest.mark.parametrize("M", [1, 32, 256, 2048])
@pytest.mark.parametrize("r", [8, 128])
def test_cfg4_adapter_switch_shapes(M, r):
    from workloads import CFG4, make_adapters
    N, K = CFG4["N"], CFG4["K"]
    p = make_problem(M, N, K, r, seed=CFG4["seed"] * 1000 + M + r, alpha=CFG4["alpha"], lora_scale=1.0, bias=False)
    x = Dev(p)
    adapters = make_adapters(N, r, 2, seed=100 * M + r)
    rng = np.random.default_rng(M + r)
    cols = np.unique(np.concatenate([rng.choice(N, 256, replace=False), np.arange(N - 64, N)]))
    rows = np.arange(M) if M <= 256 else np.unique(np.concatenate([rng.choice(M, 64, replace=False), [0, M - 1]]))
    h = host_arrays(p)
    base = O.base_product_rows_cols(h["a"], h["b"], h["a_sf"], h["b_sf"], K, rows, cols)
    for lb, s in adapters:
        lbd = lb.cuda()
        sd = torch.tensor([s], dtype=torch.float32, device="cuda")
        out = x.new_out()
        L.nvfp4lora_mm(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lbd, sd, r, None, out, M, N, K)
        adp = L.prepare_nvfp4_lora_adapter(lbd, sd, x.alpha)
        outp = run_prepared(x, adp, bias=False)
        finish()
        y = O.mm_raw(h["a"], h["b"], h["a_sf"], h["b_sf"], CFG4["alpha"], h["d"], bits(lb), s, None,
                     M, N, K, r, base=base, rows=rows, cols=cols)
        ratio, bf = O.fold(bits(lb), s, CFG4["alpha"])
        yp = O.mm_prepared(h["a"], h["b"], h["a_sf"], h["b_sf"], CFG4["alpha"], h["d"], bf, ratio, None,
                           M, N, K, r, base=base, rows=rows, cols=cols)
        ri = torch.from_numpy(rows).cuda()
        ci = torch.from_numpy(cols).cuda()
        check_close(out[ri][:, ci], y, what=f"cfg4 raw M{M} r{r}")
        check_close(outp[ri][:, ci], yp, what=f"cfg4 prepared M{M} r{r}")


@pytest.mark.parametrize("M,N", [(200, 512), (16, 512)])
def test_bias_not_16_byte_aligned(M, N):
    """A bias view that starts 2 bytes into its storage takes the element-wise bias path."""
    p = make_problem(M, N, 512, 16, seed=12, alpha=2.0 ** -6, lora_scale=1.0, bias=True)
    x = Dev(p)
    store = torch.empty(N + 8, dtype=torch.bfloat16, device="cuda")
    store[1:N + 1] = x.bias
    x.bias = store[1:N + 1]
    out = run_raw(x, x.lora_scale)
    finish()
    check_close(out, oracle_raw(p, host_arrays(p), 1.0), what="unaligned bias")
