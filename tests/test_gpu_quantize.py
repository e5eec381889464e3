"""GPU parity of the NVFP4 quantizer (the fp4_quantize reading) against the CPU oracle.

Codes and scale bytes are integers: bit-exact, the whole buffers (padding included).  The
composition quantize -> GEMM is checked against the oracle GEMM of the oracle's own codes.
"""

import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_block_scaled_mm_b200 as L

pytestmark = pytest.mark.gpu


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _run(x: torch.Tensor, gs: float):
    g = torch.tensor([gs], dtype=torch.float32, device="cuda")
    codes, scales = L.fp4_quantize(x.cuda(), g)
    torch.cuda.synchronize()
    L.nvfp4lora_device_status()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _check(x: torch.Tensor, gs: float):
    codes, scales = _run(x, gs)
    want_codes, want_scales = O.quantize_nvfp4(_bf16_bits(x), gs)
    np.testing.assert_array_equal(scales, want_scales)
    np.testing.assert_array_equal(codes, want_codes)


@pytest.mark.parametrize("rows,k", [(1, 64), (16, 4096), (130, 256), (257, 1024), (600, 512), (128, 64)])
def test_quantize_bitwise_random(rows, k):
    g = torch.Generator().manual_seed(rows * 7 + k)
    x = (torch.randn(rows, k, generator=g) * torch.exp2(torch.randint(-8, 8, (rows, 1), generator=g).float()))
    x = x.to(torch.bfloat16)
    amax = x.float().abs().max().item()
    _check(x, 448.0 * 6.0 / amax)


def test_quantize_ties_signs_zero_blocks_and_saturation():
    """Blocks built to hit E2M1 ties (x * gs / scale on the midpoints), negative values that
    round to zero, all-zero blocks, saturated scales and codes, and tiny scales."""
    rows, k = 8, 256
    x = torch.zeros(rows, k)
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    # row 0: one block per sign with amax 6 (scale 1 at gs = 1): the others sit on ties
    x[0, :16] = torch.cat([mids, -mids])
    x[0, 16:32] = torch.cat([mids, torch.tensor([-0.2, -0.1, 0.1, 0.2, 0.3, -0.3, 4.5, -6.0])])
    x[1, :16] = 1.0e4                       # scale saturates at 448, codes at 6
    x[1, 16] = -3.0e4
    x[2, :] = 0.0                           # zero blocks: scale 0, codes +0
    x[3, :16] = -0.0
    x[4, :] = torch.linspace(-1e-3, 1e-3, k)   # small values: subnormal E4M3 scales
    x[5, :] = torch.linspace(-7, 7, k)
    x[6, 64:80] = 3.0                       # amax 3 -> scale 0.5
    x[7, :] = torch.randn(k) * 100
    _check(x.to(torch.bfloat16), 1.0)


@pytest.mark.parametrize("gs", [1.0, 0.37, 3.0e3])
def test_quantize_global_scale_values(gs):
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(64, 512, generator=g) * 3).to(torch.bfloat16)
    _check(x, gs)


def test_quantize_then_gemm_matches_oracle_composition():
    """fp4_quantize feeds mm_nvfp4_lora: quantize bf16 activations and weights on the GPU, run the
    GEMM with alpha = 1 / (gs_a * gs_b), and compare with the oracle GEMM of the oracle codes."""
    M, N, K = 200, 300, 512
    g = torch.Generator().manual_seed(3)
    xa = torch.randn(M, K, generator=g).to(torch.bfloat16)
    xb = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    gsa = 448.0 * 6.0 / xa.float().abs().max().item()
    gsb = 448.0 * 6.0 / xb.float().abs().max().item()
    a, a_sf = L.fp4_quantize(xa.cuda(), torch.tensor([gsa], dtype=torch.float32, device="cuda"))
    b, b_sf = L.fp4_quantize(xb.cuda(), torch.tensor([gsb], dtype=torch.float32, device="cuda"))
    alpha_v = float(np.float32(1.0 / (np.float32(gsa) * np.float32(gsb))))
    alpha = torch.tensor([alpha_v], dtype=torch.float32, device="cuda")
    out = L.mm_nvfp4_lora(a, b, a_sf, b_sf, alpha)
    torch.cuda.synchronize()
    ha, hsa = O.quantize_nvfp4(_bf16_bits(xa), gsa)
    hb, hsb = O.quantize_nvfp4(_bf16_bits(xb), gsb)
    np.testing.assert_array_equal(a.cpu().numpy(), ha)
    np.testing.assert_array_equal(b_sf.cpu().numpy(), hsb)
    y = O.mm_off(ha, hb, hsa, hsb, alpha_v, None, M, N, K)
    got = O.bf16_bits_to_f64(_bf16_bits(out))
    assert np.all(np.abs(got - y) <= O.tolerance(y))
    # and the quantized GEMM approximates the bf16 GEMM (4-bit operands: a loose bound)
    ref = xa.double() @ xb.double().T
    rel = torch.linalg.norm(torch.from_numpy(got) - ref) / torch.linalg.norm(ref)
    assert rel < 0.2


def test_quantize_full_size_workload_sampled_row_blocks():
    """The benchmarked workload (bf16 [8192, 8192] activations, the A operand of the
    8192 x 28672 x 8192 GEMM, with the quantizer bench's generator and seed) through the same
    launch; the oracle checks the
    first, a middle and the last 128-row block bit for bit (rows are independent, and a 128-row
    block's scale bytes are one contiguous run of the swizzled layout)."""
    rows, k = 8192, 8192
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(rows, k, generator=g) * 2.0).to(torch.bfloat16)
    gs = 448.0 * 6.0 / x.float().abs().max().item()
    codes, scales = _run(x, gs)
    nb = k // 16
    block_bytes = 128 * nb
    for rb in (0, rows // 256, rows // 128 - 1):
        xb = x[rb * 128:(rb + 1) * 128]
        want_codes, want_scales = O.quantize_nvfp4(_bf16_bits(xb), gs)
        np.testing.assert_array_equal(codes[rb * 128:(rb + 1) * 128], want_codes)
        np.testing.assert_array_equal(scales[rb * block_bytes:(rb + 1) * block_bytes], want_scales)
