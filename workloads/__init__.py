"""Seeded synthetic inputs shared by the tests, ``bench.py`` and ``smoke()``.

This module draws random bytes and numbers and nothing else: it holds none of the
operation's arithmetic (no decoding, no swizzle arithmetic, no products), so the CPU
oracle and the CUDA path can both take their inputs from it without sharing code.

Value distributions follow the workloads stated for the operation
(flashinfer.gemm.mm_nvfp4_lora: E2M1 codes uniform over the 16 codes, UE4M3 block
scales uniform over the positive E4M3 values in [0.25, 4], d ~ N(0, 1), lora_b ~
N(0, 0.02), bias ~ N(0, 0.1)), drawn with ``torch.Generator`` on the CPU in a fixed
order: a, b, a_sf, b_sf, d, lora_b, bias.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

#: positive E4M3 bytes 0x28 (0.25) .. 0x48 (4.0): 33 codes, all finite and normal
SF_LO = 0x28
SF_HI = 0x48


def sf_bytes(rows: int, k: int) -> int:
    """Bytes of a scale buffer whose rows are padded to a multiple of 128."""
    return -(-rows // 128) * 128 * (k // 16)


@dataclasses.dataclass
class Problem:
    """One GEMM problem's host tensors (CPU, contiguous)."""
    M: int
    N: int
    K: int
    r: int
    a: torch.Tensor          # uint8 [M, K/2]
    b: torch.Tensor          # uint8 [N, K/2]
    a_sf: torch.Tensor       # uint8 [padded(M) * K/16], swizzled layout, drawn bytewise
    b_sf: torch.Tensor       # uint8 [padded(N) * K/16]
    alpha: float
    lora_scale: Optional[float]
    d: Optional[torch.Tensor]        # bf16 [M, r]
    lora_b: Optional[torch.Tensor]   # bf16 [N, r]
    bias: Optional[torch.Tensor]     # bf16 [N]


def make_problem(M: int, N: int, K: int, r: int, seed: int, *, alpha: float,
                 lora_scale: Optional[float], bias: bool, d_std: float = 1.0,
                 lb_std: float = 0.02, bias_std: float = 0.1,
                 codes: str = "uniform", a_sf_range=(SF_LO, SF_HI),
                 b_sf_range=(SF_LO, SF_HI)) -> Problem:
    """Draw one problem.  Every byte of the padded scale buffers is drawn (padding rows
    included), so no knowledge of the swizzle is needed here.  Scale bytes are uniform over
    the inclusive byte ranges ``a_sf_range`` / ``b_sf_range`` (default: the workloads' 0x28..0x48;
    0x01..0x7E spans every positive finite UE4M3 value, subnormals 0x01..0x07 included)."""
    g = torch.Generator().manual_seed(seed)
    if codes == "uniform":
        a = torch.randint(0, 256, (M, K // 2), generator=g, dtype=torch.uint8)
        b = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.uint8)
    elif codes == "zero":
        a = torch.zeros((M, K // 2), dtype=torch.uint8)
        b = torch.zeros((N, K // 2), dtype=torch.uint8)
    else:
        raise ValueError(codes)
    a_sf = torch.randint(a_sf_range[0], a_sf_range[1] + 1, (sf_bytes(M, K),), generator=g, dtype=torch.uint8)
    b_sf = torch.randint(b_sf_range[0], b_sf_range[1] + 1, (sf_bytes(N, K),), generator=g, dtype=torch.uint8)
    d = (torch.randn(M, r, generator=g) * d_std).to(torch.bfloat16)
    lora_b = (torch.randn(N, r, generator=g) * lb_std).to(torch.bfloat16)
    bias_t = (torch.randn(N, generator=g) * bias_std).to(torch.bfloat16) if bias else None
    return Problem(M, N, K, r, a, b, a_sf, b_sf, alpha, lora_scale, d, lora_b, bias_t)


@dataclasses.dataclass
class GroupedProblem:
    """One grouped (expert-partitioned) problem's host tensors: expert e owns rows
    [m_indptr[e], m_indptr[e+1]) of a, d and out."""
    rows: int
    N: int
    K: int
    r: int
    m_indptr: torch.Tensor   # int32 [E + 1]
    a: torch.Tensor          # uint8 [rows, K/2]
    b: torch.Tensor          # uint8 [E, N, K/2]
    a_sf: torch.Tensor       # uint8, the padded swizzled layout of all rows, drawn bytewise
    b_sf: torch.Tensor       # uint8, E consecutive padded buffers, drawn bytewise
    alpha: torch.Tensor      # fp32 [E]
    d: torch.Tensor          # bf16 [rows, r]
    lora_b: torch.Tensor     # bf16 [E, N, r]
    bias: Optional[torch.Tensor]   # bf16 [E, N]


def make_grouped_problem(segments, N: int, K: int, r: int, seed: int, *, pad_rows: int = 128,
                         bias: bool = True, sf_range=(SF_LO, SF_HI), alpha_range=(2.0 ** -10, 2.0 ** -6),
                         lb_std: float = 0.02, bias_std: float = 0.1) -> GroupedProblem:
    """Draw a grouped problem whose expert e has segments[e] rows (multiples of 128 by the grouped
    reading); `pad_rows` rows past the last segment belong to no expert.  Draw order: a, b, a_sf,
    b_sf, alpha, d, lora_b, bias."""
    g = torch.Generator().manual_seed(seed)
    E = len(segments)
    offs = [0]
    for n in segments:
        offs.append(offs[-1] + int(n))
    rows = offs[-1] + pad_rows
    a = torch.randint(0, 256, (rows, K // 2), generator=g, dtype=torch.uint8)
    b = torch.randint(0, 256, (E, N, K // 2), generator=g, dtype=torch.uint8)
    a_sf = torch.randint(sf_range[0], sf_range[1] + 1, (sf_bytes(rows, K),), generator=g, dtype=torch.uint8)
    b_sf = torch.randint(sf_range[0], sf_range[1] + 1, (E * sf_bytes(N, K),), generator=g, dtype=torch.uint8)
    alpha = torch.empty(E).uniform_(alpha_range[0], alpha_range[1], generator=g).to(torch.float32)
    d = torch.randn(rows, r, generator=g).to(torch.bfloat16)
    lora_b = (torch.randn(E, N, r, generator=g) * lb_std).to(torch.bfloat16)
    bias_t = (torch.randn(E, N, generator=g) * bias_std).to(torch.bfloat16) if bias else None
    return GroupedProblem(rows, N, K, r, torch.tensor(offs, dtype=torch.int32), a, b, a_sf, b_sf, alpha, d,
                          lora_b, bias_t)


def make_adapters(N: int, r: int, count: int, seed: int, lb_std: float = 0.02):
    """``count`` adapters: lora_b ~ N(0, lb_std) bf16 [N, r], lora_scale ~ U[0.1, 4]."""
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(count):
        lb = (torch.randn(N, r, generator=g) * lb_std).to(torch.bfloat16)
        s = float(torch.empty(1).uniform_(0.1, 4.0, generator=g).item())
        out.append((lb, s))
    return out


# --------------------------------------------------------------------------------------
# The workloads (shapes, paths and scalars).  "cfg0" is the small parity case; "cfg1" is
# the decode shape the throughput metric is quoted on at M <= 16; "cfg2"/"cfg3" are the
# prefill and large MLP-up shapes; "cfg4" is the adapter-switch sweep.
# --------------------------------------------------------------------------------------

CONFIGS = {
    "cfg0": dict(M=128, N=256, K=256, r=16, path="raw", alpha=2.0 ** -6, lora_scale=2.0,
                 bias=False, seed=0),
    "cfg1": dict(M=16, N=4096, K=4096, r=64, path="raw", alpha=2.0 ** -9, lora_scale=0.5,
                 bias=True, seed=1),
    "cfg2": dict(M=4096, N=4096, K=4096, r=16, path="raw", alpha=2.0 ** -9, lora_scale=2.0,
                 bias=True, seed=2),
    "cfg3": dict(M=8192, N=28672, K=8192, r=64, path="prepared", alpha=2.0 ** -10,
                 lora_scale=0.25, bias=False, seed=3),
}

#: grouped (expert-partitioned) layer: 8 experts with these row counts (multiples of 128, one
#: empty), per-expert weights N x K, a shared rank-16 adapter scale, raw path with per-expert bias
MOE = dict(segments=(512, 128, 1024, 256, 0, 384, 128, 640), N=4096, K=4096, r=16, lora_scale=0.5, seed=6)

#: adapter-switch sweep: N=14336, K=4096, M x r grid, 8 adapters, alpha 2**-9
CFG4 = dict(N=14336, K=4096, Ms=(1, 32, 256, 2048), rs=(8, 128), adapters=8,
            alpha=2.0 ** -9, seed=4)


def config_problem(name: str, **over) -> Problem:
    c = dict(CONFIGS[name])
    c.update(over)
    return make_problem(c["M"], c["N"], c["K"], c["r"], c["seed"], alpha=c["alpha"],
                        lora_scale=c["lora_scale"], bias=c["bias"])
