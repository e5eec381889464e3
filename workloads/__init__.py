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


@dataclasses.dataclass
class BgmvProblem:
    """One routed-MoE LoRA-delta problem's host tensors (CPU, contiguous)."""
    T: int
    top_k: int
    num_experts: int
    num_adapters: int
    I: int
    H: int
    rank: int
    lora_dtype: torch.dtype
    scale: float
    act: torch.Tensor            # lora_dtype [padded_rows, I], permuted rows
    perm: torch.Tensor           # int32 [T * top_k]: expanded index -> permuted row, -1 inactive
    a_banks: list                # per expert: lora_dtype [num_adapters * stride_a]
    stride_a: int
    b_banks: list                # per expert: lora_dtype [num_adapters * stride_b]
    stride_b: int
    topk_ids: torch.Tensor       # int32 [T, top_k], distinct experts per token
    topk_weights: torch.Tensor   # fp32 [T, top_k], positive, summing to 1 per token
    lora_ids: torch.Tensor       # int32 [T], -1 = no adapter


def make_bgmv_problem(T: int, top_k: int, num_experts: int, num_adapters: int, I: int, H: int,
                      rank: int, seed: int, *, lora_dtype=torch.bfloat16, scale: float = 2.0,
                      p_no_lora: float = 0.125, p_inactive: float = 0.0625, stride_pad: int = 0,
                      act_std: float = 0.5, b_std: float = 0.02, seg_align: int = 128) -> BgmvProblem:
    """Draw one problem.  Routing: each token picks top_k distinct experts (a random permutation
    per token) with softmax weights of N(0, 1) logits; the expanded slots are laid out grouped by
    expert, each expert's segment padded to a multiple of `seg_align` rows, as a grouped FC1
    would return them; a fraction `p_inactive` of slots is marked inactive (-1) and a fraction
    `p_no_lora` of tokens gets lora id -1.  A_down ~ U(-1/sqrt(I), 1/sqrt(I)), B_down ~ N(0,
    b_std), activations ~ N(0, act_std).  Each adapter block is followed by `stride_pad` NaN
    elements (so a read outside a block shows).  Draw order: routing, weights, inactive slots,
    lora ids, act, A banks, B banks."""
    g = torch.Generator().manual_seed(seed)
    ids = torch.stack([torch.randperm(num_experts, generator=g)[:top_k] for _ in range(T)]) if T else \
        torch.zeros(0, top_k, dtype=torch.int64)
    logits = torch.randn(T, top_k, generator=g)
    w = torch.softmax(logits, dim=1).to(torch.float32)
    inactive = torch.rand(T * top_k, generator=g) < p_inactive
    no_lora = torch.rand(T, generator=g) < p_no_lora
    lora_ids = torch.randint(0, num_adapters, (T,), generator=g, dtype=torch.int32)
    lora_ids[no_lora] = -1
    # slot layout: grouped by expert (slot order within an expert by expanded index)
    flat = ids.reshape(-1)
    perm = torch.full((T * top_k,), -1, dtype=torch.int32)
    row = 0
    for e in range(num_experts):
        slots = (flat == e).nonzero().reshape(-1)
        for n, x in enumerate(slots.tolist()):
            perm[x] = row + n
        row += -(-slots.numel() // seg_align) * seg_align
    perm[inactive] = -1
    padded_rows = max(row, seg_align)
    act = (torch.randn(padded_rows, I, generator=g) * act_std).to(lora_dtype)
    stride_a = rank * I + stride_pad
    stride_b = H * rank + stride_pad
    bound = 1.0 / (I ** 0.5)
    a_banks, b_banks = [], []
    for _ in range(num_experts):
        bank = torch.full((num_adapters, stride_a), float("nan"))
        bank[:, :rank * I] = torch.empty(num_adapters, rank * I).uniform_(-bound, bound, generator=g)
        a_banks.append(bank.reshape(-1).to(lora_dtype))
    for _ in range(num_experts):
        bank = torch.full((num_adapters, stride_b), float("nan"))
        bank[:, :H * rank] = torch.randn(num_adapters, H * rank, generator=g) * b_std
        b_banks.append(bank.reshape(-1).to(lora_dtype))
    return BgmvProblem(T, top_k, num_experts, num_adapters, I, H, rank, lora_dtype, float(scale), act, perm,
                       a_banks, stride_a, b_banks, stride_b, ids.to(torch.int32), w, lora_ids)


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

#: routed-MoE FC2 LoRA delta: a decode batch of 64 tokens routed top-2 over the layer's 8 experts,
#: I = H = 4096 (the layer's width), rank 16, 4 adapters, scale 2 (an assumed serving mix; the
#: pages give no shapes for it)
BGMV = dict(T=64, top_k=2, num_experts=8, num_adapters=4, I=4096, H=4096, rank=16, scale=2.0, seed=7)

#: adapter-switch sweep: N=14336, K=4096, M x r grid, 8 adapters, alpha 2**-9
CFG4 = dict(N=14336, K=4096, Ms=(1, 32, 256, 2048), rs=(8, 128), adapters=8,
            alpha=2.0 ** -9, seed=4)


def config_problem(name: str, **over) -> Problem:
    c = dict(CONFIGS[name])
    c.update(over)
    return make_problem(c["M"], c["N"], c["K"], c["r"], c["seed"], alpha=c["alpha"],
                        lora_scale=c["lora_scale"], bias=c["bias"])
