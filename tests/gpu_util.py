"""Helpers shared by the GPU parity tests: move a workload problem to the device, run the
CUDA path through the C ABI, and compute the oracle's reference on the same bytes."""

from __future__ import annotations

import numpy as np
import torch

import oracle as O


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return O.bf16_bits_to_f64(bits(t))


class Dev:
    """A problem's tensors on cuda:0."""

    def __init__(self, p, device="cuda:0"):
        self.p = p
        self.M, self.N, self.K, self.r = p.M, p.N, p.K, p.r
        self.a = p.a.to(device)
        self.b = p.b.to(device)
        self.a_sf = p.a_sf.to(device)
        self.b_sf = p.b_sf.to(device)
        self.alpha = torch.tensor([p.alpha], dtype=torch.float32, device=device)
        self.lora_scale = (torch.tensor([p.lora_scale], dtype=torch.float32, device=device)
                           if p.lora_scale is not None else None)
        self.d = p.d.to(device) if p.d is not None else None
        self.lora_b = p.lora_b.to(device) if p.lora_b is not None else None
        self.bias = p.bias.to(device) if p.bias is not None else None

    def new_out(self):
        return torch.empty((self.M, self.N), dtype=torch.bfloat16, device=self.a.device)


def host_arrays(p):
    """The problem's bytes as the oracle wants them."""
    return dict(a=p.a.numpy(), b=p.b.numpy(), a_sf=p.a_sf.numpy(), b_sf=p.b_sf.numpy(),
                d=None if p.d is None else bits(p.d), lb=None if p.lora_b is None else bits(p.lora_b),
                bias=None if p.bias is None else bits(p.bias))


def check_close(gpu_out: torch.Tensor, y: np.ndarray, *, min_sqnr=50.0, what=""):
    """The acceptance bar: |gpu - y| <= 2^-7|y| + 2^-10 max|y| everywhere and SQNR >= 50 dB."""
    g = to_f64(gpu_out).reshape(y.shape)
    tol = O.tolerance(y)
    err = np.abs(g - y)
    bad = ~(err <= tol)
    if np.any(bad):
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside tolerance; first {idx.tolist()}: "
                             f"gpu {g[tuple(idx[0])]} oracle {y[tuple(idx[0])]} tol {tol[tuple(idx[0])]}")
    s = O.sqnr_db(y, g)
    assert s >= min_sqnr, f"{what}: SQNR {s:.2f} dB < {min_sqnr}"
    return s
