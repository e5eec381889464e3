"""GPU parity of the grouped (expert-partitioned) call against the oracle's grouped form.

flashinfer.grouped_mm.grouped_mm_bf16 (formula and Parameters: m_indptr) applied to the NVFP4 +
LoRA operation, with the reading that every m_indptr entry is a multiple of 128.  Tolerance as for
the plain call: |gpu - y| <= 2^-7|y| + 2^-10 max|y| and SQNR >= 50 dB; bitwise: zero adapter
against adapter-off, and rows past m_indptr[E] untouched.
"""

import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_block_scaled_mm_b200 as L
from workloads import make_grouped_problem
from gpu_util import bits, check_close

pytestmark = pytest.mark.gpu

SENTINEL = 0x3F80   # bf16 1.0 (a value the checked rows never take exactly here)


def run(p, lora_scale=None, out=None, lora=True):
    dev = "cuda"
    t = {k: getattr(p, k).to(dev) for k in ("m_indptr", "a", "b", "a_sf", "b_sf", "alpha", "d", "lora_b")}
    bias = p.bias.to(dev) if p.bias is not None else None
    if out is None:
        out = torch.full((p.rows, p.N), 1.0, dtype=torch.bfloat16, device=dev)
    s = None if lora_scale is None else torch.tensor([lora_scale], dtype=torch.float32, device=dev)
    L.grouped_mm_nvfp4_lora(t["a"], t["b"], t["a_sf"], t["b_sf"], t["m_indptr"], t["alpha"],
                            t["d"] if lora else None, t["lora_b"] if lora else None, s, bias=bias, out=out)
    return out


def oracle(p, lora_scale):
    return O.grouped_mm(p.a.numpy(), p.b.numpy(), p.a_sf.numpy(), p.b_sf.numpy(), p.m_indptr.numpy(),
                        p.alpha.numpy().astype(np.float64), bits(p.d), bits(p.lora_b), lora_scale,
                        None if p.bias is None else bits(p.bias), p.rows, p.N, p.K, p.r)


@pytest.mark.parametrize("segments,N,K,r,sf", [
    ([256, 0, 128, 384], 520, 1024, 40, (0x28, 0x48)),
    ([128, 128, 0, 0, 512], 264, 512, 16, (0x01, 0x7E)),
    ([0, 384], 300, 768, 72, (0x01, 0x7E)),
    ([128], 256, 256, 8, (0x28, 0x48)),
])
def test_grouped_raw_and_off_parity(segments, N, K, r, sf):
    p = make_grouped_problem(segments, N, K, r, seed=sum(segments) + N + K, sf_range=sf)
    used = int(p.m_indptr[-1])
    for s in (1.5, None):
        out = run(p, s)
        L.nvfp4lora_device_status()
        y = oracle(p, s)
        check_close(out[:used], y, what=f"grouped {segments} s={s}")
        assert torch.all(out[used:].view(torch.int16) == SENTINEL), "rows past m_indptr[E] were written"


def test_grouped_zero_adapter_is_bitwise_adapter_off():
    p = make_grouped_problem([256, 128, 0, 256], 520, 1024, 24, seed=41)
    p.d[3, 5] = float("inf")
    off = run(p, None, lora=False)
    zero = run(p, 0.0)
    L.nvfp4lora_device_status()
    assert torch.equal(zero.view(torch.int16), off.view(torch.int16))


def test_grouped_rejects_a_misaligned_table_on_the_device():
    p = make_grouped_problem([256, 128], 256, 256, 16, seed=42)
    p.m_indptr[1] = 200                 # not a multiple of 128
    out = run(p, 1.0)
    with pytest.raises(ValueError, match="m_indptr"):
        L.nvfp4lora_device_status()
    assert torch.all(out.view(torch.int16) == SENTINEL), "a rejected table computed something"
    # the context stays usable: the next valid call is correct
    q = make_grouped_problem([128, 128], 256, 256, 16, seed=43)
    good = run(q, 1.0)
    L.nvfp4lora_device_status()
    check_close(good[:256], oracle(q, 1.0), what="after a rejected table")


def test_grouped_moe_shape_sampled():
    """An MoE-like layer: 8 experts with 128..1024 rows each (padded), N = 2048, K = 4096, r = 16;
    the oracle checks every row of two experts and sampled rows of the rest."""
    segs = [512, 128, 1024, 256, 0, 384, 128, 640]
    p = make_grouped_problem(segs, 2048, 4096, 16, seed=44)
    out = run(p, 0.5)
    L.nvfp4lora_device_status()
    ind = p.m_indptr.numpy()
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([np.arange(ind[0], ind[1]), np.arange(ind[2], ind[3]),
                                     rng.choice(int(ind[-1]), 96, replace=False)]))
    y = oracle(p, 0.5)
    check_close(out[torch.from_numpy(rows).cuda()], y[rows], what="moe sampled rows")


def test_grouped_graph_replay_with_new_routing():
    """m_indptr is read on the device only, so one captured grouped call serves a new expert split
    copied into its captured table (same total row count here, different segments)."""
    dev = "cuda"
    p1 = make_grouped_problem([256, 128, 0, 128], 264, 512, 16, seed=51, pad_rows=128)
    p2 = make_grouped_problem([128, 0, 384, 0], 264, 512, 16, seed=51, pad_rows=128)
    assert p1.rows == p2.rows
    t = {k: getattr(p1, k).to(dev) for k in ("m_indptr", "a", "b", "a_sf", "b_sf", "alpha", "d", "lora_b")}
    bias = p1.bias.to(dev)
    s = torch.tensor([1.25], dtype=torch.float32, device=dev)
    out = torch.full((p1.rows, p1.N), 1.0, dtype=torch.bfloat16, device=dev)

    def call():
        L.grouped_mm_nvfp4_lora(t["a"], t["b"], t["a_sf"], t["b_sf"], t["m_indptr"], t["alpha"], t["d"],
                                t["lora_b"], s, bias=bias, out=out)

    call()                                   # warm-up outside the capture
    L.nvfp4lora_device_status()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    # the same operands (drawn with the same seed), a different split of the rows among the experts
    t["m_indptr"].copy_(p2.m_indptr.to(dev))
    out.fill_(1.0)
    graph.replay()
    L.nvfp4lora_device_status()
    used = int(p2.m_indptr[-1])
    check_close(out[:used], oracle(p2, 1.25), what="grouped graph replay")
    assert torch.all(out[used:].view(torch.int16) == SENTINEL)


def test_grouped_maximum_expert_count():
    """511 experts (the limit), most of them empty: the device-side table copy and the binary search
    over all 512 entries, with non-empty experts at both ends and in the middle."""
    segments = [0] * 511
    for e in (0, 255, 510):
        segments[e] = 128
    p = make_grouped_problem(segments, 136, 256, 8, seed=77, pad_rows=0)
    assert p.m_indptr.numel() == 512
    out = run(p, 0.75)
    L.nvfp4lora_device_status()
    check_close(out, oracle(p, 0.75), what="grouped, 511 experts")
