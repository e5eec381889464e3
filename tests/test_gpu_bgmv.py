"""GPU parity of the routed-MoE FC2 LoRA delta (flashinfer.fused_moe.bgmv_moe_gemm2_lora_delta)
against the CPU oracle, through the C ABI: every shape class of the launcher (clusters of 1 to 8
CTAs per token), both element types in and out, adapters addressed by stride with padding between
blocks, tokens without an adapter, inactive slots, the routing checks on the device, and capture
in a CUDA graph."""

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
BF, HF = torch.bfloat16, torch.float16


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def upload(p):
    import nvfp4_block_scaled_mm_b200 as L
    a = [x.to(DEV) for x in p.a_banks]
    b = [x.to(DEV) for x in p.b_banks]
    return dict(act=p.act.to(DEV), perm=p.perm.to(DEV), a=a, b=b, wa=L.fill_w_ptr(a), wb=L.fill_w_ptr(b),
                ids=p.topk_ids.to(DEV), w=p.topk_weights.to(DEV), lids=p.lora_ids.to(DEV))


def run(p, g, out_dtype=BF, out=None, check=True):
    import nvfp4_block_scaled_mm_b200 as L
    y = L.bgmv_moe_gemm2_lora_delta(g["act"], g["perm"], g["wa"], p.stride_a, g["wb"], p.stride_b, g["ids"],
                                    g["w"], g["lids"], p.rank, p.H, lora_dtype=p.lora_dtype, scale=p.scale,
                                    out_dtype=out_dtype, out=out)
    if check:
        L.nvfp4lora_device_status()
    return y


def oracle(p, tokens=None):
    dt = "bf16" if p.lora_dtype == BF else "fp16"
    return O.bgmv_moe_lora_delta(_bits(p.act), p.perm.numpy(), [_bits(x) for x in p.a_banks], p.stride_a,
                                 [_bits(x) for x in p.b_banks], p.stride_b, p.topk_ids.numpy(),
                                 p.topk_weights.numpy(), p.lora_ids.numpy(), p.rank, p.H, p.scale, dt, tokens)


def assert_parity(y, ref, lora_ids):
    got = y.detach().cpu().double().numpy()
    assert np.all(np.isfinite(got))
    bad = np.abs(got - ref) > O.tolerance(ref)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside the bound; worst {np.abs(got - ref).max()}"
    if np.any(ref != 0):
        assert O.sqnr_db(ref, got) >= 50.0
    none = np.asarray(lora_ids) < 0
    assert np.all(_bits(y)[none] == 0), "a token without an adapter must get +0 everywhere"


# (T, top_k, experts, adapters, I, H, rank, lora dtype, out dtype, stride padding, segment alignment)
SHAPES = [
    (5, 2, 4, 3, 64, 40, 8, BF, BF, 8, 4),            # tiny: clusters of 4 (I / 8 = 8 vectors)
    (37, 4, 6, 2, 520, 300, 24, HF, HF, 0, 16),       # ragged I and H, rank 24, fp16 in and out
    (300, 8, 16, 4, 1536, 2048, 64, BF, BF, 16, 128),  # enough tokens for one CTA per token
    (1, 1, 2, 2, 4096, 4096, 128, BF, HF, 0, 128),    # one token, rank 128, clusters of 8
    (64, 2, 8, 4, 4096, 4096, 16, HF, BF, 0, 128),    # the decode batch, fp16 in, bf16 out
    (150, 16, 32, 2, 256, 512, 8, BF, BF, 8, 8),      # top_k 16
    (24, 16, 20, 2, 1024, 520, 128, BF, BF, 0, 16),   # the largest slot set: top_k 16 x rank 128, clusters
    (320, 16, 20, 2, 1024, 264, 128, HF, BF, 8, 128),  # the same with one CTA per token
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"T{s[0]}k{s[1]}E{s[2]}I{s[4]}H{s[5]}r{s[6]}")
def test_delta_matches_the_oracle(shape):
    T, top_k, E, La, I, H, r, ldt, odt, pad, seg = shape
    p = W.make_bgmv_problem(T, top_k, E, La, I, H, r, seed=T + r, lora_dtype=ldt, scale=1.5, stride_pad=pad,
                            seg_align=seg)
    y = run(p, upload(p), out_dtype=odt)
    assert y.dtype == odt and tuple(y.shape) == (T, H)
    assert_parity(y, oracle(p), p.lora_ids.numpy())


def test_workload_shape_full_and_deterministic():
    p = W.make_bgmv_problem(**W.BGMV)
    g = upload(p)
    y1 = run(p, g)
    y2 = run(p, g)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert (p.lora_ids < 0).any() and (p.perm < 0).any()
    assert_parity(y1, oracle(p), p.lora_ids.numpy())


def test_no_adapter_no_active_slot_and_no_tokens():
    import nvfp4_block_scaled_mm_b200 as L
    p = W.make_bgmv_problem(20, 2, 4, 2, 128, 96, 16, seed=3)
    g = upload(p)
    g["lids"].fill_(-1)
    y = run(p, g, out=torch.full((20, 96), 7.0, dtype=BF, device=DEV))
    assert torch.all(y.view(torch.int16) == 0)
    g = upload(p)
    g["perm"].fill_(-1)
    y = run(p, g, out=torch.full((20, 96), 7.0, dtype=BF, device=DEV))
    assert torch.all(y.view(torch.int16) == 0)
    g = upload(p)
    y = L.bgmv_moe_gemm2_lora_delta(g["act"], g["perm"][:0], g["wa"], p.stride_a, g["wb"], p.stride_b,
                                    g["ids"][:0], g["w"][:0], g["lids"][:0], p.rank, p.H)
    L.nvfp4lora_device_status()
    assert tuple(y.shape) == (0, 96)


@pytest.mark.parametrize("fault", ["expert", "row", "misaligned"])
def test_routing_out_of_range_is_reported_and_skipped(fault):
    import nvfp4_block_scaled_mm_b200 as L
    p = W.make_bgmv_problem(12, 2, 4, 2, 256, 128, 16, seed=8, p_no_lora=0.0, p_inactive=0.0, seg_align=16)
    g = upload(p)
    if fault == "expert":
        g["ids"][3, 1] = 4                                      # num_experts = 4
    elif fault == "row":
        g["perm"][7] = p.act.shape[0]                           # one past the last row
    else:
        g["wa"][0, 2] += 2                                      # a bank address off its 16-byte boundary
    run(p, g, check=False)
    with pytest.raises(ValueError, match="routing entry"):
        L.nvfp4lora_device_status()
    L.nvfp4lora_device_status()                                 # the word was cleared
    y = run(p, upload(p))                                       # and the next call is whole
    assert_parity(y, oracle(p), p.lora_ids.numpy())


def test_graph_replay_with_new_routing():
    """The routing is read on the device only, so one captured call serves new routing tables
    copied into its captured tensors."""
    p1 = W.make_bgmv_problem(48, 4, 8, 3, 512, 384, 32, seed=21)
    p2 = W.make_bgmv_problem(48, 4, 8, 3, 512, 384, 32, seed=22)
    g1, g2 = upload(p1), upload(p2)
    r1, r2 = p1.act.shape[0], p2.act.shape[0]
    act = torch.zeros(max(r1, r2), 512, dtype=BF, device=DEV)   # one buffer that holds either
    act[:r1].copy_(g1["act"])
    g1["act"] = act
    out = torch.empty(48, 384, dtype=BF, device=DEV)
    run(p1, g1, out=out)                                        # warm-up outside the capture
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(p1, g1, out=out, check=False)
    act[:r2].copy_(g2["act"])
    for name in ("perm", "ids", "w", "lids", "wa", "wb"):
        g1[name].copy_(g2[name])
    graph.replay()
    torch.cuda.synchronize()
    assert_parity(out, oracle(p2), p2.lora_ids.numpy())
