"""GPU tests of the API contract: CUDA-graph adapter switching, stale-adapter detection and
argument errors (flashinfer.gemm.mm_nvfp4_lora: Parameters, Notes: Shape rules and CUDA
graphs; prepare_nvfp4_lora_adapter: Parameters: out, Returns)."""

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_mm_b200 as L
from workloads import make_adapters, make_problem
from gpu_util import Dev

pytestmark = pytest.mark.gpu


def same(x, y):
    return torch.equal(x.view(torch.int16), y.view(torch.int16))


@pytest.fixture(params=[(16, 4096, 1024, 64), (200, 300, 512, 16)], ids=["decode", "tiled"])
def prob(request):
    M, N, K, r = request.param
    p = make_problem(M, N, K, r, seed=M + 11, alpha=2.0 ** -9, lora_scale=1.5, bias=True)
    return Dev(p)


def raw(x, d, lb, s, out=None):
    return L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, d, lb, s, bias=x.bias, out=out)


def test_lora_scale_none_is_adapter_off(prob):
    x = prob
    off = L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, bias=x.bias)
    none = L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, x.lora_b, None, bias=x.bias)
    torch.cuda.synchronize()
    assert same(off, none)


def test_graph_raw_path_copy_into_captured_tensors(prob):
    """Raw path: a captured call keeps its pointers; copy_ of a new adapter into the captured
    tensors changes what the replay computes (Notes: CUDA graphs)."""
    x = prob
    adapters = make_adapters(x.N, x.r, 3, seed=5)
    lb_cap = adapters[0][0].cuda()
    s_cap = torch.tensor([adapters[0][1]], dtype=torch.float32, device="cuda")
    out_cap = x.new_out()
    raw(x, x.d, lb_cap, s_cap, out_cap)          # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        raw(x, x.d, lb_cap, s_cap, out_cap)
    for lb, s in adapters[1:]:
        lb_cap.copy_(lb.cuda())
        s_cap.fill_(s)
        g.replay()
        ref = raw(x, x.d, lb.cuda(), torch.tensor([s], dtype=torch.float32, device="cuda"))
        torch.cuda.synchronize()
        assert same(out_cap, ref)
    L.nvfp4lora_device_status()


def test_graph_prepared_path_refold_in_graph(prob):
    """Prepared path: capture [refold(out=adapter); call]; a copy_ into the captured sources is
    folded by every replay, bitwise as an eager prepare + call would give."""
    x = prob
    adapters = make_adapters(x.N, x.r, 3, seed=6)
    lb_src = adapters[0][0].cuda()
    s_src = torch.tensor([adapters[0][1]], dtype=torch.float32, device="cuda")
    adp = L.prepare_nvfp4_lora_adapter(lb_src, s_src, x.alpha)
    out_cap = x.new_out()
    L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp, bias=x.bias, out=out_cap)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        L.prepare_nvfp4_lora_adapter(lb_src, s_src, x.alpha, out=adp)
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp, bias=x.bias, out=out_cap)
    for lb, s in adapters[1:] + [(adapters[0][0], 0.0)]:
        lb_src.copy_(lb.cuda())
        s_src.fill_(s)
        g.replay()
        torch.cuda.synchronize()
        got = out_cap.clone()
        folded = adp.b_folded.clone()
        fresh_lb = lb.cuda()
        fresh_s = torch.tensor([s], dtype=torch.float32, device="cuda")
        eager = L.prepare_nvfp4_lora_adapter(fresh_lb, fresh_s, x.alpha)
        ref = L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=eager, bias=x.bias)
        torch.cuda.synchronize()
        assert same(folded, eager.b_folded)
        assert same(got, ref)
        if s == 0.0:
            off = L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, bias=x.bias)
            torch.cuda.synchronize()
            assert same(got, off)
    L.nvfp4lora_device_status()


def test_stale_adapter_detection(prob):
    x = prob
    lb = x.lora_b.clone()
    s = x.lora_scale.clone()
    adp = L.prepare_nvfp4_lora_adapter(lb, s, x.alpha)
    L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp)
    lb.add_(1.0)                                            # written since the prepare
    with pytest.raises(L.StaleAdapterError):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp)
    L.prepare_nvfp4_lora_adapter(lb, s, x.alpha, out=adp)   # re-prepare clears it
    L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp)
    s.fill_(2.0)
    with pytest.raises(L.StaleAdapterError):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp)
    L.prepare_nvfp4_lora_adapter(lb, s, x.alpha, out=adp)
    other_alpha = x.alpha.clone()
    with pytest.raises(L.StaleAdapterError):                # another alpha tensor
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, other_alpha, x.d, lora_adapter=adp)
    lb.set_(lb.clone())                                     # moved
    with pytest.raises(L.StaleAdapterError):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, lora_adapter=adp)
    with pytest.raises(ValueError):                         # refold with another alpha
        L.prepare_nvfp4_lora_adapter(lb, s, other_alpha, out=adp)
    L.nvfp4lora_device_status()


def test_argument_errors(prob):
    x = prob
    adp = L.prepare_nvfp4_lora_adapter(x.lora_b, x.lora_scale, x.alpha)
    with pytest.raises(ValueError, match="not both"):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, x.d, x.lora_b, x.lora_scale, lora_adapter=adp)
    with pytest.raises(ValueError, match="bfloat16"):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, out_dtype=torch.float16)
    with pytest.raises(ValueError):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, backend="cudnn")
    bad_d = torch.zeros(x.M, 12, dtype=torch.bfloat16, device="cuda")
    bad_lb = torch.zeros(x.N, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="multiple of 8"):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, bad_d, bad_lb, x.lora_scale)
    a_short = x.a[:, : x.a.shape[1] - 64].contiguous()      # K not a multiple of 256
    b_short = x.b[:, : x.b.shape[1] - 64].contiguous()
    with pytest.raises(ValueError, match="multiple of 256"):
        L.mm_nvfp4_lora(a_short, b_short, x.a_sf, x.b_sf, x.alpha)
    with pytest.raises(ValueError, match="a_sf has"):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf[:100], x.b_sf, x.alpha)
    with pytest.raises(ValueError, match="prepared path still requires d"):
        L.mm_nvfp4_lora(x.a, x.b, x.a_sf, x.b_sf, x.alpha, lora_adapter=adp)
    L.nvfp4lora_device_status()


def test_larger_scale_buffers_accepted(prob):
    """Parameters: a_sf / b_sf -- larger contiguous backing buffers are accepted."""
    x = prob
    big_a = torch.cat([x.a_sf, torch.full((4096,), 0x7F, dtype=torch.uint8, device="cuda")])
    big_b = torch.cat([x.b_sf, torch.full((4096,), 0x7F, dtype=torch.uint8, device="cuda")])
    ref = raw(x, x.d, x.lora_b, x.lora_scale)
    got = L.mm_nvfp4_lora(x.a, x.b, big_a, big_b, x.alpha, x.d, x.lora_b, x.lora_scale, bias=x.bias)
    torch.cuda.synchronize()
    assert same(got, ref)


def test_bounded_wait_runs_out_and_the_context_stays_usable(prob):
    """The failure path of the kernels' bounded waits: a wait that nothing completes gives up
    after its limit, the device error word reports it once, and the GPU keeps computing."""
    import time
    x = prob
    L.nvfp4lora_device_status()                       # nothing pending
    t0 = time.perf_counter()
    L.nvfp4lora_selftest_wait_timeout(20_000_000)     # 20 ms
    with pytest.raises(L.DeviceTimeoutError):
        L.nvfp4lora_device_status()
    waited = time.perf_counter() - t0
    assert 0.015 < waited < 5.0, waited
    L.nvfp4lora_device_status()                       # the word was cleared
    # the context is intact: a GEMM after the timeout equals one before it, bit for bit
    before = raw(x, x.d, x.lora_b, x.lora_scale)
    torch.cuda.synchronize()
    after = raw(x, x.d, x.lora_b, x.lora_scale)
    torch.cuda.synchronize()
    assert same(before, after)
    L.nvfp4lora_device_status()
