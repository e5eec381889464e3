"""Host-only checks of the C ABI: the library loads, exports every symbol the header
declares, and rejects rule violations before touching CUDA (no GPU needed)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4lora.h")


@pytest.fixture(scope="module")
def lib():
    from nvfp4_block_scaled_mm_b200.build import build
    path = build(quiet=True)
    return ctypes.CDLL(path)


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4LORA_API\s+[\w\s\*]+?\b(nvfp4lora_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("nvfp4lora_mm", "nvfp4lora_prepare", "nvfp4lora_refold", "nvfp4lora_mm_prepared",
                 "nvfp4lora_device_status", "nvfp4lora_last_error", "nvfp4lora_version"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_binding_exposes_the_same_names():
    import nvfp4_block_scaled_mm_b200 as L
    for name in declared_symbols():
        if name in ("nvfp4lora_last_error", "nvfp4lora_version"):
            continue
        assert callable(getattr(L, name)), name


P = ctypes.c_void_p
I64 = ctypes.c_int64


def _mm(lib, **kw):
    f = lib.nvfp4lora_mm
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, I64, P, I64, P, P, P, P, I64, P, P, I64, I64, I64, P]
    lib.nvfp4lora_last_error.restype = ctypes.c_char_p
    args = dict(a=0x10000, b=0x20000, a_sf=0x30000, a_sf_bytes=1 << 30, b_sf=0x40000, b_sf_bytes=1 << 30,
                alpha=0x50000, d=0x60000, lora_b=0x70000, lora_scale=0x80000, r=16, bias=None,
                out=0x90000, M=128, N=256, K=256)
    args.update(kw)
    st = f(args["a"], args["b"], args["a_sf"], args["a_sf_bytes"], args["b_sf"], args["b_sf_bytes"],
           args["alpha"], args["d"], args["lora_b"], args["lora_scale"], args["r"], args["bias"], args["out"],
           args["M"], args["N"], args["K"], None)
    return st, lib.nvfp4lora_last_error().decode()


@pytest.mark.parametrize("kw,needle", [
    (dict(M=0), "M >= 1"),
    (dict(N=0), "N >= 1"),
    (dict(K=300), "multiple of 256"),
    (dict(K=0), "multiple of 256"),
    (dict(r=12), "multiple of 8"),
    (dict(r=136), "multiple of 8"),
    (dict(r=0), "multiple of 8"),
    (dict(a=0x10004), "16-byte aligned"),
    (dict(out=0x90002), "16-byte aligned"),
    (dict(alpha=None), "non-null"),
    (dict(d=None), "d and lora_b"),
    (dict(a_sf_bytes=128 * 16 - 1), "a_sf has"),
    (dict(M=129, a_sf_bytes=128 * 16), "a_sf has"),
    (dict(N=257, b_sf_bytes=256 * 16), "b_sf has"),
    (dict(M=1 << 31), "2^30"),
])
def test_rule_violations_are_rejected_before_cuda(lib, kw, needle):
    st, msg = _mm(lib, **kw)
    assert st == 1, (st, msg)
    assert needle in msg, msg


def test_adapter_off_ignores_rank(lib):
    """lora_scale = NULL is the adapter-off call: a bad r is not a violation there.  (The
    call then proceeds to CUDA, which fails without a GPU with a CUDA status, not 1.)"""
    st, msg = _mm(lib, lora_scale=None, r=3, d=None, lora_b=None)
    assert st != 1, msg


def test_prepare_rules(lib):
    f = lib.nvfp4lora_prepare
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, I64, I64, P, P, ctypes.c_uint64, P, P]
    buf = ctypes.create_string_buffer(128)
    assert f(0x1000, 0x2000, 0x3000, 16, 12, 0x4000, 0x5000, 0, buf, None) == 1
    assert f(0x1000, 0x2000, 0x3000, 0, 16, 0x4000, 0x5000, 0, buf, None) == 1
    assert f(0x1000, 0x2000, 0x3000, 16, 16, 0x4000, 0x2000, 0, buf, None) == 1   # ratio aliases lora_scale
    assert f(0x1000, 0x2000, 0x3000, 16, 16, 0x4000, 0x5000, 0, None, None) == 1


def test_version_string(lib):
    lib.nvfp4lora_version.restype = ctypes.c_char_p
    assert b"sm_100a" in lib.nvfp4lora_version()


def test_selftest_limit_is_checked_before_cuda(lib):
    f = lib.nvfp4lora_selftest_wait_timeout
    f.restype = ctypes.c_int
    f.argtypes = [I64, P]
    lib.nvfp4lora_last_error.restype = ctypes.c_char_p
    for bad in (0, -5, 2_000_000_000):
        assert f(bad, None) == 1
        assert b"limit_ns" in lib.nvfp4lora_last_error()


def test_quantize_rules_are_checked_before_cuda(lib):
    f = lib.nvfp4lora_quantize
    f.restype = ctypes.c_int
    f.argtypes = [P, I64, I64, P, P, P, I64, P]
    lib.nvfp4lora_last_error.restype = ctypes.c_char_p
    ok = dict(x=0x10000, rows=130, K=256, gs=0x20000, codes=0x30000, scales=0x40000, nbytes=256 * 16)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["x"], a["rows"], a["K"], a["gs"], a["codes"], a["scales"], a["nbytes"], None)

    for bad, word in ((dict(K=96), b"K"), (dict(K=0), b"K"), (dict(rows=0), b"rows"),
                      (dict(nbytes=256 * 16 - 1), b"scales needs"), (dict(x=0x10008), b"aligned"),
                      (dict(scales=None), b"non-null"), (dict(gs=None), b"non-null"),
                      (dict(gs=0x20002), b"global_scale must be 4-byte aligned")):
        assert call(**bad) == 1, bad
        assert word in lib.nvfp4lora_last_error(), (bad, lib.nvfp4lora_last_error())


def test_binding_refuses_tensors_on_another_device():
    """The binding's device rule, exercised with CPU and meta tensors (no GPU needed): an operand
    on another device than the anchor raises ValueError naming it; None operands are skipped."""
    import torch
    import nvfp4_block_scaled_mm_b200 as L
    a = torch.empty(4, device="cpu")
    L._same_device("a", a, b=torch.empty(2, device="cpu"), d=None)
    with pytest.raises(ValueError, match="lora_b is on meta"):
        L._same_device("a", a, b=torch.empty(2, device="cpu"), lora_b=torch.empty(2, device="meta"))


def test_grouped_rules_are_checked_before_cuda(lib):
    f = lib.nvfp4lora_grouped_mm
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, I64, P, I64, P, I64, P, P, P, P, I64, P, P, I64, I64, I64, P]
    lib.nvfp4lora_last_error.restype = ctypes.c_char_p
    ok = dict(a=0x10000, b=0x20000, a_sf=0x30000, a_sf_bytes=1 << 30, b_sf=0x40000, b_sf_bytes=1 << 30,
              ind=0x50000, E=4, alpha=0x60000, d=0x70000, lb=0x80000, s=0x90000, r=16, bias=None,
              out=0xA0000, rows=512, N=256, K=256)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["a"], a["b"], a["a_sf"], a["a_sf_bytes"], a["b_sf"], a["b_sf_bytes"], a["ind"], a["E"],
                 a["alpha"], a["d"], a["lb"], a["s"], a["r"], a["bias"], a["out"], a["rows"], a["N"], a["K"], None)

    for bad, word in ((dict(E=0), b"num_experts"), (dict(E=512), b"num_experts"), (dict(ind=None), b"m_indptr"),
                      (dict(ind=0x50002), b"m_indptr"), (dict(b_sf_bytes=4 * 256 * 16 - 1), b"b_sf"),
                      (dict(K=200), b"K = 200"), (dict(r=12), b"rank"), (dict(d=None), b"non-null"),
                      (dict(a_sf_bytes=512 * 16 - 1), b"a_sf")):
        assert call(**bad) == 1, bad
        assert word in lib.nvfp4lora_last_error(), (bad, lib.nvfp4lora_last_error())


def test_lora_delta_rules_are_checked_before_cuda(lib):
    f = lib.nvfp4lora_bgmv_moe_gemm2_lora_delta
    f.restype = ctypes.c_int
    f.argtypes = [P, I64, I64, P, P, I64, P, I64, P, P, P, I64, I64, I64, I64, I64, ctypes.c_int32, ctypes.c_float,
                  ctypes.c_int32, P, P]
    lib.nvfp4lora_last_error.restype = ctypes.c_char_p
    ok = dict(act=0x10000, rows=256, I=512, perm=0x20000, wa=0x30000, sa=16 * 512, wb=0x40000, sb=256 * 16,
              ids=0x50000, w=0x60000, lids=0x70000, T=8, top_k=2, E=4, rank=16, H=256, ldt=0, scale=1.0, odt=0,
              out=0x80000)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["act"], a["rows"], a["I"], a["perm"], a["wa"], a["sa"], a["wb"], a["sb"], a["ids"], a["w"],
                 a["lids"], a["T"], a["top_k"], a["E"], a["rank"], a["H"], a["ldt"], a["scale"], a["odt"], a["out"],
                 None)

    for bad, word in ((dict(rank=12), b"rank"), (dict(rank=136), b"rank"), (dict(top_k=0), b"top_k"),
                      (dict(top_k=17), b"top_k"), (dict(I=100), b"I = 100"), (dict(H=0), b"hidden_size"),
                      (dict(E=0), b"num_experts"), (dict(sa=12), b"lora_stride"), (dict(sb=-8), b"lora_stride"),
                      (dict(ldt=2), b"dtype"), (dict(odt=-1), b"dtype"), (dict(T=-1), b"num_tokens"),
                      (dict(perm=None), b"non-null"), (dict(out=None), b"non-null"),
                      (dict(act=0x10008), b"16-byte"), (dict(wa=0x30004), b"8-byte"),
                      (dict(ids=0x50002), b"4-byte")):
        assert call(**bad) == 1, bad
        assert word in lib.nvfp4lora_last_error(), (bad, lib.nvfp4lora_last_error())
    # no tokens: nothing to do, and nothing is enqueued (no CUDA call is made)
    assert call(T=0, perm=None, out=None) == 0


def test_lora_delta_binding_rules():
    import torch
    import nvfp4_block_scaled_mm_b200 as L
    with pytest.raises(ValueError, match="CUDA tensor"):
        L.fill_w_ptr([torch.zeros(4, dtype=torch.bfloat16)])
    with pytest.raises(ValueError, match="at least one"):
        L.fill_w_ptr([])
    with pytest.raises(ValueError, match="lora_dtype"):
        L.bgmv_moe_gemm2_lora_delta(torch.zeros(1, 8), None, None, 0, None, 0, None, None, None, 8, 8,
                                    lora_dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        L.bgmv_moe_gemm2_lora_delta(torch.zeros(1, 8, dtype=torch.bfloat16), None, None, 0, None, 0, None, None,
                                    None, 8, 8)
