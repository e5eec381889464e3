"""A few calls of one configurable shape, for attaching a profiler to a single kernel launch.

    python -m nvfp4_block_scaled_mm_b200.profile_case --shape M,N,K,r --path raw|prepared|off [--calls 4]
    python -m nvfp4_block_scaled_mm_b200.profile_case --grouped 512,128,1024 --shape 0,N,K,r [--calls 4]

Inputs are the seeded synthetic ones of the workloads; one copy of each is held on the device.
The calls run eagerly on the current stream, then the device error word is checked.
"""

from __future__ import annotations

import argparse
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main() -> int:
    import torch
    import nvfp4_block_scaled_mm_b200 as L
    from workloads import make_grouped_problem, make_problem

    ap = argparse.ArgumentParser()
    ap.add_argument("--shape", required=True, help="M,N,K,r (M ignored with --grouped)")
    ap.add_argument("--path", choices=["raw", "prepared", "off"], default="raw")
    ap.add_argument("--grouped", default=None, help="comma-separated rows per expert (multiples of 128)")
    ap.add_argument("--calls", type=int, default=4)
    args = ap.parse_args()
    M, N, K, r = (int(x) for x in args.shape.split(","))
    dev = "cuda"
    s = torch.tensor([0.5], dtype=torch.float32, device=dev)
    if args.grouped:
        p = make_grouped_problem([int(x) for x in args.grouped.split(",")], N, K, r, seed=9)
        t = {k: getattr(p, k).to(dev) for k in ("m_indptr", "a", "b", "a_sf", "b_sf", "alpha", "d", "lora_b")}
        for _ in range(args.calls):
            L.grouped_mm_nvfp4_lora(t["a"], t["b"], t["a_sf"], t["b_sf"], t["m_indptr"], t["alpha"], t["d"],
                                    t["lora_b"], None if args.path == "off" else s)
    else:
        p = make_problem(M, N, K, r, seed=9, alpha=2.0 ** -9, lora_scale=0.5, bias=False)
        a, b, a_sf, b_sf, d, lb = (x.to(dev) for x in (p.a, p.b, p.a_sf, p.b_sf, p.d, p.lora_b))
        alpha = torch.tensor([p.alpha], dtype=torch.float32, device=dev)
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        adp = L.prepare_nvfp4_lora_adapter(lb, s, alpha) if args.path == "prepared" else None
        for _ in range(args.calls):
            if args.path == "prepared":
                L.mm_nvfp4_lora(a, b, a_sf, b_sf, alpha, d, lora_adapter=adp, out=out)
            elif args.path == "raw":
                L.mm_nvfp4_lora(a, b, a_sf, b_sf, alpha, d, lb, s, out=out)
            else:
                L.mm_nvfp4_lora(a, b, a_sf, b_sf, alpha, out=out)
    L.nvfp4lora_device_status()
    print("profile_case: %d calls done" % args.calls)
    return 0


if __name__ == "__main__":
    sys.exit(main())
