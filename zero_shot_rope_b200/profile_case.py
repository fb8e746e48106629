"""Run one attention case a few times through the C ABI, for profilers.

  python -m zero_shot_rope_b200.profile_case prefill --seqlen 32768 --w-pre 8192 --reps 3
  python -m zero_shot_rope_b200.profile_case decode --seqlen 131072 --reps 3

Inputs are seeded synthetic N(0, 1) tensors (zero_shot_rope_b200.synth).  The
first repetition is a warm-up; skip it in the profiler (``ncu -s``).
"""
from __future__ import annotations

import argparse

import torch

from . import build, synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kind", choices=["prefill", "decode"])
    ap.add_argument("--seqlen", type=int, default=32768)
    ap.add_argument("--hq", type=int, default=32)
    ap.add_argument("--hkv", type=int, default=8)
    ap.add_argument("--w-pre", type=int, default=32768)
    ap.add_argument("--w0", type=int, default=4096)
    ap.add_argument("--theta", type=float, default=1e6)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--plain", action="store_true")
    a = ap.parse_args()
    build.build()
    from . import jetlong as jl

    dev = torch.device("cuda:0")
    flags = jl.JL_FLAG_PLAIN_CAUSAL if a.plain else 0
    if a.kind == "prefill":
        q, k, v, cu = synth.random_case(3, (a.seqlen,), a.hq, a.hkv, 128, torch.bfloat16)
        q, k, v, cu = q.to(dev), k.to(dev), v.to(dev), cu.to(dev)
        out = torch.empty_like(q)
        ws = torch.empty(jl.jl_bifocal_prefill_workspace_size(1, a.seqlen, a.hq, a.hkv, 128), dtype=torch.uint8,
                         device=dev)
        for _ in range(a.reps):
            jl.jl_bifocal_prefill(q, k, v, cu, a.seqlen, a.w_pre, a.w0, a.theta, out=out, flags=flags,
                                  workspace=ws)
    else:
        g = torch.Generator().manual_seed(5)
        cap = a.seqlen
        kc = torch.randn(1, cap, a.hkv, 128, generator=g).to(torch.bfloat16).to(dev)
        vc = torch.randn(1, cap, a.hkv, 128, generator=g).to(torch.bfloat16).to(dev)
        q = torch.randn(1, a.hq, 128, generator=g).to(torch.bfloat16).to(dev)
        sl = torch.tensor([a.seqlen], dtype=torch.int32, device=dev)
        out = torch.empty_like(q)
        ws = torch.empty(jl.jl_bifocal_decode_workspace_size(1, a.hq, a.hkv, 128, cap), dtype=torch.uint8,
                         device=dev)
        for _ in range(a.reps):
            jl.jl_bifocal_decode(q, kc, vc, sl, cap, a.w_pre, a.w0, a.theta, out=out, flags=flags, workspace=ws)
    torch.cuda.synchronize()
    print("done", a.kind, a.seqlen)


if __name__ == "__main__":
    main()
