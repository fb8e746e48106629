"""Time the attention calls across local-window sizes w0.

  python -m zero_shot_rope_b200.sweep [--seqlen 131072] [--w-pre 32768] [--w0 512 1024 2048 4096]

The local window decides how many key tiles of each query tile are scored
twice (base and grouped operands on the tile that straddles distance w0) and
how many keys a decode step rotates, so its cost is the one knob of the
method that moves the tile mix.  Prints one markdown table: prefill TFLOP/s
(causal QK^T + PV FLOPs / CUDA-event time) and decode microseconds per token,
each beside the plain-causal call on the same inputs.  Inputs are seeded
synthetic N(0, 1) tensors (zero_shot_rope_b200.synth), Qwen3-style 32/8 heads,
head_dim 128, bf16.
"""
from __future__ import annotations

import argparse
import statistics

import torch

from . import build, synth


def _time(fn, reps):
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--seqlen", type=int, default=131072)
    ap.add_argument("--w-pre", type=int, default=32768)
    ap.add_argument("--w0", type=int, nargs="+", default=[512, 1024, 2048, 4096, 8192])
    ap.add_argument("--hq", type=int, default=32)
    ap.add_argument("--hkv", type=int, default=8)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    build.build()
    from . import jetlong as jl

    dev = torch.device("cuda:0")
    L, Hq, Hkv, D = a.seqlen, a.hq, a.hkv, 128
    q, k, v, cu = synth.random_case(3, (L,), Hq, Hkv, D, torch.bfloat16)
    q, k, v, cu = q.to(dev), k.to(dev), v.to(dev), cu.to(dev)
    out = torch.empty_like(q)
    ws = torch.empty(jl.jl_bifocal_prefill_workspace_size(1, L, Hq, Hkv, D), dtype=torch.uint8, device=dev)
    flops = 4.0 * D * Hq * L * (L + 1) / 2
    # decode: the same keys as a cache, one query at position L - 1
    kc, vc = k.view(1, L, Hkv, D), v.view(1, L, Hkv, D)
    qd = q[L - 1:L].contiguous()
    od = torch.empty_like(qd)
    sl = torch.tensor([L], dtype=torch.int32, device=dev)
    wsd = torch.empty(jl.jl_bifocal_decode_workspace_size(1, Hq, Hkv, D, L), dtype=torch.uint8, device=dev)
    G = jl.jl_group_size(L, a.w_pre)

    def prefill(w0, flags):
        return lambda: jl.jl_bifocal_prefill(q, k, v, cu, L, a.w_pre, w0, 1e6, out=out, flags=flags, workspace=ws)

    def decode(w0, flags, n=20):
        return lambda: [jl.jl_bifocal_decode(qd, kc, vc, sl, L, a.w_pre, w0, 1e6, out=od, flags=flags,
                                             workspace=wsd) for _ in range(n)]

    plain_ms = _time(prefill(0, jl.JL_FLAG_PLAIN_CAUSAL), a.reps)
    plain_us = _time(decode(0, jl.JL_FLAG_PLAIN_CAUSAL), a.reps) * 1e3 / 20
    print(f"L = {L}, {Hq}/{Hkv} heads, D = {D}, w_pre = {a.w_pre} (G = {G}), bf16")
    print()
    print("| w0 | prefill ms | prefill TFLOP/s | vs plain | decode us/token | vs plain |")
    print("|---:|---:|---:|---:|---:|---:|")
    print(f"| plain | {plain_ms:.2f} | {flops / plain_ms / 1e9:.1f} | 1.000 | {plain_us:.1f} | 1.000 |")
    for w0 in a.w0:
        ms = _time(prefill(w0, 0), a.reps)
        us = _time(decode(w0, 0), a.reps) * 1e3 / 20
        print(f"| {w0} | {ms:.2f} | {flops / ms / 1e9:.1f} | {ms / plain_ms:.3f} | {us:.1f} | {us / plain_us:.3f} |",
              flush=True)


if __name__ == "__main__":
    main()
