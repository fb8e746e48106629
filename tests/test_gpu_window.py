"""Sliding-window layers on the GPU: keys at distance >= window are hidden and
the visible ones follow the bifocal rule.  The CUDA path (through the C ABI)
against the fp64 oracle, prefill on both kernels, chunked prefill and decode
on both decode kernels."""
import pytest
import torch

import oracle
from zero_shot_rope_b200 import synth
from tests.gpu_util import assert_close, jl, to_np

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def prefill_window_gpu(q, k, v, cu_q, cu_k, w_pre, w0, window, theta, flags=0):
    J = jl()
    Tq, Hq, _ = q.shape
    lens = (cu_q[1:] - cu_q[:-1]).tolist()
    qd = q.to(DEV)
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((Hq, Tq), float("nan"), dtype=torch.float32, device=DEV)
    out, lse = J.jl_bifocal_prefill_kv(qd, k.to(DEV), v.to(DEV), cu_q.to(DEV), cu_k.to(DEV), max(max(lens), 1),
                                       w_pre, w0, theta, out=out, lse=lse, flags=flags, window=window)
    torch.cuda.synchronize()
    return out, lse


CASES = [
    # (seqlens, Hq, Hkv, w_pre, w0, window)
    ((1000,), 8, 2, 256, 200, 64),        # window < w0: plain sliding window
    ((1000,), 8, 2, 256, 200, 500),       # w0 < window < L, not tile-aligned
    ((777,), 4, 4, 160, 100, 128),        # tile-aligned window
    ((1500,), 4, 1, 512, 0, 300),         # w0 = 0: every visible pair grouped
    ((600,), 4, 2, 100, 50, 1),           # each query sees only itself
    ((64, 0, 513, 1, 260), 8, 2, 128, 96, 200),  # varlen with an empty sequence
    ((2048,), 4, 2, 4096, 64, 700),       # G = 1
    ((1000,), 8, 2, 256, 200, 5000),      # window wider than the sequence
]


@pytest.mark.parametrize("seqlens,Hq,Hkv,w_pre,w0,window", CASES)
@pytest.mark.parametrize("kernel", ["tensor", "simt"])
def test_windowed_prefill_full(seqlens, Hq, Hkv, w_pre, w0, window, kernel):
    J = jl()
    q, k, v, cu = synth.random_case(sum(seqlens) + window + w0, seqlens, Hq, Hkv, 128, torch.bfloat16)
    flags = J.JL_FLAG_SIMT if kernel == "simt" else 0
    out, lse = prefill_window_gpu(q, k, v, cu, cu, w_pre, w0, window, 1e6, flags=flags)
    ro, rl = oracle.bifocal_attention(q, k, v, cu, w_pre, w0, 1e6, window=window)
    assert_close(to_np(out), ro, torch.bfloat16, "out")
    assert_close(to_np(lse), rl, torch.bfloat16, "lse")


def test_windowed_prefill_plain_and_fp32():
    J = jl()
    q, k, v, cu = synth.random_case(12, (900,), 8, 2, 128, torch.bfloat16)
    out, lse = prefill_window_gpu(q, k, v, cu, cu, 200, 64, 333, 1e6, flags=J.JL_FLAG_PLAIN_CAUSAL)
    ro, rl = oracle.bifocal_attention(q, k, v, cu, 200, 64, 1e6, plain=True, window=333)
    assert_close(to_np(out), ro, torch.bfloat16, "plain out")
    q, k, v, cu = synth.random_case(13, (300, 41), 4, 2, 64, torch.float32)
    out, lse = prefill_window_gpu(q, k, v, cu, cu, 100, 30, 77, 1e4)
    ro, rl = oracle.bifocal_attention(q, k, v, cu, 100, 30, 1e4, window=77)
    assert_close(to_np(out), ro, torch.float32, "fp32 out")
    assert_close(to_np(lse), rl, torch.float32, "fp32 lse")


def test_windowed_chunk_against_cache():
    # the last 300 tokens of a 1000-token sequence, window 333
    q_all, k, v, cu_k = synth.random_case(14, (1000,), 8, 2, 128, torch.bfloat16)
    q = q_all[700:].contiguous()
    cu_q = torch.tensor([0, 300], dtype=torch.int32)
    out, lse = prefill_window_gpu(q, k, v, cu_q, cu_k, 256, 100, 333, 1e6)
    ro, rl = oracle.bifocal_attention_kv(q, k, v, cu_q, cu_k, 256, 100, 1e6, window=333)
    assert_close(to_np(out), ro, torch.bfloat16, "out")
    assert_close(to_np(lse), rl, torch.bfloat16, "lse")


def test_zero_window_is_bitwise_the_prefill():
    J = jl()
    q, k, v, cu = synth.random_case(15, (700, 1300), 8, 2, 128, torch.bfloat16)
    a, la = J.jl_bifocal_prefill(q.to(DEV), k.to(DEV), v.to(DEV), cu.to(DEV), 1300, 512, 200, 1e6,
                                 lse=torch.empty(8, 2000, device=DEV))
    b, lb = prefill_window_gpu(q, k, v, cu, cu, 512, 200, 0, 1e6)
    assert torch.equal(a, b) and torch.equal(la, lb)


DEC = [
    # (seqlens, cap, Hq, Hkv, D, w_pre, w0, window, dtype)
    ((1000,), 1024, 32, 8, 128, 250, 64, 300, torch.bfloat16),
    ((3333, 17, 2048), 4000, 16, 8, 128, 700, 300, 1000, torch.bfloat16),
    ((2500,), 2600, 8, 2, 128, 512, 400, 100, torch.bfloat16),      # window < w0
    ((2500, 9), 2600, 8, 2, 128, 512, 100, 1, torch.bfloat16),       # window 1
    ((1200,), 1200, 8, 8, 128, 300, 0, 5000, torch.bfloat16),        # window > L
    ((900, 33), 1000, 4, 4, 64, 200, 10, 129, torch.float32),        # CUDA-core decode kernel
    ((700,), 700, 4, 2, 64, 150, 50, 333, torch.bfloat16),
    ((5000, 611), 5000, 16, 4, 64, 900, 100, 700, torch.bfloat16),   # 256-key tiles, window off the grid
]


@pytest.mark.parametrize("seqlens,cap,Hq,Hkv,D,w_pre,w0,window,dtype", DEC)
def test_windowed_decode(seqlens, cap, Hq, Hkv, D, w_pre, w0, window, dtype):
    J = jl()
    B = len(seqlens)
    g = torch.Generator().manual_seed(sum(seqlens) + window)
    q = torch.randn(B, Hq, D, generator=g).to(dtype)
    kc = torch.randn(B, cap, Hkv, D, generator=g).to(dtype)
    vc = torch.randn(B, cap, Hkv, D, generator=g).to(dtype)
    sl = torch.tensor(seqlens, dtype=torch.int32, device=DEV)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)
    out, lse = J.jl_bifocal_decode_window(q.to(DEV), kc.to(DEV), vc.to(DEV), sl, max(seqlens), w_pre, w0, window,
                                          1e6, lse=lse)
    torch.cuda.synchronize()
    ro, rl = oracle.bifocal_decode(q, kc, vc, list(seqlens), w_pre, w0, 1e6, window=window)
    assert_close(to_np(out), ro, dtype, "out")
    assert_close(to_np(lse), rl, dtype, "lse")


def test_zero_window_decode_is_bitwise_the_decode():
    J = jl()
    g = torch.Generator().manual_seed(3)
    q = torch.randn(2, 32, 128, generator=g).to(torch.bfloat16).to(DEV)
    kc = torch.randn(2, 3000, 8, 128, generator=g).to(torch.bfloat16).to(DEV)
    vc = torch.randn(2, 3000, 8, 128, generator=g).to(torch.bfloat16).to(DEV)
    sl = torch.tensor([2999, 1500], dtype=torch.int32, device=DEV)
    a, _ = J.jl_bifocal_decode(q, kc, vc, sl, 3000, 1000, 300, 1e6)
    b, _ = J.jl_bifocal_decode_window(q, kc, vc, sl, 3000, 1000, 300, 0, 1e6)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
