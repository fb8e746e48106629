"""Decode parity on the GPU: the split-KV kernel (through the C ABI) against
the fp64 oracle at every tested step."""
import numpy as np
import pytest
import torch

import oracle
from zero_shot_rope_b200 import synth
from tests.gpu_util import assert_close, jl, to_np

pytestmark = pytest.mark.gpu


def decode_gpu(q, kc, vc, seqlens, max_seqlen, w_pre, w0, theta, flags=0):
    J = jl()
    dev = torch.device("cuda:0")
    B, Hq, _ = q.shape
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
    out, lse = J.jl_bifocal_decode(q.to(dev), kc.to(dev), vc.to(dev),
                                   torch.tensor(seqlens, dtype=torch.int32, device=dev), max_seqlen,
                                   w_pre, w0, theta, lse=lse, flags=flags)
    torch.cuda.synchronize()
    return out, lse


SMALL = [
    # (seqlens, cap, Hq, Hkv, D, w_pre, w0, dtype)
    ((1,), 8, 4, 1, 128, 1, 0, torch.bfloat16),
    ((100,), 128, 8, 2, 128, 40, 16, torch.bfloat16),
    ((1000,), 1024, 32, 8, 128, 250, 64, torch.bfloat16),       # G = 4
    ((1001,), 1024, 32, 8, 128, 250, 64, torch.bfloat16),       # G = 5 (just crossed)
    ((3333, 17, 2048), 4000, 16, 8, 128, 700, 300, torch.bfloat16),
    ((5000,), 5000, 8, 8, 128, 900, 0, torch.bfloat16),
    ((600,), 700, 8, 1, 128, 100, 600, torch.bfloat16),          # all keys local
    ((700,), 700, 4, 2, 64, 150, 50, torch.bfloat16),
    # head_dim 64 runs 256-key tiles: one key past a tile, several splits of
    # ragged lengths with eight query heads per kv head, a single key
    ((257,), 300, 8, 8, 64, 100, 20, torch.bfloat16),
    ((3333, 17, 2048), 4000, 16, 2, 64, 700, 300, torch.bfloat16),
    ((1,), 8, 4, 1, 64, 1, 0, torch.bfloat16),
    ((900, 33), 1000, 4, 4, 64, 200, 10, torch.float32),
    ((2500,), 2600, 16, 2, 128, 512, 100, torch.float32),
]


@pytest.mark.parametrize("seqlens,cap,Hq,Hkv,D,w_pre,w0,dtype", SMALL)
def test_decode_small_cases(seqlens, cap, Hq, Hkv, D, w_pre, w0, dtype):
    B = len(seqlens)
    g = torch.Generator().manual_seed(sum(seqlens) + D)
    q = torch.randn(B, Hq, D, generator=g).to(dtype)
    kc = torch.randn(B, cap, Hkv, D, generator=g).to(dtype)
    vc = torch.randn(B, cap, Hkv, D, generator=g).to(dtype)
    out, lse = decode_gpu(q, kc, vc, list(seqlens), max(seqlens), w_pre, w0, 1e6)
    ro, rl = oracle.bifocal_decode(q, kc, vc, list(seqlens), w_pre, w0, 1e6)
    assert_close(to_np(out), ro, dtype, "out")
    assert_close(to_np(lse), rl, dtype, "lse")
    po, pl = decode_gpu(q, kc, vc, list(seqlens), max(seqlens), w_pre, w0, 1e6,
                        flags=jl().JL_FLAG_PLAIN_CAUSAL)
    rpo, rpl = oracle.bifocal_decode(q, kc, vc, list(seqlens), w_pre, w0, 1e6, plain=True)
    assert_close(to_np(po), rpo, dtype, "plain out")


def test_decode_128k_all_256_steps():
    """The decode workload in full, in the benchmark's launch configuration:
    all 256 steps (L = 131072 .. 131327; G = 4 at the first step, 5 after),
    every output and LSE element of every step against the oracle.  The
    oracle's steps run in a pool of spawned host processes."""
    from tests import oracle_pool

    J = jl()
    w = synth.WORKLOADS["decode_128k"]
    kc, vc = synth.decode_cache(w)
    dev = torch.device("cuda:0")
    kd, vd = kc.to(dev), vc.to(dev)
    cap = kc.shape[1]
    n = w.decode_steps
    qs = torch.stack([synth.decode_query(w, t) for t in range(n)]).to(dev)  # [n, 1, Hq, D]
    lens = torch.tensor([w.seqlens[0] + t for t in range(n)], dtype=torch.int32, device=dev)
    outs = torch.full_like(qs, float("nan"))
    lses = torch.full((n, 1, w.n_q_heads), float("nan"), dtype=torch.float32, device=dev)
    ws = torch.zeros(J.jl_bifocal_decode_workspace_size(1, w.n_q_heads, w.n_kv_heads, w.head_dim, cap),
                     dtype=torch.uint8, device=dev)
    for t in range(n):
        J.jl_bifocal_decode(qs[t], kd, vd, lens[t:t + 1], cap, w.w_pretrained, w.w0, w.rope_theta,
                            out=outs[t], lse=lses[t], workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    got_o, got_l = to_np(outs), to_np(lses)
    del kd, vd
    checked = set()
    discr = {0, 1, 128, 255}  # steps that also run the plain-causal oracle
    with oracle_pool.pool(min(24, oracle_pool.n_workers())) as p:
        jobs = [("decode_128k", t, t in discr) for t in range(n)]
        for t, ro, rl, po in p.imap_unordered(oracle_pool.decode_step, jobs):
            assert_close(got_o[t], ro, torch.bfloat16, f"step {t}")
            assert_close(got_l[t], rl, torch.bfloat16, f"step {t} lse")
            assert np.linalg.norm(got_o[t] - ro) / np.linalg.norm(ro) < 1e-2, t
            if po is not None:
                # the grouped branch moves the result by far more than the error
                assert np.abs(po - ro).mean() > 5 * np.abs(got_o[t] - ro).mean(), t
            checked.add(t)
    assert checked == set(range(n))


@pytest.mark.parametrize("step", [0, 1])
def test_decode_128k_head_dim_64(step):
    """The decode workload's sizes at head_dim 64 (the tensor-core decode with
    the zero-padded PV), steps 0 and 1 (G = 4, then 5), in full."""
    w = synth.WORKLOADS["decode_128k"]
    g = torch.Generator().manual_seed(640 + step)
    cap = w.seqlens[0] + 1
    kc = torch.randn(1, cap, w.n_kv_heads, 64, generator=g).to(torch.bfloat16)
    vc = torch.randn(1, cap, w.n_kv_heads, 64, generator=g).to(torch.bfloat16)
    q = torch.randn(1, w.n_q_heads, 64, generator=g).to(torch.bfloat16)
    L = w.seqlens[0] + step
    out, lse = decode_gpu(q, kc, vc, [L], cap, w.w_pretrained, w.w0, w.rope_theta)
    ro, rl = oracle.bifocal_decode(q, kc, vc, [L], w.w_pretrained, w.w0, w.rope_theta)
    assert_close(to_np(out), ro, torch.bfloat16, f"D64 step {step}")
    assert_close(to_np(lse), rl, torch.bfloat16, f"D64 step {step} lse")
    assert np.linalg.norm(to_np(out) - ro) / np.linalg.norm(ro) < 1e-2


def test_decode_zero_length_writes_zero():
    dev = torch.device("cuda:0")
    q = torch.randn(2, 8, 128).to(torch.bfloat16)
    kc = torch.randn(2, 64, 2, 128).to(torch.bfloat16)
    vc = torch.randn(2, 64, 2, 128).to(torch.bfloat16)
    out, lse = decode_gpu(q, kc, vc, [0, 50], 64, 16, 8, 1e4)
    assert torch.all(out[0] == 0) and torch.all(torch.isinf(lse[0]))
    ro, _ = oracle.bifocal_decode(q[1:], kc[1:], vc[1:], [50], 16, 8, 1e4)
    assert_close(to_np(out[1:]), ro, torch.bfloat16, "row 1")


@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (64, torch.bfloat16), (128, torch.float32)])
def test_decode_ignores_garbage_past_the_length(D, dtype):
    # cache rows at and past L may hold anything (here NaN): they must not
    # reach the result (a 0 * NaN in the PV product would)
    g = torch.Generator().manual_seed(17)
    L, cap = 1000, 1200
    q = torch.randn(1, 8, D, generator=g).to(dtype)
    kc = torch.randn(1, cap, 2, D, generator=g).to(dtype)
    vc = torch.randn(1, cap, 2, D, generator=g).to(dtype)
    kc[:, L:] = float("nan")
    vc[:, L:] = float("nan")
    out, lse = decode_gpu(q, kc, vc, [L], cap, 300, 64, 1e6)
    ro, rl = oracle.bifocal_decode(q, kc, vc, [L], 300, 64, 1e6)
    assert_close(to_np(out), ro, dtype, "out")
    assert_close(to_np(lse), rl, dtype, "lse")


def test_decode_replays_from_a_cuda_graph():
    # The lengths live on the device and the split plan is sized by
    # max_seqlen (here the cache capacity), so a captured step replays
    # correctly after the caller updates q and seqlens in place, including
    # steps where G changes.
    J = jl()
    dev = torch.device("cuda:0")
    B, cap, Hq, Hkv, D, w_pre, w0 = 3, 3000, 16, 4, 128, 1000, 300
    g = torch.Generator().manual_seed(77)
    kc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    kcd, vcd = kc.to(dev), vc.to(dev)
    q_st = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device=dev)
    sl_st = torch.full((B,), 1, dtype=torch.int32, device=dev)
    out = torch.empty_like(q_st)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(J.jl_bifocal_decode_workspace_size(B, Hq, Hkv, D, cap), dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        J.jl_bifocal_decode(q_st, kcd, vcd, sl_st, cap, w_pre, w0, 1e6, out=out, lse=lse, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        J.jl_bifocal_decode(q_st, kcd, vcd, sl_st, cap, w_pre, w0, 1e6, out=out, lse=lse, workspace=ws)
    for step, lens in enumerate(([999, 1000, 2000], [1000, 1001, 2001], [1, 2999, 3000])):
        q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
        q_st.copy_(q.to(dev))
        sl_st.copy_(torch.tensor(lens, dtype=torch.int32).to(dev))
        graph.replay()
        torch.cuda.synchronize()
        ro, rl = oracle.bifocal_decode(q, kc, vc, lens, w_pre, w0, 1e6)
        assert_close(to_np(out), ro, torch.bfloat16, f"out step {step}")
        assert_close(to_np(lse), rl, torch.bfloat16, f"lse step {step}")
    assert int(ws[:4].view(torch.int32).item()) == 0


BALANCE = [
    # (seqlens, Hq, Hkv, D): fewer (sequence, kv head) pairs than SMs put the
    # splits on the device-planned balanced layout (one unit per SM)
    ((0, 1, 129, 5000, 20000, 7, 12345, 256), 32, 8, 128),     # empty, tiny and long sequences
    ((0, 1, 129, 5000, 20000, 7, 12345, 256), 32, 8, 64),
    (tuple(range(300, 300 + 18 * 700, 700)), 16, 8, 128),      # 144 pairs: one unit per pair
    (tuple(range(50, 50 + 37 * 97, 97)), 16, 4, 128),          # 148 pairs: the (split, head, sequence) grid
    ((3000,) * 5 + (1,), 8, 1, 128),                           # one kv head: up to 148 units
    (tuple(range(1, 1 + 70 * 37, 37)), 4, 2, 128),             # 70 sequences: the plan's chunks of 32
]


@pytest.mark.parametrize("seqlens,Hq,Hkv,D", BALANCE)
def test_decode_balanced_splits(seqlens, Hq, Hkv, D):
    # every key of every (sequence, kv head) falls in exactly one unit: the
    # combined result matches the oracle for ragged lengths, and repeated
    # calls with other lengths in the same workspace stay correct
    B, cap = len(seqlens), max(seqlens)
    g = torch.Generator().manual_seed(B * 1000 + D)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    for lens in (list(seqlens), [max(0, x - 129) for x in reversed(seqlens)]):
        out, lse = decode_gpu(q, kc, vc, lens, cap, 3000, 500, 1e6)
        ro, rl = oracle.bifocal_decode(q, kc, vc, lens, 3000, 500, 1e6)
        assert_close(to_np(out), ro, torch.bfloat16, f"out {lens[:3]}")
        assert_close(to_np(lse), rl, torch.bfloat16, f"lse {lens[:3]}")


@pytest.mark.parametrize("Hkv,D,dtype", [(2, 128, torch.bfloat16), (2, 64, torch.bfloat16),
                                         (2, 128, torch.float32), (80, 128, torch.bfloat16)])
def test_decode_length_past_max_seqlen_writes_zero(Hkv, D, dtype):
    # a length above max_seqlen (within the cache) is outside the contract:
    # zeros and LSE -inf, on every decode kernel and split plan (80 kv heads x
    # 2 sequences is past one unit per SM: the per-split grid)
    g = torch.Generator().manual_seed(Hkv + D)
    q = torch.randn(2, 2 * Hkv, D, generator=g).to(dtype)
    kc = torch.randn(2, 100, Hkv, D, generator=g).to(dtype)
    vc = torch.randn(2, 100, Hkv, D, generator=g).to(dtype)
    out, lse = decode_gpu(q, kc, vc, [50, 90], 60, 30, 8, 1e4)
    assert torch.all(out[1] == 0) and torch.all(torch.isinf(lse[1]))
    ro, rl = oracle.bifocal_decode(q[:1], kc[:1], vc[:1], [50], 30, 8, 1e4)
    assert_close(to_np(out[:1]), ro, dtype, "row 0")
    assert_close(to_np(lse[:1]), rl, dtype, "row 0 lse")
