"""Prefill of a chunk of new tokens against keys that include an existing
cache, on the GPU: the CUDA path (through the C ABI) against the fp64 oracle.
The chunk's queries sit at the last positions of each sequence and G follows
the current length, so chunk offsets that are not tile-aligned and chunks that
move G across a boundary are the cases that matter."""
import numpy as np
import pytest
import torch

import oracle
from zero_shot_rope_b200 import synth
from tests.gpu_util import assert_close, jl, prefill_gpu, to_np

pytestmark = pytest.mark.gpu


def chunk_case(seed, lq, lk, Hq, Hkv, D=128, dtype=torch.bfloat16):
    """Keys/values for lengths ``lk``; the queries are the last ``lq`` rows of
    each sequence's own query stream."""
    q_all, k, v, cu_k = synth.random_case(seed, lk, Hq, Hkv, D, dtype)
    rows = np.concatenate([np.arange(int(cu_k[s + 1]) - n, int(cu_k[s + 1])) for s, n in enumerate(lq)]
                          + [np.zeros(0, dtype=np.int64)]).astype(np.int64)
    q = q_all[torch.from_numpy(rows)].contiguous()
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    return q, k, v, cu_q, cu_k


def prefill_kv_gpu(q, k, v, cu_q, cu_k, w_pre, w0, theta, flags=0):
    J = jl()
    dev = torch.device("cuda:0")
    Tq, Hq, _ = q.shape
    lens = (cu_q[1:] - cu_q[:-1]).tolist()
    qd = q.to(dev)
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((Hq, Tq), float("nan"), dtype=torch.float32, device=dev)
    out, lse = J.jl_bifocal_prefill_kv(qd, k.to(dev), v.to(dev), cu_q.to(dev), cu_k.to(dev),
                                       max(max(lens), 1), w_pre, w0, theta, out=out, lse=lse, flags=flags)
    torch.cuda.synchronize()
    return out, lse


KV_CASES = [
    # (Lq per sequence, Lk per sequence, Hq, Hkv, w_pre, w0)
    ((300,), (1000,), 8, 2, 256, 200),            # offset 700: not tile-aligned, G = 4
    ((128,), (1024,), 4, 1, 255, 64),             # G(1024) = 5, G(896) = 4: the chunk moves G
    ((1,), (777,), 4, 4, 160, 100),               # one-token chunk = a decode step
    ((129,), (129,), 4, 2, 64, 16),               # chunk = whole sequence
    ((200,), (3000,), 8, 2, 1000, 0),             # w0 = 0: every pair grouped
    ((50,), (2000,), 4, 2, 4096, 64),             # G = 1
    ((0, 1, 128, 77, 256), (50, 1, 128, 900, 5000), 8, 2, 1024, 96),  # varlen, an empty chunk
]


@pytest.mark.parametrize("lq,lk,Hq,Hkv,w_pre,w0", KV_CASES)
@pytest.mark.parametrize("kernel", ["tensor", "prerotated", "simt"])
def test_chunk_against_cache_full(lq, lk, Hq, Hkv, w_pre, w0, kernel):
    # "tensor": grouped keys rotated in the tile; "prerotated": the ablation
    # that writes them for the whole key set in a pre-pass
    J = jl()
    q, k, v, cu_q, cu_k = chunk_case(sum(lk) + Hq + w0, lq, lk, Hq, Hkv)
    flags = {"tensor": 0, "prerotated": J.JL_FLAG_PREROTATE_K, "simt": J.JL_FLAG_SIMT}[kernel]
    out, lse = prefill_kv_gpu(q, k, v, cu_q, cu_k, w_pre, w0, 1e6, flags=flags)
    ro, rl = oracle.bifocal_attention_kv(q, k, v, cu_q, cu_k, w_pre, w0, 1e6)
    assert_close(to_np(out), ro, torch.bfloat16, "out")
    assert_close(to_np(lse), rl, torch.bfloat16, "lse")


def test_chunk_plain_causal():
    J = jl()
    q, k, v, cu_q, cu_k = chunk_case(21, (333,), (2222,), 8, 2)
    out, lse = prefill_kv_gpu(q, k, v, cu_q, cu_k, 500, 128, 1e6, flags=J.JL_FLAG_PLAIN_CAUSAL)
    ro, rl = oracle.bifocal_attention_kv(q, k, v, cu_q, cu_k, 500, 128, 1e6, plain=True)
    assert_close(to_np(out), ro, torch.bfloat16, "out")
    assert_close(to_np(lse), rl, torch.bfloat16, "lse")


def test_chunk_fp32_simt():
    q, k, v, cu_q, cu_k = chunk_case(4, (40, 9), (300, 9), 4, 2, D=64, dtype=torch.float32)
    out, lse = prefill_kv_gpu(q, k, v, cu_q, cu_k, 100, 30, 1e4)
    ro, rl = oracle.bifocal_attention_kv(q, k, v, cu_q, cu_k, 100, 30, 1e4)
    assert_close(to_np(out), ro, torch.float32, "out")
    assert_close(to_np(lse), rl, torch.float32, "lse")


def test_whole_sequence_chunk_is_bitwise_the_prefill():
    # with Lq = Lk the chunked call is the ordinary prefill
    q, k, v, cu = synth.random_case(8, (700, 1300), 8, 2, 128, torch.bfloat16)
    a, la = prefill_gpu(q, k, v, cu, 512, 200, 1e6)
    b, lb = prefill_kv_gpu(q, k, v, cu, cu, 512, 200, 1e6)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_chunks_reassemble_the_prefill():
    # causal attention of the last rows does not depend on how the sequence
    # was cut, as long as G comes from the full length: run the prefill once,
    # then the same rows as two chunks against the full key set
    q, k, v, cu = synth.random_case(9, (1500,), 8, 2, 128, torch.bfloat16)
    full, lf = prefill_gpu(q, k, v, cu, 400, 150, 1e6)
    for lo in (0, 333, 1000, 1499):
        cu_q = torch.tensor([0, 1500 - lo], dtype=torch.int32)
        o, l_ = prefill_kv_gpu(q[lo:].contiguous(), k, v, cu_q, cu, 400, 150, 1e6)
        err = (o.float() - full[lo:].float()).abs()
        assert err.max().item() < 2e-2 and err.mean().item() < 2e-3, lo
        assert (l_ - lf[:, lo:]).abs().max().item() < 2e-3, lo


def test_one_token_chunk_matches_decode():
    J = jl()
    dev = torch.device("cuda:0")
    L, Hq, Hkv = 2345, 16, 2
    q, k, v, cu_q, cu_k = chunk_case(13, (1,), (L,), Hq, Hkv)
    a, la = prefill_kv_gpu(q, k, v, cu_q, cu_k, 600, 200, 1e6)
    kc, vc = k.view(1, L, Hkv, 128).to(dev), v.view(1, L, Hkv, 128).to(dev)
    b, lb = J.jl_bifocal_decode(q.to(dev), kc, vc, torch.tensor([L], dtype=torch.int32, device=dev), L,
                                600, 200, 1e6, lse=torch.empty(1, Hq, device=dev))
    torch.cuda.synchronize()
    err = (a.float() - b.float()).abs()
    assert err.max().item() < 2e-2
    assert (la.view(-1) - lb.view(-1)).abs().max().item() < 2e-3
