"""Prefill parity on the GPU: the CUDA path (through the C ABI) against the
fp64 oracle, element by element, plus bitwise invariants between modes."""
import numpy as np
import pytest
import torch

import oracle
from zero_shot_rope_b200 import synth
from tests.gpu_util import assert_close, jl, oracle_rows_threaded, prefill_gpu, sample_rows, to_np

pytestmark = pytest.mark.gpu


def test_tiny_fp32_workload_full():
    w = synth.WORKLOADS["tiny_fp32"]
    q, k, v, cu = synth.prefill_inputs(w)
    out, lse = prefill_gpu(q, k, v, cu, w.w_pretrained, w.w0, w.rope_theta)
    ro, rl = oracle.bifocal_attention(q, k, v, cu, w.w_pretrained, w.w0, w.rope_theta)
    assert_close(to_np(out), ro, torch.float32, "out")
    assert_close(to_np(lse), rl, torch.float32, "lse")


CASES = [
    # (seqlens, Hq, Hkv, w_pre, w0)
    ((1,), 2, 1, 1, 0),
    ((100,), 4, 2, 40, 16),          # one partial tile, G = 3
    ((128,), 4, 1, 64, 64),          # exactly one tile, G = 2
    ((129,), 2, 2, 64, 1),           # tail tile of one row
    ((300,), 8, 2, 100, 128),        # G = 3, tile-aligned window
    ((777,), 4, 4, 160, 200),        # G = 5, window not tile-aligned
    ((1500,), 4, 1, 512, 0),         # w0 = 0: every pair grouped
    ((1024,), 4, 2, 256, 2000),      # window longer than the sequence
    ((1024,), 4, 2, 4096, 64),       # G = 1
    ((64, 0, 513, 1, 260), 8, 2, 128, 96),  # varlen with an empty sequence
]


@pytest.mark.parametrize("seqlens,Hq,Hkv,w_pre,w0", CASES)
@pytest.mark.parametrize("kernel", ["tensor", "prerotated", "simt"])
def test_bf16_cases_full(seqlens, Hq, Hkv, w_pre, w0, kernel):
    # "tensor": grouped keys rotated in the tile (the product path);
    # "prerotated": the ablation that writes them in a pre-pass
    J = jl()
    q, k, v, cu = synth.random_case(sum(seqlens) + 7 * Hq + w0, seqlens, Hq, Hkv, 128, torch.bfloat16)
    flags = {"tensor": 0, "prerotated": J.JL_FLAG_PREROTATE_K, "simt": J.JL_FLAG_SIMT}[kernel]
    out, lse = prefill_gpu(q, k, v, cu, w_pre, w0, 1e6, flags=flags)
    ro, rl = oracle.bifocal_attention(q, k, v, cu, w_pre, w0, 1e6)
    assert_close(to_np(out), ro, torch.bfloat16, "out")
    assert_close(to_np(lse), rl, torch.bfloat16, "lse")


@pytest.mark.parametrize("seqlens,w_pre,w0", [((2048,), 4096, 300), ((700, 1300), 1300, 128)])
def test_group_one_is_bitwise_plain_causal(seqlens, w_pre, w0):
    # The pages: the base model is reproduced exactly inside its native context.
    J = jl()
    q, k, v, cu = synth.random_case(11, seqlens, 8, 2, 128, torch.bfloat16)
    a, la = prefill_gpu(q, k, v, cu, w_pre, w0, 1e6)
    b, lb = prefill_gpu(q, k, v, cu, w_pre, w0, 1e6, flags=J.JL_FLAG_PLAIN_CAUSAL)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_group_one_is_bitwise_plain_causal_at_full_32k_shape():
    # The same property on the 32K workload itself (16 query / 8 KV heads,
    # w_pretrained 32768 so G = 1, w0 4096): every output and LSE element of
    # the bifocal call equals the plain-causal call bit for bit.
    J = jl()
    w = synth.WORKLOADS["prefill_32k_g1"]
    assert oracle.group_size(w.seqlens[0], w.w_pretrained) == 1
    q, k, v, cu = synth.prefill_inputs(w)
    a, la = prefill_gpu(q, k, v, cu, w.w_pretrained, w.w0, w.rope_theta)
    b, lb = prefill_gpu(q, k, v, cu, w.w_pretrained, w.w0, w.rope_theta, flags=J.JL_FLAG_PLAIN_CAUSAL)
    assert torch.equal(a, b) and torch.equal(la, lb)
    assert torch.isfinite(a.float()).all()


def test_tensor_kernel_matches_simt_kernel():
    J = jl()
    q, k, v, cu = synth.random_case(5, (3000,), 8, 2, 128, torch.bfloat16)
    a, la = prefill_gpu(q, k, v, cu, 1024, 333, 1e6)
    b, lb = prefill_gpu(q, k, v, cu, 1024, 333, 1e6, flags=J.JL_FLAG_SIMT)
    err = (a.float() - b.float()).abs()
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3
    ro, _ = oracle.bifocal_attention(q, k, v, cu, 1024, 333, 1e6, rows=np.arange(0, 3000, 97))
    assert_close(to_np(a)[np.arange(0, 3000, 97)], ro, torch.bfloat16, "tensor vs oracle")


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (3, 1)])
def test_kernel_error_word_stays_clear_in_a_256_byte_workspace(Hq, Hkv):
    # the in-tile key correction needs no K-sized scratch: the default
    # workspace is the 256-byte error word alone
    J = jl()
    q, k, v, cu = synth.random_case(3, (1000,), Hq, Hkv, 128, torch.bfloat16)
    dev = torch.device("cuda:0")
    assert J.jl_bifocal_prefill_workspace_size(1, 1000, Hq, Hkv, 128) == 256
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    out, _ = J.jl_bifocal_prefill(q.to(dev), k.to(dev), v.to(dev), cu.to(dev), 1000, 300, 200, 1e6, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    ro, _ = oracle.bifocal_attention(q, k, v, cu, 300, 200, 1e6, rows=np.arange(0, 1000, 37))
    assert_close(to_np(out)[np.arange(0, 1000, 37)], ro, torch.bfloat16, "out")


@pytest.mark.parametrize("name", ["prefill_32k_g1", "prefill_128k_g4", "varlen_4seq"])
def test_full_size_workload_sampled_rows(name):
    """Full-size workload in the benchmark's launch configuration; the oracle
    evaluates a stratified sample of rows for every head (per sequence: the
    first and last 256 rows, rows at the window and tile and group
    boundaries, 512 seeded random rows)."""
    w = synth.WORKLOADS[name]
    q, k, v, cu = synth.prefill_inputs(w)
    out, lse = prefill_gpu(q, k, v, cu, w.w_pretrained, w.w0, w.rope_theta)
    Gs = [oracle.group_size(L, w.w_pretrained) for L in w.seqlens]
    rows = sample_rows(w.seqlens, w.w0, Gs)
    ro, rl = oracle_rows_threaded(oracle.bifocal_attention, rows, q, k, v, cu, w.w_pretrained, w.w0,
                                  w.rope_theta)
    got = to_np(out)[rows]
    assert_close(got, ro, torch.bfloat16, name + " out")
    assert_close(to_np(lse)[:, rows], rl, torch.bfloat16, name + " lse")
    err = np.abs(got - ro)
    # the relative L2 error is a sharper diagnostic than max-abs on small outputs
    assert np.linalg.norm(got - ro) / np.linalg.norm(ro) < 1e-2
    if max(Gs) > 1:
        # discrimination: the grouped branch changes the result by much more
        # than the kernel's error (a kernel that ignored grouping would fail)
        far = rows[::4]
        po, _ = oracle_rows_threaded(oracle.bifocal_attention, far, q, k, v, cu, w.w_pretrained, w.w0,
                                     w.rope_theta, plain=True)
        diff = np.abs(po - ro[::4]).mean()
        assert diff > 5 * err.mean(), (diff, err.mean())


@pytest.mark.parametrize("w_pre,G", [(7000, 3), (3000, 7)])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (3, 1)])
def test_key_correction_over_many_tiles_with_carries(w_pre, G, Hq, Hkv):
    # 128 is not a multiple of G = 3 or 7, so the key correction's per-tile
    # step takes both of its values; over ~150 grouped key tiles the carried
    # fp32 rotation must stay on the oracle (both kernels; sampled rows,
    # every head)
    L, w0 = 20000, 512
    assert oracle.group_size(L, w_pre) == G
    q, k, v, cu = synth.random_case(100 + G, (L,), Hq, Hkv, 128, torch.bfloat16)
    out, lse = prefill_gpu(q, k, v, cu, w_pre, w0, 1e6)
    rows = sample_rows([L], w0, [G], n_edge=64, n_random=128, seed=G)
    ro, rl = oracle_rows_threaded(oracle.bifocal_attention, rows, q, k, v, cu, w_pre, w0, 1e6)
    got = to_np(out)[rows]
    assert_close(got, ro, torch.bfloat16, "out")
    assert_close(to_np(lse)[:, rows], rl, torch.bfloat16, "lse")
    assert np.linalg.norm(got - ro) / np.linalg.norm(ro) < 1e-2


def test_planted_needles_peaked_attention():
    # A key planted so that its score with one query is large under the
    # method's own geometry (aligned with the query after the correction
    # rotation for remote pairs, aligned as is inside the window) makes that
    # row's attention peak on it: a wrong correction angle or a pair routed
    # to the wrong branch moves most of the probability mass.  The plain
    # causal oracle does not find the remote needles, so the rows also
    # discriminate between the two modes.
    L, Hq, Hkv, D, w_pre, w0, theta = 4096, 8, 2, 128, 1024, 256, 1e6   # G = 4
    G = oracle.group_size(L, w_pre)
    rng = np.random.default_rng(4242)
    pos = np.arange(L)[:, None]
    qt = oracle.rope_rotate(rng.standard_normal((L, Hq, D)), pos, theta)
    kt = oracle.rope_rotate(rng.standard_normal((L, Hkv, D)), pos, theta)
    v = rng.standard_normal((L, Hkv, D))
    needles = []  # (row, distance)
    for n, d in enumerate([300, 1000, 2500, 4000, 5, 200]):
        i = L - 1 - 7 * n
        j = i - d
        for kv in range(Hkv):
            qi = qt[i, kv * (Hq // Hkv)]
            if d >= w0:   # grouped score <R(delta_i) q, R(delta_j) k> large
                shift = oracle.correction_shift(i, G) - oracle.correction_shift(j, G)
                kt[j, kv] = 1.5 * oracle.rope_rotate(qi, shift, theta)
            else:
                kt[j, kv] = 1.5 * qi
            v[j, kv] = 4.0
        needles.append((i, d))
    q = torch.from_numpy(qt).to(torch.bfloat16)
    k = torch.from_numpy(kt).to(torch.bfloat16)
    vv = torch.from_numpy(v).to(torch.bfloat16)
    cu = torch.tensor([0, L], dtype=torch.int32)
    rows = np.array(sorted(i for i, _ in needles))
    out, lse = prefill_gpu(q, k, vv, cu, w_pre, w0, theta)
    ro, rl = oracle.bifocal_attention(q, k, vv, cu, w_pre, w0, theta, rows=rows)
    assert_close(to_np(out)[rows], ro, torch.bfloat16, "needle rows")
    assert_close(to_np(lse)[:, rows], rl, torch.bfloat16, "needle lse")
    planted = [kv * (Hq // Hkv) for kv in range(Hkv)]
    assert np.all(ro[:, planted, :].mean(axis=-1) > 3.9)   # the needle value is 4
    po, _ = oracle.bifocal_attention(q, k, vv, cu, w_pre, w0, theta, rows=rows, plain=True)
    remote = [n for n, r in enumerate(rows) if dict(needles)[r] >= w0]
    assert po[remote][:, planted, :].mean() < 2.0


D64_CASES = [
    # (seqlens, Hq, Hkv, w_pre, w0): even GQA groups run the two-head kernel,
    # odd ones the one-head kernel
    ((100,), 4, 2, 40, 16),
    ((129,), 2, 1, 64, 1),
    ((777,), 8, 2, 160, 200),
    ((1500,), 4, 2, 512, 0),
    ((64, 0, 513, 1, 260), 8, 4, 128, 96),
    ((1024,), 16, 8, 4096, 64),          # G = 1
    ((600,), 4, 4, 100, 50),             # group of 1: one-head kernel
    ((300, 513), 3, 1, 128, 64),         # group of 3
]


@pytest.mark.parametrize("seqlens,Hq,Hkv,w_pre,w0", D64_CASES)
@pytest.mark.parametrize("prerotated", [False, True])
def test_head_dim_64_bf16_full(seqlens, Hq, Hkv, w_pre, w0, prerotated):
    J = jl()
    q, k, v, cu = synth.random_case(sum(seqlens) + 64 + w0, seqlens, Hq, Hkv, 64, torch.bfloat16)
    out, lse = prefill_gpu(q, k, v, cu, w_pre, w0, 1e4, flags=J.JL_FLAG_PREROTATE_K if prerotated else 0)
    ro, rl = oracle.bifocal_attention(q, k, v, cu, w_pre, w0, 1e4)
    assert_close(to_np(out), ro, torch.bfloat16, "out")
    assert_close(to_np(lse), rl, torch.bfloat16, "lse")


def test_head_dim_64_tensor_matches_simt_and_chunks():
    J = jl()
    q, k, v, cu = synth.random_case(17, (2000,), 8, 2, 64, torch.bfloat16)
    a, _ = prefill_gpu(q, k, v, cu, 512, 300, 1e4)
    b, _ = prefill_gpu(q, k, v, cu, 512, 300, 1e4, flags=J.JL_FLAG_SIMT)
    err = (a.float() - b.float()).abs()
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3
    # a chunk of the last 700 tokens against the whole sequence, with a window
    dev = torch.device("cuda:0")
    cu_q = torch.tensor([0, 700], dtype=torch.int32)
    o2, l2 = J.jl_bifocal_prefill_kv(q[1300:].contiguous().to(dev), k.to(dev), v.to(dev), cu_q.to(dev),
                                     cu.to(dev), 700, 512, 300, 1e4, window=900,
                                     lse=torch.empty(8, 700, device=dev))
    torch.cuda.synchronize()
    ro, rl = oracle.bifocal_attention_kv(q[1300:], k, v, cu_q, cu, 512, 300, 1e4, window=900)
    assert_close(to_np(o2), ro, torch.bfloat16, "chunk out")
    assert_close(to_np(l2), rl, torch.bfloat16, "chunk lse")


def test_full_length_head_dim_64_sampled_rows():
    # 32K tokens, 32/8 heads, D = 64, G = 4 (the two-head kernel at head_dim 64)
    L, Hq, Hkv, w_pre, w0 = 32768, 32, 8, 8192, 4096
    q, k, v, cu = synth.random_case(64, (L,), Hq, Hkv, 64, torch.bfloat16)
    out, lse = prefill_gpu(q, k, v, cu, w_pre, w0, 1e6)
    rows = sample_rows([L], w0, [oracle.group_size(L, w_pre)], seed=64)
    ro, rl = oracle_rows_threaded(oracle.bifocal_attention, rows, q, k, v, cu, w_pre, w0, 1e6)
    got = to_np(out)[rows]
    assert_close(got, ro, torch.bfloat16, "out")
    assert_close(to_np(lse)[:, rows], rl, torch.bfloat16, "lse")
    assert np.linalg.norm(got - ro) / np.linalg.norm(ro) < 1e-2
