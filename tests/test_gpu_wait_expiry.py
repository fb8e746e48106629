"""Failure detection without a GPU fault: the kernels' bounded waits.

Every pipeline wait in the prefill and decode kernels gives up after a time
limit, sets a bit of the call's error word, stops the kernel's other roles,
lets its own copies and tensor-core work finish, frees TMEM and returns.  The
test hook jl_debug_set_wait_limit shortens that limit (nothing is withheld:
every load and product is issued as usual) so that waits run out; the calls
must then return, report the timeout in the error word, and leave the context
usable: the next calls with the default limit match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from zero_shot_rope_b200 import synth
from tests.gpu_util import assert_close, jl, to_np

pytestmark = pytest.mark.gpu

PREFILL_TIMEOUT_BITS = 1 | 2 | 4 | 32   # producer, MMA issuer, softmax, key correction
DECODE_TIMEOUT_BITS = 16               # tensor-core decode


def _prefill(J, q, k, v, cu, L, flags=0):
    dev = torch.device("cuda:0")
    Hq, Hkv = q.shape[1], k.shape[1]
    ws = torch.zeros(J.jl_bifocal_prefill_workspace_size(1, q.shape[0], Hq, Hkv, q.shape[2], torch.bfloat16, flags),
                     dtype=torch.uint8, device=dev)
    out, _ = J.jl_bifocal_prefill(q.to(dev), k.to(dev), v.to(dev), cu.to(dev), L, 1024, 256, 1e6, flags=flags,
                                  workspace=ws)
    torch.cuda.synchronize()
    return out, int(ws[:4].view(torch.int32).item())


def _decode(J, q, kc, vc, L):
    dev = torch.device("cuda:0")
    B, Hq, D = q.shape
    cap, Hkv = kc.shape[1], kc.shape[2]
    ws = torch.zeros(J.jl_bifocal_decode_workspace_size(B, Hq, Hkv, D, cap), dtype=torch.uint8, device=dev)
    out, _ = J.jl_bifocal_decode(q.to(dev), kc.to(dev), vc.to(dev),
                                 torch.tensor([L] * B, dtype=torch.int32, device=dev), cap, 1024, 256, 1e6,
                                 workspace=ws)
    torch.cuda.synchronize()
    return out, int(ws[:4].view(torch.int32).item())


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (3, 1)])   # the two-head and the one-head prefill kernel
def test_prefill_wait_expiry_is_reported_and_the_next_call_is_correct(Hq, Hkv):
    J = jl()
    L = 6000
    q, k, v, cu = synth.random_case(91, (L,), Hq, Hkv, 128, torch.bfloat16)
    lib = J.lib()
    try:
        assert lib.jl_debug_set_wait_limit(1) == 0
        _, err = _prefill(J, q, k, v, cu, L)
    finally:
        assert lib.jl_debug_set_wait_limit(0) == 0
    assert err != 0 and (err & ~PREFILL_TIMEOUT_BITS) == 0, hex(err)
    out, err = _prefill(J, q, k, v, cu, L)
    assert err == 0
    rows = np.arange(0, L, 97)
    ro, _ = oracle.bifocal_attention(q, k, v, cu, 1024, 256, 1e6, rows=rows)
    assert_close(to_np(out)[rows], ro, torch.bfloat16, "after recovery")


@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (64, torch.bfloat16)])
def test_decode_wait_expiry_is_reported_and_the_next_call_is_correct(D, dtype):
    # the tensor-core decode (bf16); the fp32 CUDA-core decode issues its loads
    # so far ahead that its waits complete within their first hardware probe,
    # so a shortened limit does not reach it
    J = jl()
    g = torch.Generator().manual_seed(92)
    B, L, Hq, Hkv = 2, 20000, 16, 4
    q = torch.randn(B, Hq, D, generator=g).to(dtype)
    kc = torch.randn(B, L, Hkv, D, generator=g).to(dtype)
    vc = torch.randn(B, L, Hkv, D, generator=g).to(dtype)
    lib = J.lib()
    try:
        assert lib.jl_debug_set_wait_limit(1) == 0
        _, err = _decode(J, q, kc, vc, L)
    finally:
        assert lib.jl_debug_set_wait_limit(0) == 0
    assert err != 0 and (err & ~DECODE_TIMEOUT_BITS) == 0, hex(err)
    out, err = _decode(J, q, kc, vc, L)
    assert err == 0
    ro, _ = oracle.bifocal_decode(q, kc, vc, [L] * B, 1024, 256, 1e6)
    assert_close(to_np(out), ro, dtype, "after recovery")
