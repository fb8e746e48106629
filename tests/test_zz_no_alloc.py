"""The allocation-free decode entry point, jl_bifocal_decode_noalloc.

Callers such as plugins inside a runtime that owns all device memory, or
latency-critical generation loops that must not allocate, get the same decode
with the library's fixed in-image scratch instead of a caller workspace.  These
tests call it through the C ABI and compare it with jl_bifocal_decode (which
takes a caller workspace) on two calls in a row.  The file is named so that
pytest collects it last.
"""
import pytest
import torch

from tests.gpu_util import assert_close, jl


def _case(seed, B, L, cap, Hq, Hkv, D):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    return q, kc, vc


def test_noalloc_rejects_a_decode_larger_than_its_scratch():
    J = jl()
    # 2048 sequences x 32 heads need more partials than the fixed scratch holds
    need = J.jl_bifocal_decode_workspace_size(2048, 32, 8, 128, 4096)
    assert need > J.JL_DECODE_NOALLOC_SCRATCH_BYTES
    import ctypes
    P = ctypes.c_void_p
    s = J.lib().jl_bifocal_decode_noalloc(P(1 << 12), P(1 << 12), P(1 << 12), P(1 << 12), 2048, 4096, 4096, 32, 8,
                                          128, 1024, 64, 1e6, P(1 << 12), None, J.JL_BF16, 0, None)
    assert J.status_string(s) == "JL_ERR_WORKSPACE"
    assert "scratch" in J.last_error()


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    J = jl()
    dev = torch.device("cuda:0")
    # two calls in a row with different shapes and lengths (G = 4, then 5)
    cases = [(_case(1, 2, None, 3000, 32, 8, 128), [2000, 2999], 3000, 750, 256),
             (_case(2, 1, None, 5000, 16, 4, 128), [4001], 5000, 1000, 64)]
    for (q, kc, vc), lens, cap, w_pre, w0 in cases:
        qd, kd, vd = q.to(dev), kc.to(dev), vc.to(dev)
        sl = torch.tensor(lens, dtype=torch.int32, device=dev)
        ref_o, ref_l = J.jl_bifocal_decode(qd, kd, vd, sl, cap, w_pre, w0, 1e6,
                                           lse=torch.empty(len(lens), q.shape[1], device=dev))
        out = torch.full_like(qd, float("nan"))
        lse = torch.full((len(lens), q.shape[1]), float("nan"), device=dev)
        J.jl_bifocal_decode_noalloc(qd, kd, vd, sl, cap, w_pre, w0, 1e6, out, lse=lse)
        torch.cuda.synchronize()
        assert_close(out.double().cpu().numpy(), ref_o.double().cpu().numpy(), torch.bfloat16, "noalloc out")
        assert_close(lse.double().cpu().numpy(), ref_l.double().cpu().numpy(), torch.bfloat16, "noalloc lse")
