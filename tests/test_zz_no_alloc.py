"""The allocation-free decode entry point, jl_bifocal_decode_noalloc.

Callers such as plugins inside a runtime that owns all device memory, or
latency-critical generation loops that must not allocate, get the same decode
with the library's fixed in-image scratch instead of a caller workspace.  These
tests call it through the C ABI and compare it with jl_bifocal_decode (which
takes a caller workspace) on two calls in a row.  Both entry points launch the
same kernels with the same split plan, so the results must be identical bit
for bit.  The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from tests.gpu_util import jl


def _case(seed, B, cap, Hq, Hkv, D):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, cap, Hkv, D, generator=g).to(torch.bfloat16)
    return q, kc, vc


def _noalloc_raw(J, **kw):
    a = dict(q=1 << 12, kc=1 << 12, vc=1 << 12, sl=1 << 12, B=1, cap=64, maxL=64, Hq=8, Hkv=2, D=128,
             w_pre=16, w0=8, theta=1e6, out=1 << 12, lse=None, dtype=J.JL_BF16, flags=0)
    a.update(kw)
    P = ctypes.c_void_p
    return J.lib().jl_bifocal_decode_noalloc(P(a["q"]), P(a["kc"]), P(a["vc"]), P(a["sl"]), a["B"], a["cap"],
                                             a["maxL"], a["Hq"], a["Hkv"], a["D"], a["w_pre"], a["w0"],
                                             a["theta"], P(a["out"]), P(a["lse"]), a["dtype"], a["flags"], None)


def test_noalloc_rejects_a_decode_larger_than_its_scratch():
    J = jl()
    # 2048 sequences x 32 heads need more partials than the fixed scratch holds
    need = J.jl_bifocal_decode_workspace_size(2048, 32, 8, 128, 4096)
    assert need > J.JL_DECODE_NOALLOC_SCRATCH_BYTES
    s = _noalloc_raw(J, B=2048, cap=4096, maxL=4096, Hq=32, Hkv=8, w_pre=1024, w0=64)
    assert J.status_string(s) == "JL_ERR_WORKSPACE"
    assert "scratch" in J.last_error()


@pytest.mark.parametrize("kw,status", [
    (dict(D=256), "JL_ERR_UNSUPPORTED"),        # checked before the scratch size
    (dict(B=70000), "JL_ERR_UNSUPPORTED"),
    (dict(q=None), "JL_ERR_INVALID_ARG"),
    (dict(Hq=24, Hkv=2), "JL_ERR_UNSUPPORTED"),
    (dict(maxL=65), "JL_ERR_INVALID_ARG"),
])
def test_noalloc_checks_arguments_like_the_workspace_decode(kw, status):
    J = jl()
    assert J.status_string(_noalloc_raw(J, **kw)) == status, J.last_error()


def test_noalloc_empty_batch_is_a_no_op():
    J = jl()
    assert _noalloc_raw(J, B=0) == J.JL_OK


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    J = jl()
    dev = torch.device("cuda:0")
    # two calls in a row with different shapes and lengths (G = 4, then 5)
    cases = [(_case(1, 2, 3000, 32, 8, 128), [2000, 2999], 3000, 750, 256),
             (_case(2, 1, 5000, 16, 4, 128), [4001], 5000, 1000, 64)]
    for (q, kc, vc), lens, cap, w_pre, w0 in cases:
        qd, kd, vd = q.to(dev), kc.to(dev), vc.to(dev)
        sl = torch.tensor(lens, dtype=torch.int32, device=dev)
        ref_o, ref_l = J.jl_bifocal_decode(qd, kd, vd, sl, cap, w_pre, w0, 1e6,
                                           lse=torch.empty(len(lens), q.shape[1], device=dev))
        out = torch.full_like(qd, float("nan"))
        lse = torch.full((len(lens), q.shape[1]), float("nan"), device=dev)
        J.jl_bifocal_decode_noalloc(qd, kd, vd, sl, cap, w_pre, w0, 1e6, out, lse=lse)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o), "noalloc out differs from the workspace decode"
        assert torch.equal(lse, ref_l), "noalloc lse differs from the workspace decode"
        # no bounded wait ran out in the kernels
        assert J.jl_bifocal_decode_noalloc_error() == 0
