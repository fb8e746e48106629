"""C-ABI library checks that need no GPU: it loads, exports every function
include/jetlong.h declares, computes G like the oracle, and rejects bad
arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from zero_shot_rope_b200 import build, jetlong
    build.build()  # no-op when the library is current
    return jetlong


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(jl_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    jl = _lib()
    names = declared_functions()
    assert {"jl_group_size", "jl_bifocal_prefill", "jl_bifocal_decode"} <= set(names)
    raw = ctypes.CDLL(jl.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_group_size_matches_oracle_bit_exactly():
    jl = _lib()
    for w in (1, 3, 256, 4096, 32768):
        for L in list(range(0, 3000)) + [131071, 131072, 131073, 1 << 20, (1 << 31) - 1]:
            assert jl.jl_group_size(L, w) == oracle.group_size(L, w)


def test_group_size_rejects_bad_arguments():
    jl = _lib()
    for L, w in [(-1, 10), (5, 0), (5, -3)]:
        with pytest.raises(jl.JetLongError) as e:
            jl.jl_group_size(L, w)
        assert e.value.status == jl.JL_ERR_INVALID_ARG
    g = jl.lib().jl_group_size(10, 3, None)
    assert g == jl.JL_ERR_INVALID_ARG


def _prefill_raw(jl, **kw):
    args = dict(q=1 << 12, k=1 << 12, v=1 << 12, out=1 << 12, lse=None, cu=1 << 12, batch=1, T=16,
                maxL=16, Hq=4, Hkv=2, D=128, w_pre=8, w0=4, theta=1e4, dtype=jl.JL_BF16, flags=0,
                ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    P = ctypes.c_void_p
    return jl.lib().jl_bifocal_prefill(
        P(args["q"]), P(args["k"]), P(args["v"]), P(args["out"]), P(args["lse"]), P(args["cu"]),
        args["batch"], args["T"], args["maxL"], args["Hq"], args["Hkv"], args["D"], args["w_pre"],
        args["w0"], args["theta"], args["dtype"], args["flags"], P(args["ws"]), args["ws_bytes"],
        P(args["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), "JL_ERR_INVALID_ARG"),
    (dict(cu=None), "JL_ERR_INVALID_ARG"),
    (dict(Hq=3, Hkv=2), "JL_ERR_INVALID_ARG"),
    (dict(Hkv=0), "JL_ERR_INVALID_ARG"),
    (dict(D=96), "JL_ERR_UNSUPPORTED"),
    (dict(w_pre=0), "JL_ERR_INVALID_ARG"),
    (dict(w0=-1), "JL_ERR_INVALID_ARG"),
    (dict(theta=0.0), "JL_ERR_INVALID_ARG"),
    (dict(theta=float("nan")), "JL_ERR_INVALID_ARG"),
    (dict(dtype=7), "JL_ERR_INVALID_ARG"),
    (dict(flags=0x80), "JL_ERR_INVALID_ARG"),
    (dict(q=(1 << 12) + 2), "JL_ERR_INVALID_ARG"),
    (dict(maxL=0), "JL_ERR_INVALID_ARG"),
    (dict(maxL=17), "JL_ERR_INVALID_ARG"),
    (dict(batch=-1), "JL_ERR_INVALID_ARG"),
    (dict(batch=70000, T=70000, maxL=1), "JL_ERR_UNSUPPORTED"),
    (dict(Hq=70000, Hkv=1), "JL_ERR_UNSUPPORTED"),    # grid y extent (heads) above 65535
    (dict(ws=None, ws_bytes=0), "JL_ERR_WORKSPACE"),
    (dict(ws=(1 << 20) + 16, ws_bytes=1 << 30), "JL_ERR_WORKSPACE"),
])
def test_prefill_rejects_bad_arguments_before_launch(kw, status):
    jl = _lib()
    s = _prefill_raw(jl, **kw)
    assert jl.status_string(s) == status, jl.last_error()
    assert jl.last_error()


def test_prefill_empty_batch_is_a_no_op():
    jl = _lib()
    assert _prefill_raw(jl, batch=0) == jl.JL_OK
    assert _prefill_raw(jl, T=0, maxL=0) == jl.JL_OK


def _decode_raw(jl, **kw):
    args = dict(q=1 << 12, kc=1 << 12, vc=1 << 12, sl=1 << 12, B=1, cap=64, maxL=64, Hq=8, Hkv=2, D=128,
                w_pre=16, w0=8, theta=1e6, out=1 << 12, lse=None, ws=1 << 20, ws_bytes=1 << 30,
                dtype=jl.JL_BF16, flags=0, stream=None)
    args.update(kw)
    P = ctypes.c_void_p
    return jl.lib().jl_bifocal_decode(
        P(args["q"]), P(args["kc"]), P(args["vc"]), P(args["sl"]), args["B"], args["cap"], args["maxL"],
        args["Hq"], args["Hkv"], args["D"], args["w_pre"], args["w0"], args["theta"], P(args["out"]),
        P(args["lse"]), P(args["ws"]), args["ws_bytes"], args["dtype"], args["flags"], P(args["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), "JL_ERR_INVALID_ARG"),
    (dict(sl=None), "JL_ERR_INVALID_ARG"),
    (dict(Hq=24, Hkv=2), "JL_ERR_UNSUPPORTED"),
    (dict(Hq=32, Hkv=2), "JL_ERR_UNSUPPORTED"),
    (dict(D=80), "JL_ERR_UNSUPPORTED"),
    (dict(maxL=65), "JL_ERR_INVALID_ARG"),
    (dict(cap=0), "JL_ERR_INVALID_ARG"),
    (dict(flags=0x2), "JL_ERR_INVALID_ARG"),
    (dict(ws=None), "JL_ERR_WORKSPACE"),
    (dict(ws_bytes=16), "JL_ERR_WORKSPACE"),
    (dict(ws=(1 << 20) + 64), "JL_ERR_WORKSPACE"),
    (dict(w_pre=0), "JL_ERR_INVALID_ARG"),
    (dict(B=70000), "JL_ERR_UNSUPPORTED"),
    (dict(Hq=70000, Hkv=70000), "JL_ERR_UNSUPPORTED"),  # grid y extent (kv heads) above 65535
])
def test_decode_rejects_bad_arguments_before_launch(kw, status):
    jl = _lib()
    s = _decode_raw(jl, **kw)
    assert jl.status_string(s) == status, jl.last_error()


def test_workspace_sizes_are_consistent():
    jl = _lib()
    assert jl.jl_bifocal_decode_workspace_size(1, 32, 8, 128, 131327) > 0
    small = jl.jl_bifocal_decode_workspace_size(1, 32, 8, 128, 1024)
    big = jl.jl_bifocal_decode_workspace_size(4, 32, 8, 128, 1024)
    assert big >= small > 0
    import torch
    assert jl.jl_bifocal_prefill_workspace_size(1, 1024, 2, 1, 64, torch.float32) == 0
    # the product path needs only the 256-byte error word; the pre-rotation
    # ablation also holds the grouped keys (one K-sized buffer)
    assert jl.jl_bifocal_prefill_workspace_size(1, 1024, 32, 8, 128, torch.bfloat16) == 256
    assert jl.jl_bifocal_prefill_workspace_size(1, 1024, 32, 8, 128, torch.bfloat16,
                                                jl.JL_FLAG_PREROTATE_K) >= 256 + 1024 * 8 * 128 * 2


def _prefill_kv_raw(jl, **kw):
    args = dict(q=1 << 12, k=1 << 12, v=1 << 12, out=1 << 12, lse=None, cuq=1 << 12, cuk=1 << 12, batch=1,
                Tq=16, Tk=40, maxL=16, Hq=4, Hkv=2, D=128, w_pre=8, w0=4, window=0, theta=1e4,
                dtype=jl.JL_BF16, flags=0, ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    P = ctypes.c_void_p
    return jl.lib().jl_bifocal_prefill_kv(
        P(args["q"]), P(args["k"]), P(args["v"]), P(args["out"]), P(args["lse"]), P(args["cuq"]),
        P(args["cuk"]), args["batch"], args["Tq"], args["Tk"], args["maxL"], args["Hq"], args["Hkv"],
        args["D"], args["w_pre"], args["w0"], args["window"], args["theta"], args["dtype"], args["flags"],
        P(args["ws"]), args["ws_bytes"], P(args["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(cuk=None), "JL_ERR_INVALID_ARG"),
    (dict(cuq=None), "JL_ERR_INVALID_ARG"),
    (dict(Tk=15), "JL_ERR_INVALID_ARG"),          # fewer keys than queries
    (dict(Tk=-1), "JL_ERR_INVALID_ARG"),
    (dict(maxL=17), "JL_ERR_INVALID_ARG"),
    (dict(k=(1 << 12) + 8), "JL_ERR_INVALID_ARG"),
    (dict(window=-1), "JL_ERR_INVALID_ARG"),
    (dict(ws=None, ws_bytes=0), "JL_ERR_WORKSPACE"),  # sized by the key count
])
def test_prefill_kv_rejects_bad_arguments_before_launch(kw, status):
    jl = _lib()
    s = _prefill_kv_raw(jl, **kw)
    assert jl.status_string(s) == status, jl.last_error()


def test_prefill_kv_empty_queries_is_a_no_op():
    jl = _lib()
    assert _prefill_kv_raw(jl, Tq=0, maxL=0) == jl.JL_OK
    assert _prefill_kv_raw(jl, batch=0) == jl.JL_OK


def test_decode_window_rejects_a_negative_window_and_validates_like_decode():
    jl = _lib()
    P = ctypes.c_void_p

    def call(window, **kw):
        a = dict(q=1 << 12, kc=1 << 12, vc=1 << 12, sl=1 << 12, ws=1 << 20, ws_bytes=1 << 30, D=128)
        a.update(kw)
        return jl.lib().jl_bifocal_decode_window(
            P(a["q"]), P(a["kc"]), P(a["vc"]), P(a["sl"]), 1, 64, 64, 8, 2, a["D"], 16, 8, window, 1e6,
            P(1 << 12), P(None), P(a["ws"]), a["ws_bytes"], jl.JL_BF16, 0, P(None))

    assert jl.status_string(call(-1)) == "JL_ERR_INVALID_ARG"
    assert jl.status_string(call(16, q=None)) == "JL_ERR_INVALID_ARG"
    assert jl.status_string(call(16, D=80)) == "JL_ERR_UNSUPPORTED"
    assert jl.status_string(call(16, ws=None)) == "JL_ERR_WORKSPACE"


@pytest.mark.parametrize("B,Hq,Hkv,D", [(1, 32, 8, 128), (3, 16, 4, 128), (64, 32, 8, 128), (2, 8, 8, 64)])
def test_decode_workspace_covers_every_shorter_plan(B, Hq, Hkv, D):
    # a sliding window plans its splits over fewer keys than max_seqlen: the
    # workspace for max_seqlen must cover every such plan, i.e. be monotone
    jl = _lib()
    lens = sorted(set(list(range(1, 20000, 13)) + [2304, 2305, 131072]))
    sizes = [jl.jl_bifocal_decode_workspace_size(B, Hq, Hkv, D, L) for L in lens]
    assert all(x > 0 for x in sizes)
    assert all(b >= a for a, b in zip(sizes, sizes[1:]))


def test_library_never_reaches_the_oracle():
    # the product path (package sources and the CUDA library) neither imports
    # nor calls the CPU oracle: there is no CPU fallback through it
    pkg = os.path.join(ROOT, "zero_shot_rope_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", txt, flags=re.M), fn
                assert "bifocal_attention(" not in txt or fn.endswith((".cu", ".cuh")), fn


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the behaviour without a GPU")
def test_calls_fail_loudly_without_a_gpu():
    # no device: a valid call reports a CUDA error instead of computing
    # anything on the host (there is no CPU fallback)
    jl = _lib()
    status = _prefill_raw(jl, ws=1 << 20, ws_bytes=1 << 30)
    assert jl.status_string(status) == "JL_ERR_CUDA"
    assert jl.last_error()
    status = _decode_raw(jl)
    assert jl.status_string(status) == "JL_ERR_CUDA"
