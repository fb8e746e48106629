"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
binding and compare with the fp64 oracle under the stated tolerances."""
import numpy as np
import torch

# tolerances: bf16 max-abs 2e-2 and mean-abs 2e-3; fp32 max-abs 1e-4
TOL = {torch.bfloat16: (2e-2, 2e-3), torch.float32: (1e-4, 1e-5)}


def jl():
    from zero_shot_rope_b200 import build, jetlong
    build.build()
    return jetlong


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, want, dtype, what=""):
    max_tol, mean_tol = TOL[dtype]
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    finite = np.isfinite(want)
    assert np.array_equal(finite, np.isfinite(got)), f"{what}: non-finite pattern differs"
    if not finite.any():
        return 0.0, 0.0
    err = np.abs(got[finite] - want[finite])
    mx, mn = float(err.max()), float(err.mean())
    assert mx <= max_tol and mn <= mean_tol, f"{what}: max-abs {mx:.3e} mean-abs {mn:.3e}"
    return mx, mn


def prefill_gpu(q, k, v, cu, w_pre, w0, theta, flags=0, with_lse=True):
    J = jl()
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    cud = cu.to(dev)
    T, Hq, _ = q.shape
    lens = (cu[1:] - cu[:-1]).tolist()
    lse = torch.full((Hq, T), float("nan"), dtype=torch.float32, device=dev) if with_lse else None
    out = torch.full_like(qd, float("nan"))
    out, lse = J.jl_bifocal_prefill(qd, kd, vd, cud, max(max(lens), 1), w_pre, w0, theta, out=out,
                                    lse=lse, flags=flags)
    torch.cuda.synchronize()
    return out, lse


def sample_rows(lengths, w0, G_list, n_edge=256, n_random=512, seed=0):
    """Stratified sample of global rows, per sequence: the first and last
    ``n_edge`` rows, rows around w0, around the first multiples of G and of
    the 128-row tile, around the quarter points, and ``n_random`` seeded
    random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    start = 0
    for L, G in zip(lengths, G_list):
        if L == 0:
            continue
        local = set(range(min(L, n_edge))) | set(range(max(0, L - n_edge), L))
        marks = [w0, 128, 256, L // 2] + [m * G for m in (1, 2, 3, 4, 1000)] + [(L // 4) * t for t in (1, 2, 3)]
        marks += [128 * m for m in (33, 100, 511)]
        for c in marks:
            for d in (-1, 0, 1):
                if 0 <= c + d < L:
                    local.add(c + d)
        local |= set(int(x) for x in rng.integers(0, L, size=n_random))
        rows |= {start + r for r in local}
        start += L
    return np.array(sorted(rows), dtype=np.int64)


def oracle_rows_threaded(fn, rows, *args, threads=None, **kw):
    """Evaluate the prefill oracle ``fn(*args, rows=part, **kw)`` on parts of
    ``rows`` in a pool of threads (NumPy releases the GIL in its large array
    operations; one BLAS thread each) and reassemble (out, lse)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits

    n = threads or max(1, min(32, (os.cpu_count() or 2) - 1))
    parts = [p for p in np.array_split(np.asarray(rows), min(n, max(1, len(rows) // 32))) if len(p)]
    with threadpool_limits(1), ThreadPoolExecutor(len(parts)) as ex:
        res = list(ex.map(lambda part: fn(*args, rows=part, **kw), parts))
    return np.concatenate([r[0] for r in res], axis=0), np.concatenate([r[1] for r in res], axis=1)
