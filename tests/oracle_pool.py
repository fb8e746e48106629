"""Oracle evaluations in a pool of spawned CPU processes (test infrastructure).

The fp64 oracle is single-threaded in its elementwise work, so the large
parity cases spread their independent pieces (decode steps, groups of query
rows) over the host's cores.  The pool is started with ``spawn``: a process
forked after the test process has initialised CUDA can hang.  Workers rebuild
the seeded synthetic inputs themselves (zero_shot_rope_b200.synth draws random
numbers only) and call the oracle as it stands.
"""
from __future__ import annotations

import multiprocessing as mp
import os

_CACHE = {}


def _init():
    from threadpoolctl import threadpool_limits

    threadpool_limits(1)  # one BLAS thread per worker: the pool supplies the parallelism


def n_workers(cap: int = 32) -> int:
    return max(1, min(cap, (os.cpu_count() or 2) - 1))


def pool(n: int | None = None):
    return mp.get_context("spawn").Pool(n or n_workers(), initializer=_init)


def _decode_cache(name):
    if name not in _CACHE:
        from zero_shot_rope_b200 import synth

        w = synth.WORKLOADS[name]
        _CACHE.clear()
        _CACHE[name] = (w,) + tuple(synth.decode_cache(w))
    return _CACHE[name]


def decode_step(args):
    """Oracle output of decode step ``step`` of workload ``name``:
    (step, out [B, Hq, D], lse [B, Hq], plain-mode out)."""
    import oracle
    from zero_shot_rope_b200 import synth

    name, step, with_plain = args
    w, kc, vc = _decode_cache(name)
    L = w.seqlens[0] + step
    q = synth.decode_query(w, step)
    out, lse = oracle.bifocal_decode(q, kc, vc, [L], w.w_pretrained, w.w0, w.rope_theta)
    po = None
    if with_plain:
        po, _ = oracle.bifocal_decode(q, kc, vc, [L], w.w_pretrained, w.w0, w.rope_theta, plain=True)
    return step, out, lse, po
