#!/usr/bin/env python
"""Benchmark of Dynamic Bifocal RoPE attention on B200.

One step = one bifocal causal prefill of a 131072-token sequence (32 query / 8
KV heads, head_dim 128, w_pretrained 32768 so G = 4, w0 4096, bf16) followed
by the 256 decode steps of the decode workload (a 131072..131327-token
standard-RoPE cache, G recomputed every step: 4, then 5).  Inputs are seeded
synthetic tensors already resident in HBM; every input is larger than L2, so
no flush is needed between iterations.

metric / value: prefill TFLOP/s, algorithmic FLOPs 4 * D * Hq * sum L(L+1)/2
(causal QK^T + PV only) over the prefill's device time.  The decode part is
reported under "decode" (us/token and HBM GB/s, K+V bytes 2 * L * Hkv * D * 2
per step).  The overheads over plain causal attention come from bifocal and
plain steps run alternately after the timed region, so both see the same
clocks.

python bench.py --gpus N --steps K --warmup W [--impl reference]
Under torchrun (N > 1) every rank runs an independent replica ("replicas
only": the path has no exchange step); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from zero_shot_rope_b200 import synth  # noqa: E402

METRIC = "bifocal prefill TFLOP/s @128K (frac of bf16 peak); decode µs/tok + HBM GB/s"
PREFILL = "prefill_128k_g4"
DECODE = "decode_128k"


def prefill_flops(w) -> float:
    D, Hq = w.head_dim, w.n_q_heads
    return float(sum(4.0 * D * Hq * L * (L + 1) / 2 for L in w.seqlens))


def rows_flops(w, rows) -> float:
    # algorithmic FLOPs of the given query rows (positions) over all heads
    return float(sum(4.0 * w.head_dim * w.n_q_heads * (int(r) + 1) for r in rows))


def decode_bytes(w, L) -> int:
    return 2 * L * w.n_kv_heads * w.head_dim * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_traffic(name):
    """DRAM bytes per launch from the committed ncu summary, valid only while
    the kernel source is unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(name)
    if not d:
        return None
    h = hashlib.sha256()
    for src in d["sources"]:
        path = os.path.join(ROOT, src)
        if not os.path.exists(path):
            return None
        with open(path, "rb") as f:
            h.update(f.read())
    return d["bytes_per_launch"] if h.hexdigest()[:16] == d["source_sha"] else None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = os.path.join("/tmp", f"jl_clocks_{os.getpid()}.csv")
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                if self.uuid and self.uuid.replace("GPU-", "") not in parts[1]:
                    continue
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def oracle_sample_rows(w, n, seed):
    rng = np.random.default_rng(seed)
    L = w.seqlens[0]
    return np.sort(rng.choice(np.arange(w.w0, L), size=n, replace=False))


def cpu_oracle(w, q, k, v, cu, rows):
    import oracle
    from threadpoolctl import threadpool_info

    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    t0 = time.perf_counter()
    oracle.bifocal_attention(q, k, v, cu, w.w_pretrained, w.w0, w.rope_theta, rows=rows)
    dt = time.perf_counter() - t0
    return dt, threads


def run_reference(args, world, rank):
    """Reference arm: the fp64 CPU oracle as it stands, on a bounded sample."""
    if rank != 0:
        return
    w = synth.WORKLOADS[PREFILL]
    q, k, v, cu = synth.prefill_inputs(w)
    n_rows = args.ref_rows
    times = []
    threads = 1
    for s in range(args.warmup + args.steps):
        rows = oracle_sample_rows(w, n_rows, seed=s)
        dt, threads = cpu_oracle(w, q, k, v, cu, rows)
        if s >= args.warmup:
            times.append((dt, rows_flops(w, rows)))
    tot_t = sum(t for t, _ in times)
    tot_f = sum(f for _, f in times)
    value = tot_f / tot_t / 1e12
    sample = f"{n_rows} query rows x {w.n_q_heads} heads of the {w.seqlens[0]}-token prefill per step (fp64 oracle)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "seq_len": w.seqlens[0],
                                        "heads": f"{w.n_q_heads}/{w.n_kv_heads}", "head_dim": w.head_dim,
                                        "G": 4, "w0": w.w0},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def measure_extras(jl, dev, peaks, clocks_cls, local):
    """Further workloads, timed after the headline's timed region (so the
    headline is unchanged): the other prefill configurations, head_dim 64,
    the pre-rotation ablation, a chunk of new tokens against a long cache, and
    the decode pair bifocal / plain with the SM clock sampled while it runs."""
    burst = peaks["bf16_tflops"]
    ex = {}

    def prefill_case(seqlens, hq, hkv, D, w_pre, w0, theta, q=None, k=None, v=None, flags=0, reps=3):
        if q is None:
            q, k, v, _ = synth.random_case(3, seqlens, hq, hkv, D, torch.bfloat16)
            q, k, v = q.to(dev), k.to(dev), v.to(dev)
        cu = [0]
        for L in seqlens:
            cu.append(cu[-1] + L)
        cu = torch.tensor(cu, dtype=torch.int32, device=dev)
        out = torch.empty_like(q)
        ws = torch.zeros(jl.jl_bifocal_prefill_workspace_size(len(seqlens), q.shape[0], hq, hkv, D, torch.bfloat16,
                                                              flags), dtype=torch.uint8, device=dev)
        ms = _median_ms(lambda: jl.jl_bifocal_prefill(q, k, v, cu, max(seqlens), w_pre, w0, theta, out=out,
                                                      flags=flags, workspace=ws), reps)
        flops = sum(4.0 * D * hq * L * (L + 1) / 2 for L in seqlens)
        tf = flops / ms / 1e9
        return {"ms": ms, "tflops": tf, "frac_of_burst_peak": tf / burst, "error_word": int(ws[:4].view(torch.int32).item())}

    for key, name in (("prefill_c2", "prefill_32k_g1"), ("prefill_c5", "varlen_4seq")):
        w = synth.WORKLOADS[name]
        q, k, v, _ = synth.prefill_inputs(w)
        ex[key] = prefill_case(w.seqlens, w.n_q_heads, w.n_kv_heads, w.head_dim, w.w_pretrained, w.w0,
                               w.rope_theta, q.to(dev), k.to(dev), v.to(dev))
        ex[key]["workload"] = name
        del q, k, v
    ex["prefill_d64"] = prefill_case((131072,), 32, 8, 64, 32768, 4096, 1e6)
    ex["prefill_d64"]["workload"] = "131072 tokens, 32/8 heads, head_dim 64, G 4, w0 4096"
    w = synth.WORKLOADS["prefill_128k_g4"]
    q, k, v, _ = synth.prefill_inputs(w)
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    ex["prefill_c3_prerotate_ablation"] = prefill_case(w.seqlens, 32, 8, 128, w.w_pretrained, w.w0, w.rope_theta,
                                                       q, k, v, flags=jl.JL_FLAG_PREROTATE_K)
    # a chunk of 512 new tokens at the end of the 131072-token sequence
    L, n = w.seqlens[0], 512
    qc = q[L - n:].contiguous()
    oc = torch.empty_like(qc)
    cuq = torch.tensor([0, n], dtype=torch.int32, device=dev)
    cuk = torch.tensor([0, L], dtype=torch.int32, device=dev)
    fl_chunk = sum(4.0 * 128 * 32 * (L - n + i + 1) for i in range(n))
    chunk = {"workload": "512 new tokens against a 131072-token cache, 32/8 heads, G 4"}
    for lab, fl in (("in_tile", 0), ("prerotate_ablation", jl.JL_FLAG_PREROTATE_K)):
        ws = torch.zeros(jl.jl_bifocal_prefill_workspace_size(1, L, 32, 8, 128, torch.bfloat16, fl),
                         dtype=torch.uint8, device=dev)
        ms = _median_ms(lambda: jl.jl_bifocal_prefill_kv(qc, k, v, cuq, cuk, n, w.w_pretrained, w.w0, w.rope_theta,
                                                         out=oc, flags=fl, workspace=ws), 20)
        chunk[lab] = {"us": ms * 1e3, "tflops": fl_chunk / ms / 1e9}
    ex["prefill_chunk512"] = chunk
    del q, k, v, qc, oc
    # decode at head_dim 64, and the 128K decode pair with the clock sampled
    for D in (64, 128):
        g = torch.Generator().manual_seed(5)
        L = 131072
        kc = torch.randn(1, L, 8, D, generator=g).to(torch.bfloat16).to(dev)
        vc = torch.randn(1, L, 8, D, generator=g).to(torch.bfloat16).to(dev)
        qd = torch.randn(1, 32, D, generator=g).to(torch.bfloat16).to(dev)
        sl = torch.tensor([L], dtype=torch.int32, device=dev)
        od = torch.empty_like(qd)
        ws = torch.zeros(jl.jl_bifocal_decode_workspace_size(1, 32, 8, D, L), dtype=torch.uint8, device=dev)
        clk = clocks_cls(local)
        clk.start()
        times = {0: [], jl.JL_FLAG_PLAIN_CAUSAL: []}
        for _ in range(5):
            for fl in times:
                times[fl].append(_median_ms(lambda: [jl.jl_bifocal_decode(qd, kc, vc, sl, L, 32768, 4096, 1e6,
                                                                          out=od, flags=fl, workspace=ws)
                                                     for _ in range(50)], 1) * 1e3 / 50)
        c = clk.stop()
        bi, pl = statistics.median(times[0]), statistics.median(times[jl.JL_FLAG_PLAIN_CAUSAL])
        gbs = 2 * L * 8 * D * 2 / bi / 1e3
        mhz = c.get("sm_mhz")
        ex[f"decode_d{D}_pair"] = {
            "workload": f"one decode step at L = {L}, 32/8 heads, head_dim {D}, G 4 (50 back-to-back calls)",
            "us_per_tok": bi, "hbm_gbs": gbs, "frac": gbs / peaks["hbm_gbs"], "plain_us_per_tok": pl,
            "overhead_vs_plain": bi / pl - 1, "sm_mhz_median": mhz,
            "kcycles_per_tok": bi * mhz / 1e3 if mhz else None,
            "plain_kcycles_per_tok": pl * mhz / 1e3 if mhz else None, "clock_reasons": c.get("reasons")}
        del kc, vc
    # batched decode with ragged lengths (uniform in [cap / 8, cap]), 32/8
    # heads, head_dim 128; 20 steps replayed from a CUDA graph
    for B, cap in ((8, 32768), (32, 8192)):
        gd = torch.Generator(device=dev).manual_seed(B)
        lens = torch.randint(cap // 8, cap + 1, (B,), generator=torch.Generator().manual_seed(B)).tolist()
        kc = torch.randn(B, cap, 8, 128, generator=gd, device=dev, dtype=torch.bfloat16)
        vc = torch.randn(B, cap, 8, 128, generator=gd, device=dev, dtype=torch.bfloat16)
        qd = torch.randn(B, 32, 128, generator=gd, device=dev, dtype=torch.bfloat16)
        sl = torch.tensor(lens, dtype=torch.int32, device=dev)
        od = torch.empty_like(qd)
        ws = torch.zeros(jl.jl_bifocal_decode_workspace_size(B, 32, 8, 128, cap), dtype=torch.uint8, device=dev)
        res = {}
        for lab, fl in (("bifocal", 0), ("plain", jl.JL_FLAG_PLAIN_CAUSAL)):
            call = lambda: jl.jl_bifocal_decode(qd, kc, vc, sl, cap, 4096, 1024, 1e6, out=od, flags=fl,
                                                workspace=ws)
            s_ = torch.cuda.Stream()
            s_.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s_):
                call()
            torch.cuda.current_stream().wait_stream(s_)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(20):
                    call()
            res[lab] = statistics.median(_median_ms(graph.replay, 1) for _ in range(5)) * 1e3 / 20
            del graph
        nbytes = sum(2 * L * 8 * 128 * 2 for L in lens)
        gbs = nbytes / res["bifocal"] / 1e3
        ex[f"decode_ragged_b{B}"] = {
            "workload": f"one decode step of {B} sequences, lengths uniform in [{cap // 8}, {cap}] (seeded), "
                        "32/8 heads, head_dim 128, w_pre 4096, w0 1024 (20 steps from a CUDA graph)",
            "us_per_step": res["bifocal"], "hbm_gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
            "plain_us_per_step": res["plain"], "plain_hbm_gbs": nbytes / res["plain"] / 1e3}
        del kc, vc
    return ex


def run_ours(args, world, rank, local):
    from zero_shot_rope_b200 import jetlong as jl

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wp = synth.WORKLOADS[PREFILL]
    wd = synth.WORKLOADS[DECODE]
    peaks, peak_kind = load_peaks()

    # ---- inputs (seeded CPU draws, then resident in HBM)
    q_h, k_h, v_h, cu_h = synth.prefill_inputs(wp)
    q, k, v, cu = q_h.to(dev), k_h.to(dev), v_h.to(dev), cu_h.to(dev)
    out = torch.empty_like(q)
    T = wp.total_tokens
    ws_p = torch.empty(jl.jl_bifocal_prefill_workspace_size(1, T, wp.n_q_heads, wp.n_kv_heads, wp.head_dim),
                       dtype=torch.uint8, device=dev)
    kc_h, vc_h = synth.decode_cache(wd)
    kc, vc = kc_h.to(dev), vc_h.to(dev)
    n_dec = args.decode_steps
    cap = kc.shape[1]
    qd_h = torch.stack([synth.decode_query(wd, t) for t in range(n_dec)])  # [n, 1, Hq, D]
    qd = qd_h.to(dev)
    od = torch.empty_like(qd)
    lens = torch.tensor([wd.seqlens[0] + t for t in range(n_dec)], dtype=torch.int32, device=dev)
    ws_d = torch.empty(jl.jl_bifocal_decode_workspace_size(1, wd.n_q_heads, wd.n_kv_heads, wd.head_dim, cap),
                       dtype=torch.uint8, device=dev)
    pf_flops = prefill_flops(wp)
    dec_bytes = sum(decode_bytes(wd, wd.seqlens[0] + t) for t in range(n_dec))

    def prefill(flags=0):
        jl.jl_bifocal_prefill(q, k, v, cu, T, wp.w_pretrained, wp.w0, wp.rope_theta, out=out, flags=flags,
                              workspace=ws_p)

    def decode_all(flags=0):
        for t in range(n_dec):
            jl.jl_bifocal_decode(qd[t], kc, vc, lens[t:t + 1], cap, wd.w_pretrained, wd.w0, wd.rope_theta,
                                 out=od[t], flags=flags, workspace=ws_d)

    # ---- warm-up
    for _ in range(args.warmup):
        prefill()
        decode_all()
    torch.cuda.synchronize()

    # ---- timed region: K steps, device-resident inputs
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for s in range(args.steps):
        ev[s][0].record()
        prefill()
        ev[s][1].record()
        decode_all()
        ev[s][2].record()
    t_end.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    pre_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    pre_ms_max = max_over_ranks(sum(pre_ms), world, dev)
    dec_ms_max = max_over_ranks(sum(dec_ms), world, dev)
    value = world * args.steps * pf_flops / (pre_ms_max * 1e-3) / 1e12
    launches_per_step = 1 + 2 * n_dec  # prefill: attention; decode: partial + combine

    # ---- plain-causal comparison (outside the timed region): bifocal and
    # plain steps alternate so both see the same clocks (a long step runs
    # under the power cap), and the overheads come from these pairs
    pair_ms = {0: [], jl.JL_FLAG_PLAIN_CAUSAL: []}
    for _ in range(2):
        for fl in (0, jl.JL_FLAG_PLAIN_CAUSAL):
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record()
            prefill(fl)
            e1.record()
            decode_all(fl)
            e2.record()
            torch.cuda.synchronize()
            pair_ms[fl].append((e0.elapsed_time(e1), e1.elapsed_time(e2)))
    pair_pre = {fl: statistics.mean(x[0] for x in v) for fl, v in pair_ms.items()}
    pair_dec = {fl: statistics.mean(x[1] for x in v) for fl, v in pair_ms.items()}
    plain_pre_ms, plain_dec_ms = pair_pre[jl.JL_FLAG_PLAIN_CAUSAL], pair_dec[jl.JL_FLAG_PLAIN_CAUSAL]

    extras = None
    if not args.no_extras:
        extras = measure_extras(jl, dev, peaks, ClockSampler, local)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        outp = torch.empty(q_h.shape, dtype=q_h.dtype).pin_memory()
        qdp = qd_h.pin_memory()
        odp = torch.empty(qd_h.shape, dtype=qd_h.dtype).pin_memory()
        h2d = (qp.numel() + kp.numel() + vp.numel()) * 2 + qdp.numel() * 2
        d2h = outp.numel() * 2 + odp.numel() * 2

        def e2e_step():
            q.copy_(qp, non_blocking=True)
            k.copy_(kp, non_blocking=True)
            v.copy_(vp, non_blocking=True)
            prefill()
            outp.copy_(out, non_blocking=True)
            for t in range(n_dec):
                qd[t].copy_(qdp[t], non_blocking=True)
                jl.jl_bifocal_decode(qd[t], kc, vc, lens[t:t + 1], cap, wd.w_pretrained, wd.w0, wd.rope_theta,
                                     out=od[t], workspace=ws_d)
                odp[t].copy_(od[t], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        pre_e2e = []
        for _ in range(args.steps):
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            b0.record()
            q.copy_(qp, non_blocking=True)
            k.copy_(kp, non_blocking=True)
            v.copy_(vp, non_blocking=True)
            prefill()
            outp.copy_(out, non_blocking=True)
            b1.record()
            pre_e2e.append((b0, b1))
            for t in range(n_dec):
                qd[t].copy_(qdp[t], non_blocking=True)
                jl.jl_bifocal_decode(qd[t], kc, vc, lens[t:t + 1], cap, wd.w_pretrained, wd.w0, wd.rope_theta,
                                     out=od[t], workspace=ws_d)
                odp[t].copy_(od[t], non_blocking=True)
        a1.record()
        torch.cuda.synchronize()
        barrier(world)
        pre_e2e_ms = max_over_ranks(sum(b0.elapsed_time(b1) for b0, b1 in pre_e2e), world, dev)
        e2e = {"value": world * args.steps * pf_flops / (pre_e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": max_over_ranks(a0.elapsed_time(a1), world, dev) / args.steps}

    # ---- CPU baseline (rank 0, N = 1 only): the oracle on a bounded sample
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = oracle_sample_rows(wp, args.cpu_rows, seed=123)
        dt, threads = cpu_oracle(wp, q_h, k_h, v_h, cu_h, rows)
        cpu = {"value": rows_flops(wp, rows) / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{len(rows)} random query rows x {wp.n_q_heads} heads of the {wp.seqlens[0]}-token "
                         f"prefill (fp64 NumPy oracle, {dt:.1f} s)"}
        # the decode leg beside it: one full decode step (L = 131072) in the oracle
        import oracle
        L0 = int(wd.seqlens[0])
        t0 = time.perf_counter()
        oracle.bifocal_decode(qd_h[0], kc_h[:, :L0], vc_h[:, :L0], [L0], wd.w_pretrained, wd.w0, wd.rope_theta)
        dt_d = time.perf_counter() - t0
        cpu["decode"] = {"us_per_tok": dt_d * 1e6, "gbs": 2 * L0 * wd.n_kv_heads * wd.head_dim * 2 / dt_d / 1e9,
                         "sample": f"one decode step at L = {L0} (fp64 NumPy oracle)"}

    if rank != 0:
        return
    mean_pre_ms = statistics.mean(pre_ms)
    achieved = pf_flops / (mean_pre_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    dec_us_tok = 1e3 * statistics.mean(dec_ms) / n_dec
    dec_gbs = dec_bytes / (statistics.mean(dec_ms) * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{wp.name} + {wd.name}", "seq_len": wp.seqlens[0],
                   "heads": f"{wp.n_q_heads}/{wp.n_kv_heads}", "head_dim": wp.head_dim,
                   "w_pretrained": wp.w_pretrained, "G": 4, "w0": wp.w0, "rope_theta": wp.rope_theta,
                   "decode_steps": n_dec, "decode_L": [wd.seqlens[0], wd.seqlens[0] + n_dec - 1],
                   "parallelism": f"replicas x{world}", "l2": "inputs larger than L2 (no flush needed)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": kernel_traffic("bifocal_prefill2_kernel"),
                     "kernel": "bifocal_prefill2_kernel (two heads per CTA, in-tile key correction)",
                     "peak_kind": f"{peak_kind} bf16 burst (cuBLAS 8192^3, best of 10)",
                     "frac_of_sustained_peak": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])},
        "decode": {"us_per_tok": dec_us_tok, "hbm_gbs": dec_gbs, "hbm_peak_gbs": peaks["hbm_gbs"],
                   "frac": dec_gbs / peaks["hbm_gbs"], "bytes_per_step": dec_bytes / n_dec,
                   "traffic": kernel_traffic("decode_tc_kernel"),
                   "paired_us_per_tok": 1e3 * pair_dec[0] / n_dec,
                   "plain_us_per_tok": 1e3 * plain_dec_ms / n_dec,
                   "overhead_vs_plain": (pair_dec[0] - plain_dec_ms) / plain_dec_ms},
        "prefill": {"ms": mean_pre_ms, "paired_ms": pair_pre[0], "plain_ms": plain_pre_ms,
                    "plain_tflops": pf_flops / (plain_pre_ms * 1e-3) / 1e12,
                    "bifocal_over_plain_time": pair_pre[0] / plain_pre_ms},
        "clocks": clk,
        "extras": extras,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def _median_ms(fn, reps):
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def _case_inputs(args, dev):
    seqlens = tuple(args.seqlens) if args.seqlens else (args.seqlen,)
    q, k, v, cu = synth.random_case(3, seqlens, args.hq, args.hkv, args.head_dim, torch.bfloat16)
    return seqlens, q.to(dev), k.to(dev), v.to(dev), cu.to(dev)


def run_case(args):
    """--only: run one call --reps times through the C ABI (a profiler driver:
    the first call is a warm-up to skip with ``ncu -s``), then print its
    median time."""
    from zero_shot_rope_b200 import build
    from zero_shot_rope_b200 import jetlong as jl

    build.build()
    dev = torch.device("cuda:0")
    flags = (jl.JL_FLAG_PLAIN_CAUSAL if args.plain else 0) | (jl.JL_FLAG_PREROTATE_K if args.prerotate else 0)
    D = args.head_dim
    if args.only in ("prefill", "chunk"):
        seqlens, q, k, v, cu = _case_inputs(args, dev)
        if args.only == "prefill":
            out = torch.empty_like(q)
            ws = torch.zeros(jl.jl_bifocal_prefill_workspace_size(len(seqlens), q.shape[0], args.hq, args.hkv, D,
                                                                  torch.bfloat16, flags), dtype=torch.uint8, device=dev)
            fn = lambda: jl.jl_bifocal_prefill(q, k, v, cu, max(seqlens), args.w_pre, args.w0, 1e6, out=out,  # noqa
                                               flags=flags, workspace=ws)
            flops = sum(4.0 * D * args.hq * L * (L + 1) / 2 for L in seqlens)
        else:
            L, n = seqlens[0], args.chunk
            qc = q[L - n:].contiguous()
            out = torch.empty_like(qc)
            cuq = torch.tensor([0, n], dtype=torch.int32, device=dev)
            ws = torch.zeros(jl.jl_bifocal_prefill_workspace_size(1, L, args.hq, args.hkv, D, torch.bfloat16, flags),
                             dtype=torch.uint8, device=dev)
            fn = lambda: jl.jl_bifocal_prefill_kv(qc, k, v, cuq, cu, n, args.w_pre, args.w0, 1e6, out=out,  # noqa
                                                  flags=flags, workspace=ws)
            flops = sum(4.0 * D * args.hq * (L - n + i + 1) for i in range(n))
        for _ in range(args.reps):
            fn()
        torch.cuda.synchronize()
        ms = _median_ms(fn, 3) if args.time else None
        print(json.dumps({"case": args.only, "seqlens": list(seqlens), "heads": f"{args.hq}/{args.hkv}",
                          "head_dim": D, "flags": flags, "error_word": int(ws[:4].view(torch.int32).item()),
                          "ms": ms, "tflops": flops / ms / 1e9 if ms else None}), flush=True)
    else:
        g = torch.Generator().manual_seed(5)
        cap = args.seqlen
        kc = torch.randn(1, cap, args.hkv, D, generator=g).to(torch.bfloat16).to(dev)
        vc = torch.randn(1, cap, args.hkv, D, generator=g).to(torch.bfloat16).to(dev)
        qd = torch.randn(1, args.hq, D, generator=g).to(torch.bfloat16).to(dev)
        sl = torch.tensor([cap], dtype=torch.int32, device=dev)
        out = torch.empty_like(qd)
        ws = torch.zeros(jl.jl_bifocal_decode_workspace_size(1, args.hq, args.hkv, D, cap), dtype=torch.uint8,
                         device=dev)
        fn = lambda: jl.jl_bifocal_decode(qd, kc, vc, sl, cap, args.w_pre, args.w0, 1e6, out=out,  # noqa
                                          flags=flags & jl.JL_FLAG_PLAIN_CAUSAL, workspace=ws)
        for _ in range(args.reps):
            fn()
        torch.cuda.synchronize()
        us = _median_ms(lambda: [fn() for _ in range(20)], 3) * 1e3 / 20 if args.time else None
        print(json.dumps({"case": "decode", "L": cap, "heads": f"{args.hq}/{args.hkv}", "head_dim": D,
                          "flags": flags, "us_per_call": us,
                          "gbs": 2 * cap * args.hkv * D * 2 / us / 1e3 if us else None}), flush=True)


def run_sweep_w0(args):
    """--sweep-w0: prefill TFLOP/s and decode us/token across local-window
    sizes, each beside the plain-causal call on the same inputs (markdown)."""
    from zero_shot_rope_b200 import build
    from zero_shot_rope_b200 import jetlong as jl

    build.build()
    dev = torch.device("cuda:0")
    L, Hq, Hkv, D = args.seqlen, args.hq, args.hkv, args.head_dim
    _, q, k, v, cu = _case_inputs(args, dev)
    out = torch.empty_like(q)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    flops = 4.0 * D * Hq * L * (L + 1) / 2
    kc, vc = k.view(1, L, Hkv, D), v.view(1, L, Hkv, D)
    qd = q[L - 1:L].contiguous()
    od = torch.empty_like(qd)
    sl = torch.tensor([L], dtype=torch.int32, device=dev)
    wsd = torch.zeros(jl.jl_bifocal_decode_workspace_size(1, Hq, Hkv, D, L), dtype=torch.uint8, device=dev)
    G = jl.jl_group_size(L, args.w_pre)

    def prefill(w0, flags):
        return lambda: jl.jl_bifocal_prefill(q, k, v, cu, L, args.w_pre, w0, 1e6, out=out, flags=flags,
                                             workspace=ws)

    def decode(w0, flags, n=20):
        return lambda: [jl.jl_bifocal_decode(qd, kc, vc, sl, L, args.w_pre, w0, 1e6, out=od, flags=flags,
                                             workspace=wsd) for _ in range(n)]

    plain_ms = _median_ms(prefill(0, jl.JL_FLAG_PLAIN_CAUSAL), args.reps)
    plain_us = _median_ms(decode(0, jl.JL_FLAG_PLAIN_CAUSAL), args.reps) * 1e3 / 20
    print(f"L = {L}, {Hq}/{Hkv} heads, D = {D}, w_pre = {args.w_pre} (G = {G}), bf16")
    print()
    print("| w0 | prefill ms | prefill TFLOP/s | vs plain | decode us/token | vs plain |")
    print("|---:|---:|---:|---:|---:|---:|")
    print(f"| plain | {plain_ms:.2f} | {flops / plain_ms / 1e9:.1f} | 1.000 | {plain_us:.1f} | 1.000 |")
    for w0 in args.sweep_w0:
        ms = _median_ms(prefill(w0, 0), args.reps)
        us = _median_ms(decode(w0, 0), args.reps) * 1e3 / 20
        print(f"| {w0} | {ms:.2f} | {flops / ms / 1e9:.1f} | {ms / plain_ms:.3f} | {us:.1f} | {us / plain_us:.3f} |",
              flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--cpu-rows", type=int, default=24)
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the extra workloads after the timed region")
    # one call, for profilers (--only) and the w0 sweep (--sweep-w0)
    ap.add_argument("--only", choices=["prefill", "chunk", "decode"])
    ap.add_argument("--sweep-w0", type=int, nargs="+")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--time", action="store_true", help="--only: also print the median time of 3 more calls")
    ap.add_argument("--seqlen", type=int, default=32768)
    ap.add_argument("--seqlens", type=int, nargs="+", help="--only prefill: packed sequence lengths")
    ap.add_argument("--chunk", type=int, default=512, help="--only chunk: new tokens at the end of --seqlen")
    ap.add_argument("--hq", type=int, default=32)
    ap.add_argument("--hkv", type=int, default=8)
    ap.add_argument("--head-dim", type=int, default=128)
    ap.add_argument("--w-pre", type=int, default=32768)
    ap.add_argument("--w0", type=int, default=4096)
    ap.add_argument("--plain", action="store_true")
    ap.add_argument("--prerotate", action="store_true", help="ablation: grouped keys from a pre-pass")
    args = ap.parse_args()
    if args.only:
        run_case(args)
        return
    if args.sweep_w0:
        run_sweep_w0(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            from zero_shot_rope_b200 import build

            if rank == 0:
                build.build()
            barrier(world)
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
