#!/usr/bin/env python
"""Benchmark of the packed-sequence context-parallel attention hot path on B200.

One step = the whole path on the long-context fwd+bwd workload (cp=16 virtual ranks,
T=131072 packed tokens: one 65536-token document plus lognormal short documents,
GQA 64/8, head dim 128, bf16): rank-major gather of Q, K/V and dO, the forward
attention, and the backward.  The plan (partition + tile metadata) is computed
once per layout and cached, as the method prescribes, so it is outside the timed
region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Prints one JSON line (rank 0).  `value` is unmasked attention TFLOP/s (fwd + bwd
FLOPs over the device-timed step); `e2e` is the same metric through the public
API with pinned host buffers, host<->device copies inside the timed region, on two
copy streams that overlap the kernels (each step's dO goes up during its forward,
the next step's Q/K/V during its backward; O and lse come down during the backward,
the gradients during the next step's forward).
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
N > 1 runs independent replicas (every CP rank is virtual, on one GPU).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = 5
METRIC = "unmasked attn TFLOP/s & % BF16 tensor peak (fwd/bwd); K/V gather HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=8,
                    help="end-to-end steps timed (the first upload and the last download, the pipeline's fill and drain, are spread over them)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload forward / K/V-gather measurements")
    ap.add_argument("--clocks-csv", default=None, help="where the nvidia-smi clock samples go (default: a temp file)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w, cu, seed):
    return {
        "workload": (f"long-context fwd+bwd: cp={w.cp} virtual ranks, T={w.T} packed tokens "
                     f"({len(cu) - 1} docs: one 65536-token doc + lognormal(512,1) docs, multiples of 32), "
                     f"GQA {w.hq}/{w.hkv}, head dim {w.dqk}, seed {seed}"),
        "cp": w.cp, "T": w.T, "n_docs": len(cu) - 1, "hq": w.hq, "hkv": w.hkv, "dqk": w.dqk, "dv": w.dv,
        "step": "gather Q, K/V, dO to rank-major + fwd + bwd (plan cached)",
        "l2": "inputs larger than L2 (Q and dO 2.1 GB each, K/V 268 MB each)",
        "parallelism": "replicas (all CP ranks virtual on one GPU)",
    }


def time_plan(thd, cu, cp, reps=5):
    """Host wall time (ms, median of `reps`) of thd_cp_plan for one layout: the partition and
    the tile tables, computed once per layout and cached, so never inside the step."""
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        p = thd.Plan(cu, cp)
        ts.append((time.perf_counter() - t0) * 1e3)
        p.close()
    return statistics.median(ts)


def measure_workloads(thd, syn, dev, stream, seed, peaks, iters=10, warmup=3):
    """Forward attention on the MHA (T=8192), GQA (T=32768) and expanded-MLA (T=65536)
    workloads, and the K/V-only gather on those and on the long-context workload, each
    launch timed alone with CUDA events after an L2 flush (a 256 MB write), so that no
    input is served from L2 left warm by the previous launch.  Returns one sub-object per
    workload."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    def timed(fn):
        for _ in range(warmup):
            fn()
        ms = []
        for _ in range(iters):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            ms.append(a.elapsed_time(b))
        return statistics.median(ms)

    out = {}
    for cfg in (2, 3, 4, 5):
        w = syn.WORKLOADS[cfg]
        cu = syn.cu_seqlens_of(syn.doc_lengths(cfg, seed))
        plan = thd.Plan(cu, w.cp).upload()
        g = torch.Generator(device=dev).manual_seed(seed + 1)
        k = torch.randn(w.T, w.hkv, w.dqk, device=dev, generator=g).to(torch.bfloat16)
        v = (torch.randn(w.T, w.hkv, w.dv, device=dev, generator=g) * w.v_std).to(torch.bfloat16)
        k_rm, v_rm = torch.empty_like(k), torch.empty_like(v)
        gather_ms = timed(lambda: thd.thd_kv_gather(plan, k, v, k_rm=k_rm, v_rm=v_rm))
        gather_bytes = 2 * w.T * w.hkv * (w.dqk + w.dv) * 2 + 4 * w.T
        gbs = gather_bytes / (gather_ms / 1e3) / 1e9
        rec = {"workload": (f"{w.name}: cp={w.cp}, T={w.T}, {len(cu) - 1} docs, heads {w.hq}/{w.hkv}, "
                            f"head dims {w.dqk}/{w.dv}, bf16, seed {seed}"),
               "kv_gather": {"ms": gather_ms, "gbs": gbs, "frac_of_hbm": gbs / hbm, "bytes": gather_bytes,
                             "l2": "flushed before each launch"}}
        if cfg != 5:
            q = torch.randn(w.T, w.hq, w.dqk, device=dev, generator=g).to(torch.bfloat16)
            q_rm = thd.thd_kv_gather(plan, q)
            o_rm = torch.empty(w.T, w.hq, w.dv, dtype=torch.bfloat16, device=dev)
            lse_rm = torch.empty(w.hq, w.T, dtype=torch.float32, device=dev)
            fwd_ms = timed(lambda: thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm, out=o_rm, lse=lse_rm))
            flops = plan.causal_pairs * w.hq * 2 * (w.dqk + w.dv)
            # 128 x 128 tile pairs the forward computes (its own tables: rank-major tiles,
            # position tiles for short-chunk documents)
            tile_flops = plan.n_fentries * 128 * 128 * w.hq * 2 * (w.dqk + w.dv)
            tf = flops / (fwd_ms / 1e3) / 1e12
            rec["fwd"] = {"ms": fwd_ms, "tflops": tf, "frac_of_peak": tf / burst, "flops": flops,
                          "density_ceiling": flops / tile_flops,
                          "tile_tflops": tile_flops / (fwd_ms / 1e3) / 1e12,
                          "peak_source": "bf16_tflops (burst: the launch is timed alone)",
                          "l2": "flushed before each launch"}
            del q, q_rm, o_rm, lse_rm
        torch.cuda.synchronize(dev)
        if plan.device_status() != 0:
            raise RuntimeError(f"a kernel's bounded wait gave up on {w.name}")
        out[w.name] = rec
        plan.close()
        del k, v, k_rm, v_rm
    del flush
    return out


def measure_replan(thd, syn, plan, dev, stream, seed, w):
    """Re-planning for a new batch: thd_cp_plan_update of an uploaded plan with another
    long-context layout (seed + 1), then back to this one.  A first pair of updates
    allocates the second pinned staging buffer; the pair after it is measured.
    host_ms: wall time of the call (partition and tables built on the host, copied into
    pinned staging, the copy enqueued).  copy_ms: device time of the table copy alone,
    taken with the stream held busy until the host part has returned."""
    import torch
    layouts = [syn.cu_seqlens_of(syn.doc_lengths(WORKLOAD, s_)) for s_ in (seed + 1, seed)]
    for cu in layouts:
        plan.update(cu, w.cp, stream=stream)
    res = []
    for s_, cu in zip((seed + 1, seed), layouts):
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        plan.update(cu, w.cp, stream=stream)
        host_ms = (time.perf_counter() - t0) * 1e3
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            torch.cuda._sleep(100_000_000)          # ~50 ms: the host part finishes meanwhile
        a.record(stream)
        plan.update(cu, w.cp, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        ex = plan.n_qtiles * 12 + plan.n_entries * 10 + 2 * plan.T + 2 * plan.n_qtiles + 1
        res.append({"seed": s_, "host_ms": host_ms, "copy_ms": a.elapsed_time(b), "table_bytes": 4 * ex,
                    "n_docs": len(cu) - 1, "n_entries": plan.n_entries})
    return {"new_layout": res[0], "back": res[1],
            "note": "thd_cp_plan_update on the uploaded plan: no device-wide synchronisation"}


def flop_counts(pairs, w):
    fwd = pairs * w.hq * 2 * (w.dqk + w.dv)
    bwd = pairs * w.hq * 2 * (3 * w.dqk + 2 * w.dv)
    return fwd, bwd


# ---------------------------------------------------------------- oracle (CPU) legs

def cpu_sample(w, cu, seed, n_heads):
    """A bounded sample of the workload for the oracle: the short documents, the
    first `n_heads` query heads (whole key/value groups)."""
    import numpy as np
    import torch
    from context_packed_sequence_cp_b200 import synthetic as syn
    s0 = int(cu[1])                                  # short documents follow the 65536-token one
    cu_s = (np.asarray(cu[1:], dtype=np.int64) - s0)
    T = int(cu_s[-1])
    hkv = max(1, n_heads // (w.hq // w.hkv))
    q, k, v, do = syn.make_tensors(T, n_heads, hkv, w.dqk, w.dv, torch.bfloat16, seed, with_do=True)
    pairs = int(np.sum(np.diff(cu_s) * (np.diff(cu_s) + 1) // 2))
    return cu_s, (q, k, v, do), pairs


def time_oracle_step(w, cu_s, tens, pairs, n_heads):
    from oracle import attention as A
    q, k, v, do = tens
    scale = 1.0 / math.sqrt(w.dqk)
    t0 = time.perf_counter()
    o, lse = A.attention_fwd(q, k, v, cu_s, scale)
    A.attention_bwd(q, k, v, o, lse, do, cu_s, scale)
    dt = time.perf_counter() - t0
    flops = pairs * n_heads * 2 * ((w.dqk + w.dv) + (3 * w.dqk + 2 * w.dv))
    return dt, flops


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args):
    """The fp64 oracle, as it stands, on the host cores: the reference arm."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    from context_packed_sequence_cp_b200 import synthetic as syn
    w = syn.WORKLOADS[WORKLOAD]
    cu = syn.cu_seqlens_of(syn.doc_lengths(WORKLOAD, args.seed))
    n_heads = 2
    cu_s, tens, pairs = cpu_sample(w, cu, args.seed, n_heads)
    for _ in range(args.warmup):
        time_oracle_step(w, cu_s, tens, pairs, n_heads)
    times, fl = [], 0
    for _ in range(args.steps):
        dt, fl = time_oracle_step(w, cu_s, tens, pairs, n_heads)
        times.append(dt)
    total = sum(times)
    value = fl * args.steps / total / 1e12
    sample = (f"oracle fwd+bwd (fp64 numpy) on the {len(cu_s) - 1} short documents "
              f"({int(cu_s[-1])} tokens) x {n_heads} query heads sharing one key/value head, per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, cu, args.seed),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str, path: str | None = None):
        self.bus = bus_id.lower()
        self.proc = None
        self.path = path or os.path.join(tempfile.gettempdir(), f"thdcp_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8 or self.bus[-12:] not in parts[0].lower():
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def bus_id_of(dev):
    import torch
    p = torch.cuda.get_device_properties(dev)
    return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"


def roofline_traffic(kernel_src: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the
    current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    with open(kernel_src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if d.get("source_sha256") != sha:
        return None
    return d.get("bytes_per_launch")


# ---------------------------------------------------------------- native arm

def run_native(args):
    import torch
    import context_packed_sequence_cp_b200 as thd
    from context_packed_sequence_cp_b200 import replicas
    from context_packed_sequence_cp_b200 import synthetic as syn

    info = replicas.init_from_env("nccl")
    dev = torch.device("cuda", info.local_rank)
    torch.cuda.set_device(dev)
    w = syn.WORKLOADS[WORKLOAD]
    cu = syn.cu_seqlens_of(syn.doc_lengths(WORKLOAD, args.seed))
    plan_host_ms = time_plan(thd, cu, w.cp)
    plan = thd.Plan(cu, w.cp)
    torch.cuda.synchronize(dev)
    t_up = time.perf_counter()
    plan.upload()
    torch.cuda.synchronize(dev)
    plan_upload_ms = (time.perf_counter() - t_up) * 1e3
    fwd_fl, bwd_fl = flop_counts(plan.causal_pairs, w)
    step_fl = fwd_fl + bwd_fl
    T = w.T

    g = torch.Generator(device=dev).manual_seed(args.seed + 1 + 1000 * info.rank)
    q = torch.randn(T, w.hq, w.dqk, device=dev, generator=g).to(torch.bfloat16)
    k = torch.randn(T, w.hkv, w.dqk, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(T, w.hkv, w.dv, device=dev, generator=g).to(torch.bfloat16)
    do = torch.randn(T, w.hq, w.dv, device=dev, generator=g).to(torch.bfloat16)
    q_rm, k_rm, v_rm, do_rm = (torch.empty_like(x) for x in (q, k, v, do))
    o_rm = torch.empty(T, w.hq, w.dv, dtype=torch.bfloat16, device=dev)
    lse_rm = torch.empty(w.hq, T, dtype=torch.float32, device=dev)
    dq = torch.empty(T, w.hq, w.dqk, dtype=torch.float32, device=dev)
    dk = torch.empty(T, w.hkv, w.dqk, dtype=torch.float32, device=dev)
    dv = torch.empty(T, w.hkv, w.dv, dtype=torch.float32, device=dev)
    ws = torch.empty(thd.thd_cp_attn_bwd_workspace(plan, hq=w.hq, hkv=w.hkv, dqk=w.dqk, dv=w.dv),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 7   # gather Q, gather K/V, gather dO, fwd, bwd prep, dK/dV, dQ

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        thd.thd_kv_gather(plan, q, k_rm=q_rm)
        thd.thd_kv_gather(plan, k, v, k_rm=k_rm, v_rm=v_rm)
        thd.thd_kv_gather(plan, do, k_rm=do_rm)
        if ev:
            ev[1].record(stream)
        thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm, out=o_rm, lse=lse_rm)
        if ev:
            ev[2].record(stream)
        thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq=dq, dk=dk, dv=dv, workspace=ws)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if plan.device_status() != 0:
        raise RuntimeError("a kernel's bounded wait gave up during warm-up")

    sampler = ClockSampler(bus_id_of(dev), args.clocks_csv)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    replicas.barrier(info)
    torch.cuda.synchronize(dev)
    sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    replicas.barrier(info)
    elapsed_ms = t0.elapsed_time(t1)
    max_ms = replicas.max_over_ranks(info, elapsed_ms, device=dev)
    if plan.device_status() != 0:
        raise RuntimeError("a kernel's bounded wait gave up in the timed region")

    gather_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    fwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    bwd_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps

    # ------------------------------------------------ end to end, host buffers
    e2e = None
    if args.e2e_steps > 0:
        pin = dict(pin_memory=True)
        hq_, hk_, hv_, hdo_ = (x.cpu().pin_memory() for x in (q, k, v, do))
        h_in = (hq_, hk_, hv_, hdo_)
        # Device copies of the inputs (global order) and of the gradients, two sets each:
        # step i uses set i % 2, so step i+1's inputs go up and step i's gradients come
        # down while the kernels of the neighbouring step run.  O and lse come down while
        # the backward of their own step runs.  Every step copies its own inputs to the
        # device and its results to the host; the first upload and the last download are
        # inside the timed region.
        in_sets = [tuple(torch.empty_like(x) for x in (q, k, v, do)) for _ in range(2)]
        g_sets = [tuple(torch.empty_like(x) for x in (dq, dk, dv)) for _ in range(2)]
        o_g = torch.empty_like(o_rm)
        h_out = [torch.empty(x.shape, dtype=x.dtype, **pin) for x in (o_g, lse_rm, dq, dk, dv)]
        h2d = sum(x.numel() * x.element_size() for x in h_in)
        d2h = sum(x.numel() * x.element_size() for x in h_out)
        s_up = torch.cuda.Stream(dev)
        s_down = torch.cuda.Stream(dev)

        def e2e_run(n_steps):
            ev = lambda: torch.cuda.Event()  # noqa: E731
            qkv_ready, do_ready, in_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]
            g_ready, g_out = [ev(), ev()], [ev(), ev()]
            o_out = None

            def upload(i):
                st = i % 2
                if i >= 2:
                    s_up.wait_event(in_free[st])          # gathers of step i-2 read this set
                with torch.cuda.stream(s_up):
                    for d_, h_ in zip(in_sets[st][:3], h_in[:3]):
                        d_.copy_(h_, non_blocking=True)
                    qkv_ready[st].record(s_up)
                    in_sets[st][3].copy_(h_in[3], non_blocking=True)
                    do_ready[st].record(s_up)

            begin = ev()
            begin.record(stream)
            s_up.wait_event(begin)
            s_down.wait_event(begin)
            upload(0)
            for i in range(n_steps):
                st = i % 2
                dq_in, dk_in, dv_in, ddo_in = in_sets[st]
                stream.wait_event(qkv_ready[st])
                thd.thd_kv_gather(plan, dq_in, k_rm=q_rm)
                thd.thd_kv_gather(plan, dk_in, dv_in, k_rm=k_rm, v_rm=v_rm)
                if o_out is not None:
                    stream.wait_event(o_out)              # O and lse of step i-1 are on the host
                thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm, out=o_rm, lse=lse_rm)
                thd.thd_rows_to_global(plan, o_rm, out=o_g)
                o_ready = ev()
                o_ready.record(stream)
                s_down.wait_event(o_ready)
                with torch.cuda.stream(s_down):
                    for h_, d_ in zip(h_out[:2], (o_g, lse_rm)):
                        h_.copy_(d_, non_blocking=True)
                    o_out = ev()
                    o_out.record(s_down)
                stream.wait_event(do_ready[st])
                thd.thd_kv_gather(plan, ddo_in, k_rm=do_rm)
                in_free[st].record(stream)
                if i + 1 < n_steps:
                    upload(i + 1)
                thd.thd_cp_attn_bwd(plan, q_rm, k_rm, v_rm, o_rm, lse_rm, do_rm, dq=dq, dk=dk, dv=dv, workspace=ws)
                if i >= 2:
                    stream.wait_event(g_out[st])          # gradients of step i-2 are on the host
                for s_, d_ in zip((dq, dk, dv), g_sets[st]):
                    thd.thd_rows_to_global(plan, s_, out=d_)
                g_ready[st].record(stream)
                s_down.wait_event(g_ready[st])
                with torch.cuda.stream(s_down):
                    for h_, d_ in zip(h_out[2:], g_sets[st]):
                        h_.copy_(d_, non_blocking=True)
                    g_out[st].record(s_down)
            done = ev()
            done.record(s_down)
            stream.wait_event(done)                        # every result of every step is on the host

        e2e_run(1)
        torch.cuda.synchronize(dev)
        replicas.barrier(info)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        e2e_run(args.e2e_steps)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = replicas.max_over_ranks(info, a0.elapsed_time(a1), device=dev) / args.e2e_steps
        e2e = {"value": replicas.whole_job_rate(step_fl, info.world, e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms,
               "steps": args.e2e_steps}
        del hq_, hk_, hv_, hdo_, h_in, h_out, in_sets, g_sets

    # ------------------------------------------------ rotary embedding (reported beside the step, not in it)
    # Per-document positions of the workload's layout, applied in place to a copy of Q:
    # 2 * T * hq * dqk * 2 bytes of HBM traffic per call (read + write) plus the table.
    pos_d = torch.from_numpy(thd.thd_position_ids(cu)).to(dev)
    q_rope = q.clone()
    rope_ws = torch.empty(T * (w.dqk // 2) * 8, dtype=torch.uint8, device=dev)
    for _ in range(3):
        thd.thd_rope_apply(q_rope, pos_d, workspace=rope_ws)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for _ in range(5):
        thd.thd_rope_apply(q_rope, pos_d, workspace=rope_ws)
    r1.record(stream)
    torch.cuda.synchronize(dev)
    rope_ms = r0.elapsed_time(r1) / 5
    rope_bytes = 2 * T * w.hq * w.dqk * 2 + T * (w.dqk // 2) * 8 * 2 + 4 * T
    del q_rope, rope_ws

    # ------------------------------------------------ K/V all-gather fused into the forward's loads
    # thd_cp_attn_fwd_fused_gather reads K/V from the packed tensors; compared with the
    # step's K/V gather + forward on the same inputs (launches timed back to back).
    def fg_time(fn, reps=3):
        for _ in range(2):
            fn()
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        for _ in range(reps):
            fn()
        b_.record(stream)
        torch.cuda.synchronize(dev)
        return a_.elapsed_time(b_) / reps

    def split():
        thd.thd_kv_gather(plan, k, v, k_rm=k_rm, v_rm=v_rm)
        thd.thd_cp_attn_fwd(plan, q_rm, k_rm, v_rm, out=o_rm, lse=lse_rm)

    fused_ms = fg_time(lambda: thd.thd_cp_attn_fwd_fused_gather(plan, q_rm, k, v, out=o_rm, lse=lse_rm))
    split_ms = fg_time(split)
    fused_gather = {"ms": fused_ms, "tflops": fwd_fl / (fused_ms / 1e3) / 1e12, "gather_plus_fwd_ms": split_ms,
                    "note": "thd_cp_attn_fwd_fused_gather (K/V read from the packed tensors) against "
                            "thd_kv_gather(K, V) + thd_cp_attn_fwd, outside the timed step"}

    # ------------------------------------------------ re-plan for a new layout, other workloads
    peaks, peak_src = load_peaks()
    replan = measure_replan(thd, syn, plan, dev, stream, args.seed, w)
    workloads = None
    if not args.no_workloads:
        workloads = measure_workloads(thd, syn, dev, stream, args.seed, peaks)

    # ------------------------------------------------ CPU oracle baseline (rank 0, N = 1)
    cpu = None
    if info.rank == 0 and info.world == 1 and not args.no_cpu_baseline:
        n_heads = 4
        cu_s, tens, pairs = cpu_sample(w, cu, args.seed, n_heads)
        dt, fl = time_oracle_step(w, cu_s, tens, pairs, n_heads)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"oracle fwd+bwd (fp64 numpy) on the {len(cu_s) - 1} short documents "
                          f"({int(cu_s[-1])} tokens) x {n_heads} query heads, {dt:.1f} s")}

    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    bwd_tf = bwd_fl / (bwd_ms / 1e3) / 1e12
    fwd_tf = fwd_fl / (fwd_ms / 1e3) / 1e12
    gather_bytes = (2 * T * w.hkv * (w.dqk + w.dv) * 2 + 2 * T * w.hq * w.dqk * 2 + 2 * T * w.hq * w.dv * 2
                    + 3 * 4 * T)
    gather_gbs = gather_bytes / (gather_ms / 1e3) / 1e9
    traffic = roofline_traffic(os.path.join(ROOT, "context_packed_sequence_cp_b200", "csrc", "attn_bwd_sm100.cu"))

    value = replicas.whole_job_rate(step_fl, info.world, max_ms / args.steps / 1e3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": info.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, cu, args.seed),
        "roofline": {"kernel": "bwd (thd_cp_attn_bwd: prep + fused key-major dK/dV/dQ tcgen05 kernel)", "bound": "tensor",
                     "achieved": bwd_tf, "peak": sustained, "unit": "TFLOP/s", "frac": bwd_tf / sustained,
                     "traffic": traffic, "peak_source": f"bf16_tflops_sustained ({peak_src})",
                     "flops_per_launch": bwd_fl},
        "fwd": {"ms": fwd_ms, "tflops": fwd_tf, "frac_of_peak": fwd_tf / sustained, "flops": fwd_fl},
        "bwd": {"ms": bwd_ms, "tflops": bwd_tf, "frac_of_peak": bwd_tf / sustained, "flops": bwd_fl},
        "rope": {"ms": rope_ms, "gbs": rope_bytes / (rope_ms / 1e3) / 1e9,
                 "frac_of_hbm": rope_bytes / (rope_ms / 1e3) / 1e9 / hbm, "bytes": rope_bytes,
                 "note": "thd_rope_apply on Q with per-document positions, outside the timed step"},
        "plan": {"host_ms": plan_host_ms, "upload_ms": plan_upload_ms, "q_tiles": plan.n_qtiles,
                 "note": "thd_cp_plan + thd_cp_plan_upload, once per layout (cached), outside the timed step",
                 "replan": replan},
        "workloads": workloads,
        "fused_gather": fused_gather,
        "gather": {"ms": gather_ms, "gbs": gather_gbs, "frac_of_hbm": gather_gbs / hbm, "bytes": gather_bytes,
                   "hbm_peak_gbs": hbm, "peak_source": peak_src},
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if info.rank == 0:
        print(json.dumps(line), flush=True)
    replicas.finalize(info)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
