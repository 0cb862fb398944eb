"""Benchmark of the KSA hot path on B200.

One step = one pass of the whole path over synthetic inputs already in HBM:
  prefill  (Qwen3-4B layer shape: 1 x 32768 text tokens, 32 q / 8 kv heads,
           d 128, k 8, w 8, N(0,1)*0.5 bf16, RoPE theta 1e6, fp32 LSE):
           ksa_interleave_rope + ksa_prefill_fwd;
  decode   (64 sequences x 131072 prior text tokens: 16384 summaries, full
           64-token ring, open-chunk fill uniform 0..7; 32 q / 8 kv heads,
           d 128, k 8, w 8): ksa_cache_append (TEXT) + ksa_decode.
Reported: prefill TFLOP/s on useful (visible) pairs over the ksa_prefill_fwd
time (`value`), decode GB/s over the bytes of the KV slices read, each as a
fraction of the measured B200 peak.  Inputs exceed L2 (126 MB) on both legs.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ksa|reference]
For N > 1 launch with torchrun: each rank runs its own replica (independent
batches, no collective: weak scaling), timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# workloads
PF = dict(seqlens=[32768], k=8, w=8, Hq=32, Hkv=8, d=128, scale=0.5, seed=1, theta=1e6)
# DRAM bytes (read + write) per launch of the dominant kernels, from one ncu
# --set full capture of each kernel as it now stands (set to None whenever
# one of these kernels changes, until it is captured again).
TRAFFIC = {
    # prefill_kernel<128> at this workload: 453.6 MB read (q_aug, k_aug, v_aug
    # once) + 271.6 MB written (o_aug and the LSE, part still in L2 at exit)
    "prefill": (725.2e6, "ncu capture of prefill_kernel<128>, 1 x 32768 text tokens (Qwen3-4B layer): "
                         "dram read 453.6 MB + write 271.6 MB per launch"),
    # decode_split_kernel<128,4> captured at batch 16 (1.0851 GB: 1.0778 GB
    # read, 7.3 MB written); its traffic grows in proportion to the batch
    "decode_per_seq": (1.0851e9 / 16, "ncu capture of decode_split_kernel<128,4> at batch 16 x 16384 summaries: "
                                      "1.0851 GB per 16 sequences, scaled by the batch"),
}
DC = dict(B=64, m=16384, k=8, w=8, Hq=32, Hkv=8, d=128, seed=3, theta=1e6)


def text_row_keys(i, k, w, m):
    """Keys text rows i see (Eqs. (2)-(3)): the window text from chunk
    max(c - w, 0) up to the row itself, and the summaries s_0 .. s_{c-w-1}
    (of m in the sequence); c = i // k."""
    i = np.asarray(i, dtype=np.int64)
    c = i // k
    return (i - np.maximum(c - w, 0) * k + 1) + np.clip(c - w, 0, m)


def useful_pairs(seqlens, k, w):
    """Visible (query, key) pairs per head: the text rows' keys plus k + 1
    for each summary row."""
    tot = 0
    for n in seqlens:
        m = n // k
        tot += int(text_row_keys(np.arange(n), k, w, m).sum()) + m * (k + 1)
    return tot


def text_pairs(seqlens, k, w):
    return useful_pairs(seqlens, k, w) - sum((n // k) * (k + 1) for n in seqlens)


def chunk_pairs(n0, m0, T, k, w):
    """Visible (query, key) pairs per head of a chunked-prefill block: text
    positions n0 .. n0+T-1 (Eqs. (2)-(3)) and the summaries m0 .. m1-1 of the
    chunks it completes (k + 1 keys each)."""
    text = int(text_row_keys(np.arange(n0, n0 + T), k, w, (n0 + T) // k).sum())
    return text + ((n0 + T) // k - m0) * (k + 1)


def decode_slice_rows(m, k, w, fills):
    """Cache rows one TEXT step reads per (sequence, kv head): open chunk
    (f+1) + ring min(m,w)*k + far summaries max(0, m-w)."""
    return np.asarray(fills) + 1 + min(m, w) * k + max(0, m - w)


METRIC = "KSA prefill TFLOP/s (useful pairs) & decode KV GB/s"


def workload_config(world):
    """The config of the default bench line, shared by both arms."""
    from kv_cache_compression_ksa_b200.inputs import uniform_ints
    sl = PF["seqlens"]
    fills = uniform_ints(DC["B"], 0, DC["k"] - 1, seed=DC["seed"]).numpy()
    rows = decode_slice_rows(DC["m"], DC["k"], DC["w"], fills)
    return {
        "workload": "prefill 1x32768 text tokens (Qwen3-4B layer: 32q/8kv heads, d128), k8, w8, "
                    "N(0,1)*0.5 bf16, RoPE 1e6, fp32 LSE; + decode 64 seqs x 131072 prior tokens",
        "global_batch": world, "seq_len": sl[0], "parallelism": f"replicas x{world}",
        "l2": "inputs larger than L2 (prefill q_aug 302 MB; decode slice 4.3 GB)",
        "useful_prefill_tflop": useful_pairs(sl, PF["k"], PF["w"]) * PF["Hq"] * 4 * PF["d"] / 1e12,
        "decode_slice_gb": float(rows.sum()) * DC["Hkv"] * DC["d"] * 2 * 2 / 1e9,
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region.

    The sampler starts before the warm-up (so the process is running when
    the timed region begins) and the summary keeps only the samples whose
    timestamps fall inside the window given to mark()."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        import tempfile
        self.index = index
        self.proc = None
        self.window = None
        self.path = os.path.join(tempfile.gettempdir(), f"ksa_bench_clocks_{os.getpid()}_{index}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return self
        for _ in range(150):   # up to ~3 s for the first line
            if os.path.getsize(self.path) > 0 or self.proc.poll() is not None:
                break
            time.sleep(0.02)
        return self

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            self.proc.wait()
            self.f.close()

    def summary(self):
        from datetime import datetime
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    clk, cmax = float(parts[2]), float(parts[3])
                except ValueError:
                    continue
                if self.window and not (self.window[0] - 0.03 <= ts <= self.window[1] + 0.03):
                    continue
                sm.append(clk)
                mx = cmax
                for nm, v in zip(names, parts[6:10]):
                    if v.lower() == "active":
                        reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    if n_gpus > 1 or "RANK" in os.environ:
        local = int(os.environ.get("LOCAL_RANK", 0))
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
        return dist.get_rank(), dist.get_world_size(), local
    torch.cuda.set_device(0)
    return 0, 1, 0


def max_over_ranks(x, world, device="cuda"):
    """Slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base, rank):
    """Each rank runs an independent replica of the workload (weak scaling):
    same shapes, its own inputs."""
    return base + 100 * rank


def whole_job_rate(work_per_rank, world, max_ms):
    """Aggregate throughput: the work all ranks did over the slowest rank's time."""
    return world * work_per_rank / (max_ms * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# oracle arm (CPU)
# ---------------------------------------------------------------------------
def oracle_sample(sample_rows: int, seed: int = 1):
    """Time the fp64 oracle on a bounded, deterministic sample of the prefill
    workload's text rows (all 32 heads each) and return (TFLOP/s, cores, rows)."""
    import oracle
    import torch
    from kv_cache_compression_ksa_b200.inputs import prefill_inputs
    n, k, w = PF["seqlens"][0], PF["k"], PF["w"]
    x = prefill_inputs(PF["seqlens"], k, PF["Hq"], PF["Hkv"], PF["d"], seed=PF["seed"], scale=PF["scale"])
    f64 = lambda t: t.double().numpy()
    rows = np.linspace(0, n - 1, sample_rows).astype(np.int64)
    qt, kt, vt, qs, ks, vs = (f64(t) for t in (x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum))
    pt, ps = oracle.text_positions(n), oracle.summary_positions(n, k)
    qt, kt = oracle.rope(qt, pt, PF["theta"]), oracle.rope(kt, pt, PF["theta"])
    qs, ks = oracle.rope(qs, ps, PF["theta"]), oracle.rope(ks, ps, PF["theta"])
    t0 = time.perf_counter()
    oracle.ksa_attention(n, k, w, qt, kt, vt, qs, ks, vs, tq_idx=rows, sq_idx=np.zeros(0, np.int64))
    dt = time.perf_counter() - t0
    flops = float(text_row_keys(rows, k, w, n // k).sum()) * PF["Hq"] * 4 * PF["d"]
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return flops / dt / 1e12, cores, len(rows), dt


def run_reference(args, rank, world):
    if rank != 0:
        return
    t_total = 0.0
    vals = []
    for i in range(args.warmup + args.steps):
        v, cores, nrows, dt = oracle_sample(512)
        if i >= args.warmup:
            vals.append(v)
            t_total += dt
    v = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_total / max(args.steps, 1) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(world),
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{nrows} evenly spaced text rows x 32 heads of the 32768-token prefill "
                                   "(the prefill leg: the oracle's TFLOP/s on those rows)"},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ---------------------------------------------------------------------------
# KSA arm (GPU)
# ---------------------------------------------------------------------------
def run_ksa(args, rank, world, local):
    import torch
    from kv_cache_compression_ksa_b200 import _lib as L
    from kv_cache_compression_ksa_b200 import api, build
    from kv_cache_compression_ksa_b200.inputs import fill_normal_, prefill_inputs, uniform_ints

    if rank == 0:
        build.build()
    barrier(world)
    dev = torch.device("cuda", local)
    hbm_peak, tc_peak, tc_sus, peak_src = load_peaks()

    # ---- prefill inputs (HBM resident) ----
    sl, k, w, Hq, Hkv, d = PF["seqlens"], PF["k"], PF["w"], PF["Hq"], PF["Hkv"], PF["d"]
    if args.only == "decode":
        sl = [256]
    x = prefill_inputs(sl, k, Hq, Hkv, d, seed=replica_seed(PF["seed"], rank), scale=PF["scale"], device=dev)
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, PF["theta"])
    nt, ns = sum(sl), sum(n // k for n in sl)
    rows = L.ksa_aug_rows(p, sl)
    qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    va = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    oa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, len(sl), nt), dtype=torch.uint8, device=dev)
    pf_flops = useful_pairs(sl, k, w) * Hq * 4 * d
    pf_text_flops = text_pairs(sl, k, w) * Hq * 4 * d

    do_pf = args.only in (None, "prefill")
    do_dc = args.only in (None, "decode")
    # ---- decode cache (HBM resident) ----
    B, m = (args.decode_batch if do_dc else 1), (DC["m"] if do_dc else 16)
    pd = L.make_params(DC["k"], DC["w"], DC["Hq"], DC["Hkv"], DC["d"], 0.0, DC["theta"])
    cache = api.DecodeCache(pd, B, cap=m + 64, device=dev)
    fill_normal_(cache.k, replica_seed(1000, rank))
    fill_normal_(cache.v, replica_seed(2000, rank))
    fills = uniform_ints(B, 0, DC["k"] - 1, seed=DC["seed"]).numpy()
    state0 = torch.zeros(B, 4, dtype=torch.int32)
    state0[:, 0] = torch.as_tensor(m * DC["k"] + fills, dtype=torch.int32)
    state0[:, 1] = m
    state0 = state0.to(dev)
    gen = torch.Generator(device=dev).manual_seed(5 + rank)
    kn = torch.randn(B, DC["Hkv"], DC["d"], generator=gen, device=dev).to(torch.bfloat16)
    vn = torch.randn(B, DC["Hkv"], DC["d"], generator=gen, device=dev).to(torch.bfloat16)
    qd = torch.randn(B, DC["Hq"], DC["d"], generator=gen, device=dev).to(torch.bfloat16)
    kind = torch.zeros(B, dtype=torch.int8, device=dev)
    max_text = m * DC["k"] + DC["k"]
    dws = cache.workspace(max_text)
    od = torch.empty(B, DC["Hq"], DC["d"], dtype=torch.bfloat16, device=dev)
    lsed = torch.empty(B, DC["Hq"], dtype=torch.float32, device=dev)
    slice_rows = decode_slice_rows(m, DC["k"], DC["w"], fills)
    dec_bytes = float(slice_rows.sum()) * DC["Hkv"] * DC["d"] * 2 * 2  # K and V, bf16

    st = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]

    def step(times):
        cache.state.copy_(state0)  # same step every iteration (one TEXT append + decode)
        ev[0].record(st)
        if do_pf:
            L.ksa_interleave_rope(p, x.cu_seqlens, nt, ns, rows, x.q_text, x.k_text, x.v_text, x.q_sum,
                                  x.k_sum, x.v_sum, qa, ka, va, ws)
        ev[1].record(st)
        if do_pf:
            L.ksa_prefill_fwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, ws)
        ev[2].record(st)
        if do_dc:
            L.ksa_cache_append(pd, cache.desc, kind, kn, vn)
        ev[3].record(st)
        if do_dc:
            L.ksa_decode(pd, cache.desc, kind, qd, od, lsed, max_text, dws)
        ev[4].record(st)
        if times is not None:
            torch.cuda.synchronize()
            times.append([ev[i].elapsed_time(ev[i + 1]) for i in range(4)])

    clk = ClockSampler(local).start()
    for _ in range(args.warmup):
        step(None)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    times = []
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    t_start.record(st)
    for _ in range(args.steps):
        step(times)
    t_end.record(st)
    torch.cuda.synchronize()
    clk.mark(w0, time.time())
    clk.stop()
    barrier(world)
    total_ms = t_start.elapsed_time(t_end)
    tarr = np.asarray(times)  # [steps, 4] ms: rope, prefill, append, decode
    rope_ms, pf_ms, app_ms, dec_ms = (float(np.mean(tarr[:, i])) for i in range(4))
    pf_ms_max = max_over_ranks(pf_ms, world)
    dec_ms_max = max_over_ranks(dec_ms, world)
    step_ms = max_over_ranks(float(np.sum(tarr, axis=1).mean()), world)

    value = whole_job_rate(pf_flops, world, pf_ms_max) / 1e12 if do_pf else 0.0
    dec_gbs = whole_job_rate(dec_bytes, world, dec_ms_max) / 1e9 if do_dc else 0.0
    kern_tflops = pf_text_flops / (pf_ms * 1e-3) / 1e12 if do_pf else 0.0
    if args.only == "decode":
        value = dec_gbs

    # ---- e2e through the public API: pinned host inputs -> device -> result ----
    host = [t.cpu().pin_memory() for t in (x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum)]
    cu_h = x.cu_seqlens.cpu().pin_memory()
    out_h = torch.empty(rows, Hq, d, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host) + cu_h.numel() * 4
    d2h = out_h.numel() * out_h.element_size()

    # Serving-style pipeline over two buffer sets: step i's host->device copy
    # (copy-in stream) overlaps step i-1's prefill (compute stream) and step
    # i-2's device->host copy (copy-out stream); PCIe carries both directions
    # at once.  Every step still copies its inputs in and its output back.
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    dbuf = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in host + [cu_h]] for _ in range(2)]
    out_hb = [out_h, torch.empty_like(out_h).pin_memory()]

    def e2e_run(n, e_start=None, e_end=None):
        done_c = [None, None]
        if e_start is not None:
            e_start.record(s_in)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if done_c[b] is not None:
                    s_in.wait_event(done_c[b])   # step i - 2's prefill has read buffer set b
                for dst, src in zip(dbuf[b], host + [cu_h]):
                    dst.copy_(src, non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            with torch.cuda.stream(st):
                st.wait_event(e_in)
                out = api.prefill(p, sl, dbuf[b][6], *dbuf[b][:6], want_lse=False)
                e_c = torch.cuda.Event()
                e_c.record(st)
                done_c[b] = e_c
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_c)
                out.o_aug.record_stream(s_out)
                out_hb[b].copy_(out.o_aug, non_blocking=True)
        if e_end is not None:
            s_in.wait_stream(s_out)
            s_in.wait_stream(st)
            e_end.record(s_in)

    e2e_ms, e2e_val = None, None
    if not args.profile and do_pf:
        e2e_run(max(2, args.warmup))
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(args.steps, e0, e1)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        e2e_val = whole_job_rate(pf_flops, world, e2e_ms) / 1e12

    clocks = clk.summary()
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(world), useful_prefill_tflop=pf_flops / 1e12,
                           decode_slice_gb=dec_bytes / 1e9),
            "prefill": {"ms": pf_ms, "rope_interleave_ms": rope_ms, "tflops": value / world,
                        "frac_of_bf16_peak": (value / world) / tc_peak},
            "decode": {"ms": dec_ms, "append_ms": app_ms, "gbs": dec_gbs / world,
                       "frac_of_hbm_peak": (dec_gbs / world) / hbm_peak, "batch": B, "summaries": m},
            "roofline": {"bound": "tensor", "achieved": kern_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                         "frac": kern_tflops / tc_peak,
                         "traffic": TRAFFIC["prefill"][0], "traffic_source": TRAFFIC["prefill"][1],
                         "kernel": "prefill_kernel<128> (text rows, with the summary rows on its epilogue warps; "
                                   "time of the ksa_prefill_fwd call)",
                         "peak_source": f"{peak_src} burst bf16", "peak_sustained": tc_sus},
            "roofline_decode": {"bound": "hbm", "achieved": dec_gbs / world, "peak": hbm_peak, "unit": "GB/s",
                                "frac": (dec_gbs / world) / hbm_peak,
                                "traffic": (TRAFFIC["decode_per_seq"][0] * B
                                            if m == DC["m"] and TRAFFIC["decode_per_seq"][0] is not None else None),
                                "traffic_source": TRAFFIC["decode_per_seq"][1],
                                "kernel": "decode_split_kernel<128,4> + combine (time of ksa_decode)"},
            "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "ms": e2e_ms,
                    "pipeline": "two buffer sets; host->device copies, ksa_interleave_rope + ksa_prefill_fwd, "
                                "device->host copies on three streams (step i+1's inputs load while step i "
                                "computes and step i-1's output returns)"},
            "gpu_launches": args.steps * ((5 if do_pf else 0) + (3 if do_dc else 0)),
            "clocks": clocks,
            "timed_region_ms": total_ms,
        }
        if args.only == "decode":
            line["unit"] = "GB/s"
        if world == 1 and not args.profile and args.cpu_rows > 0:
            v, cores, nrows, dt = oracle_sample(args.cpu_rows)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                    "sample": f"{nrows} evenly spaced text rows x 32 heads of the "
                                              f"32768-token prefill ({dt:.1f} s)"}
        print(json.dumps(line))


# ---------------------------------------------------------------------------
# sweep (not the bench line): the long varlen prefill batch and the decode
# grid of batch x context, one JSON line per point
# ---------------------------------------------------------------------------
SWEEP_PREFILL = [
    dict(name="varlen 131072+65536+16384+4000", seqlens=[131072, 65536, 16384, 4000], k=8, w=16, seed=2),
    dict(name="varlen 131072+65536+16384+4003", seqlens=[131072, 65536, 16384, 4003], k=8, w=16, seed=2),
    dict(name="1x32768, sliding chunk number 128", seqlens=[32768], k=8, w=128, seed=1),
    dict(name="1x32768, chunk 16", seqlens=[32768], k=16, w=8, seed=1),
    dict(name="1x32768, chunk 32", seqlens=[32768], k=32, w=8, seed=1),
    dict(name="1x32768, chunk 64 (q heads split over 2 tiles)", seqlens=[32768], k=64, w=8, seed=1),
]
# chunked prefill: (batch, cached tokens per sequence, new tokens per sequence)
SWEEP_CHUNK = [
    dict(name="1 x 4096-token block onto a 126976-token cache", B=1, n0=126976, T=4096),
    dict(name="8 x 2048-token blocks onto 30720-token caches", B=8, n0=30720, T=2048),
    dict(name="64 x 512-token blocks onto 32765-token caches", B=64, n0=32765, T=512),
]
# decode over an MLA latent cache, Table 1's MLA shape (128 heads, d_c 512, d_r 64)
SWEEP_MLA = dict(batches=[1, 16, 64], contexts=[32768, 131072], k=8, w=8, H=128, seed=9)
SWEEP_DECODE = dict(batches=[1, 16, 128], contexts=[4096, 32768, 131072, 1048576], k=8, w=8, Hq=32, Hkv=8,
                    d=128, seed=7, text_steps=64)


def run_sweep(args):
    import torch
    from kv_cache_compression_ksa_b200 import _lib as L
    from kv_cache_compression_ksa_b200 import api, build
    from kv_cache_compression_ksa_b200.inputs import fill_normal_, prefill_inputs, uniform_ints

    build.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    hbm_peak, tc_peak, tc_sus, peak_src = load_peaks()
    Hq, Hkv, d = 32, 8, 128

    def ev_time(fn, warm=3, reps=10):
        for _ in range(warm):
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
        return float(np.median(ts))

    parts = set(args.sweep_parts.split(","))
    for cfg in SWEEP_PREFILL if "prefill" in parts else []:
        sl, k, w = cfg["seqlens"], cfg["k"], cfg["w"]
        x = prefill_inputs(sl, k, Hq, Hkv, d, seed=cfg["seed"], scale=1.0, device=dev)
        p = L.make_params(k, w, Hq, Hkv, d, 0.0, 1e6)
        nt, ns = sum(sl), sum(n // k for n in sl)
        rows = L.ksa_aug_rows(p, sl)
        qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
        ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
        va = torch.empty_like(ka)
        oa = torch.empty_like(qa)
        lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
        ws = torch.empty(L.ksa_prefill_workspace_size(p, len(sl), nt), dtype=torch.uint8, device=dev)
        rope_ms = ev_time(lambda: L.ksa_interleave_rope(p, x.cu_seqlens, nt, ns, rows, x.q_text, x.k_text, x.v_text,
                                                        x.q_sum, x.k_sum, x.v_sum, qa, ka, va, ws))
        ms = ev_time(lambda: L.ksa_prefill_fwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, ws))
        flops = useful_pairs(sl, k, w) * Hq * 4 * d
        tf = flops / (ms * 1e-3) / 1e12
        print(json.dumps({"sweep": "prefill", "workload": cfg["name"] + f", 32q/8kv, d128, k{k}, w{w}, N(0,1) bf16",
                          "useful_tflop": flops / 1e12, "ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / tc_peak,
                          "rope_interleave_ms": rope_ms}), flush=True)
        # prefill -> decode hand-off of the same batch: bytes read and written
        cache = api.DecodeCache(p, len(sl), cap=max(n // k for n in sl) + 8, device=dev)
        hms = ev_time(lambda: cache.from_prefill(x.cu_seqlens, nt, ka, va, ws))
        hrows = sum(n // k + min(n // k, w) * k + (n - (n // k) * k) for n in sl)
        hbytes = hrows * Hkv * d * 2 * 2 * 2
        print(json.dumps({"sweep": "handoff", "workload": cfg["name"] + f", Hkv 8, d128, k{k}, w{w}",
                          "rows": hrows, "ms": hms, "gbs": hbytes / (hms * 1e-3) / 1e9,
                          "frac_of_hbm_peak": hbytes / (hms * 1e-3) / 1e9 / hbm_peak}), flush=True)
        del x, qa, ka, va, oa, lse, ws, cache
        torch.cuda.empty_cache()

    # chunked prefill against a decode cache whose slots are filled straight
    # from N(0,1) (the cached values do not change the work); each timed call
    # starts from the same state (n0, m0), restored before the call
    for cfg in SWEEP_CHUNK if "chunk" in parts else []:
        k, w, B, n0, T = 8, 8, cfg["B"], cfg["n0"], cfg["T"]
        p = L.make_params(k, w, Hq, Hkv, d, 0.0, 1e6)
        m0 = n0 // k
        S = (n0 - m0 * k + T) // k
        cache = api.DecodeCache(p, B, cap=m0 + S + 1, device=dev)
        fill_normal_(cache.k, 31)
        fill_normal_(cache.v, 32)
        st0 = torch.tensor([[n0, m0, 0, 0]] * B, dtype=torch.int32, device=dev)
        gen = torch.Generator(device=dev).manual_seed(33)
        rnd = lambda r, h: torch.randn(r, h, d, generator=gen, device=dev).to(torch.bfloat16)
        tx = [rnd(B * T, Hq), rnd(B * T, Hkv), rnd(B * T, Hkv)]
        sm = [rnd(B * S, Hq), rnd(B * S, Hkv), rnd(B * S, Hkv)]
        cu_t = torch.arange(0, B + 1, dtype=torch.int32, device=dev) * T
        cu_s = torch.arange(0, B + 1, dtype=torch.int32, device=dev) * S
        o_t = torch.empty(B * T, Hq, d, dtype=torch.bfloat16, device=dev)
        o_s = torch.empty(B * S, Hq, d, dtype=torch.bfloat16, device=dev)
        l_t = torch.empty(B * T, Hq, dtype=torch.float32, device=dev)
        l_s = torch.empty(B * S, Hq, dtype=torch.float32, device=dev)
        cws = cache.chunk_workspace(B * T, B * S)
        ts = []
        for it in range(13):
            cache.state.copy_(st0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            L.ksa_prefill_chunk(p, cache.desc, cu_t, B * T, cu_s, B * S, *tx, *sm, o_t, o_s, l_t, l_s, cws)
            b.record()
            torch.cuda.synchronize()
            if it >= 3:
                ts.append(a.elapsed_time(b))
        st = cache.state.cpu().numpy()
        assert (st[:, 3] == 0).all() and (st[:, 0] == n0 + T).all(), f"chunk state {st[0]}"
        ms = float(np.median(ts))
        flops = B * chunk_pairs(n0, m0, T, k, w) * Hq * 4 * d
        tf = flops / (ms * 1e-3) / 1e12
        print(json.dumps({"sweep": "prefill_chunk", "workload": cfg["name"] + ", 32q/8kv, d128, k8, w8, N(0,1) bf16",
                          "useful_tflop": flops / 1e12, "ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / tc_peak,
                          "note": "whole ksa_prefill_chunk call: plan, RoPE, summary write, gather, text rows on "
                                  "the tcgen05 prefill kernel (summary tiles from the cache), summary rows "
                                  "(warp-level MMA), scatter, cache append"}), flush=True)
        del cache, tx, sm, o_t, o_s, l_t, l_s, cws
        torch.cuda.empty_cache()

    if "mla" in parts:
        M = SWEEP_MLA
        k, w, H = M["k"], M["w"], M["H"]
        pm = L.make_mla_params(k, w, H, 512, 64, 0.0, 1e6)
        batches = [int(x) for x in args.mla_batches.split(",")] if args.mla_batches else M["batches"]
        contexts = [int(x) for x in args.mla_contexts.split(",")] if args.mla_contexts else M["contexts"]
        for B in batches:
            for n in contexts:
                m = n // k
                cache = api.MlaCache(pm, B, cap=m + 1, device=dev)
                fill_normal_(cache.latent, M["seed"] + B)
                fills = uniform_ints(B, 1, k, seed=M["seed"]).numpy()
                st = torch.zeros(B, 4, dtype=torch.int32)
                st[:, 0] = torch.as_tensor(m * k + fills, dtype=torch.int32)
                st[:, 1] = m
                cache.state.copy_(st.to(dev))
                gen = torch.Generator(device=dev).manual_seed(M["seed"])
                q = torch.randn(B, H, 576, generator=gen, device=dev).to(torch.bfloat16)
                kind = torch.zeros(B, dtype=torch.int8, device=dev)
                max_text = m * k + k
                mws = cache.workspace(max_text)
                o = torch.empty(B, H, 512, dtype=torch.bfloat16, device=dev)
                lse_m = torch.empty(B, H, dtype=torch.float32, device=dev)
                ms = ev_time(lambda: L.ksa_mla_decode(pm, cache.desc, kind, q, o, lse_m, max_text, mws))
                assert (cache.state[:, 3] == 0).all()
                rows = float(decode_slice_rows(m, k, w, fills - 1).sum())   # fills counts the step's token
                gbs = rows * 576 * 2 / (ms * 1e-3) / 1e9
                tf = rows * H * (576 + 512) * 2 / (ms * 1e-3) / 1e12
                print(json.dumps({"sweep": "mla_decode", "batch": B, "context": n, "summaries": m, "heads": H,
                                  "ms": ms, "slice_gb": rows * 576 * 2 / 1e9, "gbs": gbs,
                                  "frac_of_hbm_peak": gbs / hbm_peak, "tflops": tf,
                                  "frac_of_bf16_peak": tf / tc_peak,
                                  "note": "one TEXT step over latent rows of d_c 512 + d_r 64; " +
                                          ("tcgen05 on CTA pairs (latent dims split, partial scores exchanged "
                                           "through distributed shared memory)" if H % 128 == 0
                                           else "warp-level mma.sync")}),
                      flush=True)
                del cache, q, o, lse_m, mws
                torch.cuda.empty_cache()

    if "bwd" not in parts and "decode" not in parts:
        return
    if "bwd" not in parts:
        return run_decode_sweep(args, L, api, fill_normal_, uniform_ints, dev, hbm_peak, ev_time)
    # backward of the 32768-token prefill (bench shape): useful FLOPs 2.5x the
    # forward's (five products per visible pair: S, dP, dV, dQ, dK)
    sl, k, w = PF["seqlens"], PF["k"], PF["w"]
    x = prefill_inputs(sl, k, Hq, Hkv, d, seed=PF["seed"], scale=PF["scale"], device=dev)
    p = L.make_params(k, w, Hq, Hkv, d, 0.0, PF["theta"])
    nt, ns = sum(sl), sum(n // k for n in sl)
    rows = L.ksa_aug_rows(p, sl)
    qa = torch.empty(rows, Hq, d, dtype=torch.bfloat16, device=dev)
    ka = torch.empty(rows, Hkv, d, dtype=torch.bfloat16, device=dev)
    va = torch.empty_like(ka)
    oa = torch.empty_like(qa)
    lse = torch.empty(rows, Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(L.ksa_prefill_workspace_size(p, len(sl), nt), dtype=torch.uint8, device=dev)
    L.ksa_interleave_rope(p, x.cu_seqlens, nt, ns, rows, x.q_text, x.k_text, x.v_text, x.q_sum, x.k_sum, x.v_sum,
                          qa, ka, va, ws)
    L.ksa_prefill_fwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, ws)
    do = torch.randn(rows, Hq, d, device=dev).to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(qa), torch.empty_like(ka), torch.empty_like(va)
    wsb = torch.empty(L.ksa_prefill_bwd_workspace_size(p, len(sl), rows), dtype=torch.uint8, device=dev)
    ms = ev_time(lambda: L.ksa_prefill_bwd(p, x.cu_seqlens, nt, rows, qa, ka, va, oa, lse, do, dq, dk, dv, wsb))
    flops = 2.5 * useful_pairs(sl, k, w) * Hq * 4 * d
    tf = flops / (ms * 1e-3) / 1e12
    print(json.dumps({"sweep": "prefill_bwd", "workload": "1x32768, 32q/8kv, d128, k8, w8, N(0,1)*0.5 bf16",
                      "useful_tflop": flops / 1e12, "ms": ms, "tflops": tf, "frac_of_bf16_peak": tf / tc_peak,
                      "note": "tcgen05 kernels for the text query rows (dk/dv key-stationary, dq query-stationary: "
                              "S and dP are computed in both), summary query rows on CUDA cores"}),
          flush=True)
    del x, qa, ka, va, oa, lse, ws, do, dq, dk, dv, wsb
    torch.cuda.empty_cache()
    if "decode" in parts:
        run_decode_sweep(args, L, api, fill_normal_, uniform_ints, dev, hbm_peak, ev_time)


def run_decode_sweep(args, L, api, fill_normal_, uniform_ints, dev, hbm_peak, ev_time):
    import torch
    S = SWEEP_DECODE
    k, w = S["k"], S["w"]
    pd = L.make_params(k, w, S["Hq"], S["Hkv"], S["d"], 0.0, 1e6)
    cycle = k + 1                       # k TEXT steps and one SUMMARY step per chunk
    nsteps = S["text_steps"] // k * cycle
    replays = 4
    for B in S["batches"]:
        for n in S["contexts"]:
            m = n // k
            extra = (replays + 2) * (S["text_steps"] // k)
            cache = api.DecodeCache(pd, B, cap=m + extra, device=dev)
            fill_normal_(cache.k, 1000 + B)
            fill_normal_(cache.v, 2000 + B)
            fills = uniform_ints(B, 0, k - 1, seed=S["seed"]).numpy()
            state0 = torch.zeros(B, 4, dtype=torch.int32)
            state0[:, 0] = torch.as_tensor(m * k + fills, dtype=torch.int32)
            state0[:, 1] = m
            cache.state.copy_(state0.to(dev))
            # per step and sequence: SUMMARY when its open chunk is full, else TEXT;
            # nsteps is a whole number of cycles, so every replay starts from the same fills
            kinds = np.zeros((nsteps, B), np.int8)
            nbytes = 0.0
            f = fills.copy()
            mm = np.full(B, m, np.int64)
            for j in range(nsteps):
                full = f == k
                kinds[j] = np.where(full, 1, 0)
                rows_j = np.where(full, k + 1, f + 1 + np.minimum(mm, w) * k + np.maximum(0, mm - w))
                nbytes += float(rows_j.sum()) * S["Hkv"] * S["d"] * 2 * 2
                mm = np.where(full, mm + 1, mm)
                f = np.where(full, 0, f + 1)
            kinds_d = torch.as_tensor(kinds, device=dev)
            gen = torch.Generator(device=dev).manual_seed(S["seed"])
            kn = torch.randn(B, S["Hkv"], S["d"], generator=gen, device=dev).to(torch.bfloat16)
            vn = torch.randn(B, S["Hkv"], S["d"], generator=gen, device=dev).to(torch.bfloat16)
            qd = torch.randn(B, S["Hq"], S["d"], generator=gen, device=dev).to(torch.bfloat16)
            max_text = (m + extra + 1) * k
            dws = cache.workspace(max_text)
            od = torch.empty(B, S["Hq"], S["d"], dtype=torch.bfloat16, device=dev)
            lsed = torch.empty(B, S["Hq"], dtype=torch.float32, device=dev)

            def steps():
                for j in range(nsteps):
                    L.ksa_cache_append(pd, cache.desc, kinds_d[j], kn, vn)
                    L.ksa_decode(pd, cache.desc, kinds_d[j], qd, od, lsed, max_text, dws)

            steps()   # eager pass: loads the kernels, advances one whole number of cycles
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                steps()
            ms = ev_time(g.replay, warm=1, reps=replays - 1)
            st = cache.state.cpu().numpy()
            assert (st[:, 3] == 0).all(), f"cache state error {st[:, 3]}"
            gbs = nbytes / (ms * 1e-3) / 1e9
            print(json.dumps({"sweep": "decode", "batch": B, "context": n, "summaries": m,
                              "text_steps": S["text_steps"], "summary_steps": nsteps - S["text_steps"],
                              "ms_per_text_step": ms / S["text_steps"], "graph_ms": ms,
                              "gb_per_graph": nbytes / 1e9, "gbs": gbs, "frac_of_hbm_peak": gbs / hbm_peak}),
                  flush=True)
            del g, cache, dws, kinds_d, kn, vn, qd, od, lsed
            torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ksa", choices=["ksa", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=2048)
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="time one leg only (profiling); the JSON line then covers that leg")
    ap.add_argument("--profile", action="store_true", help="skip the e2e and CPU legs (for ncu runs)")
    ap.add_argument("--decode-batch", type=int, default=DC["B"])
    ap.add_argument("--sweep-parts", default="prefill,chunk,mla,bwd,decode",
                    help="comma list of the sweep's parts: prefill, chunk, mla, bwd, decode")
    ap.add_argument("--mla-batches", default=None, help="comma list: the MLA sweep's batches (default all)")
    ap.add_argument("--mla-contexts", default=None, help="comma list: the MLA sweep's contexts (default all)")
    ap.add_argument("--sweep", action="store_true",
                    help="time the long varlen prefill batch and the decode batch x context grid (one JSON line per point)")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", 0))
        world = int(os.environ.get("WORLD_SIZE", 1))
        run_reference(args, rank, world)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_ksa(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
