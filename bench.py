"""Benchmark of the TokenGate gated-prefill hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tokengate|reference]
                    [--workload c2_32k_k2000] [--layers 1] [--no-cpu-baseline]

One step = one pass of the whole path over one batch of seeded synthetic
input: gate scoring, top-K selection, compaction, and one token-gated
attention layer (tg_gated_prefill_layer).  Default workload: Qwen3-1.7B
shapes at N=32768 with K=2000 kept state tokens (M=2256 kept rows).

Metric: gated-prefill layer tokens/s (N / step time), with the gated
attention's TFLOP/s and its fraction of the measured bf16 peak reported
beside it.  Inputs are resident in HBM when timing starts; L2 is flushed by
a 256 MB write before every timed step (outside the step's events).

Under torchrun (N>1) every rank runs an independent replica of the workload
(the path is single-GPU; no collective on the data path), the value is the
tokens of all ranks divided by the slowest rank's time, and scaling is weak.

--impl reference times the fp64 CPU oracle on whole steps of the same workload
(every prunable row scored, every kept row attended); it is a slow program by
design (about 1.5 s per step at the default workload on 16 host threads).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import get_config, make_attention_inputs, make_gate_inputs, make_scores  # noqa: E402

METRIC = "gated-prefill layer tokens/s; gated-attn TFLOP/s (% bf16 peak) at N=32k,K=2000"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


# ------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(vals, ws, device):
    """Element-wise max of per-rank device timings over all ranks of the process group
    (a no-op on one rank): the job's time is its slowest rank's."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if ws > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_rate(ws, units_per_rank_step, steps, t_total_ms):
    """Whole-job throughput: the units every rank processed over the (slowest rank's) time."""
    return ws * units_per_rank_step * steps / (t_total_ms / 1e3)


def attention_flops(cu_kept, Hq, d):
    m = np.diff(np.asarray(cu_kept, np.int64))
    pairs = int(np.sum(m * (m + 1) // 2))
    return 4.0 * d * Hq * pairs, pairs


def stage_bytes(w, M):
    """Algorithmic HBM bytes per launch of each stage (read + write)."""
    n_prun = sum(p1 - p0 for p0, p1 in w.spans)
    return {
        # hidden rows of the span read once, one fp32 score written, Wg read once
        "score": n_prun * (2 * w.D + 4) + 2 * w.I * w.D,
        # scores read, keep flags written, compaction indices written
        "select": n_prun * 4 + w.T * 1 + M * 16,
        # kept rows read and written
        "gather": M * 2 * 2 * w.D,
    }


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"tg_clocks_{os.getpid()}_gpu{gpu_index}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def read_traffic_table():
    """Per-launch DRAM bytes from the committed ncu summary, keyed by kernel
    and the sha of the source file it was captured from."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    out = {}
    if not os.path.exists(path):
        return out
    for line in open(path):
        m = re.match(r"\|\s*(\w+)\s*\|\s*([0-9a-f]{12})\s*\|\s*([\w.]+)\s*\|\s*([0-9.]+)\s*\|", line)
        if m:
            out[(m.group(1), m.group(3))] = (m.group(2), float(m.group(4)))
    return out


def source_sha(kernel_file: str) -> str:
    import hashlib
    p = os.path.join(ROOT, "learned_token_pruning_rmsnorm_b200", "csrc", kernel_file)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:12]


KERNEL_FILES = {"score": "k_gate.cu", "select": "k_select.cu", "gather": "k_select.cu",
                "attention": "k_attention.cu"}


# ------------------------------------------------------------------ oracle (CPU baseline / reference arm)

def oracle_step(w, gi, Wg_bits, layers):
    """One whole step of the fp64 oracle over the workload: the gate score of every
    prunable row, top-K selection, compaction, and the gated-attention layers (one per
    entry of `layers`) over every kept row.  Returns (seconds, description, per-part
    seconds)."""
    import oracle
    cu, span, k = w.cu_seqlens(), w.span_array(), w.budget_array()
    n_prun = int(sum(p1 - p0 for p0, p1 in w.spans))
    t0 = time.perf_counter()
    s = oracle.score(gi["hidden"], cu, span, Wg_bits, gi["b1"], gi["w2"], gi["b2"], w.eps)
    t1 = time.perf_counter()
    s32 = np.nan_to_num(s, nan=0.0).astype(np.float32)
    keep = oracle.select_topk(s32, cu, span, k)
    comp = oracle.compact(gi["hidden"], s32, keep, cu, span)
    t2 = time.perf_counter()
    cu_kept = comp["cu_kept"]
    M = int(cu_kept[-1])
    for layer in layers:
        oracle.gated_attention(layer["q"], layer["k"], layer["v"], cu_kept, comp["pos"], comp["rank"],
                               comp["gls"].astype(np.float32), layer["g"], layer["c"], want_lse=False)
    t3 = time.perf_counter()
    _, pairs = attention_flops(cu_kept, w.Hq, w.d)
    desc = (f"oracle fp64, whole step: gate score of all {n_prun} prunable rows, select + compact, "
            f"{len(layers)} attention layer(s) over all {M} kept rows x {w.Hq} heads ({pairs} causal pairs "
            f"each); nothing extrapolated")
    return t3 - t0, desc, {"score_s": t1 - t0, "select_compact_s": t2 - t1, "attention_s": t3 - t2}


def oracle_baseline(w, gi, Wg_bits, layers, min_seconds=10.0, max_steps=8):
    """The oracle timed on whole steps (at least two, until about `min_seconds` of CPU
    work): the cpu_baseline leg of the GPU arm."""
    import oracle
    times, desc, parts = [], "", None
    while len(times) < 2 or (sum(times) < min_seconds and len(times) < max_steps):
        t, desc, parts = oracle_step(w, gi, Wg_bits, layers)
        times.append(t)
    t = float(np.mean(times))
    return {"value": w.T / t, "unit": UNIT, "cores": oracle.get_threads(), "kind": "oracle",
            "sample": f"{len(times)} whole steps; {desc}", "seconds_per_step": t, "parts_s": parts}


def run_reference(args, w):
    import oracle
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    gi = make_gate_inputs(w)
    Wg = oracle.gate_fold(gi["gamma"], gi["W1"])
    M = int(w.cu_kept()[-1])
    layers = [make_attention_inputs(w, M, layer=l) for l in range(args.layers)]
    times = []
    desc = ""
    for it in range(args.warmup + args.steps):
        t, desc, _ = oracle_step(w, gi, Wg, layers)
        if it >= args.warmup:
            times.append(t)
    t = float(np.mean(times))
    value = w.T / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": workload_config(w, args.layers),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.get_threads(), "kind": "oracle",
                             "sample": f"{args.steps} timed whole steps after {args.warmup} warm-up; {desc}"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, n_layers):
    M = int(w.cu_kept()[-1])
    return {"workload": w.name, "B": w.B, "N": list(w.seqlens) if w.B > 1 else w.seqlens[0],
            "K": list(w.budgets) if w.B > 1 else w.budgets[0], "M": M, "D": w.D, "I": w.I, "Hq": w.Hq,
            "Hkv": w.Hkv, "head_dim": w.d, "attn_layers_per_step": n_layers,
            "l2": "flushed (256 MB write) before every timed step", "parallelism": "replicas"}


# ------------------------------------------------------------------ GPU arm

def time_device_us(fn, st, flush, reps, warm=3):
    """Median device time (us) of fn() on stream st, L2 flushed before each rep.  fn is
    captured into a CUDA graph and the replays are timed, so that no host work (argument
    checks, tensor-map encoding) sits between the events."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        fn()
    gr.replay()
    torch.cuda.synchronize()
    ev = []
    for i in range(reps):
        flush.fill_(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        gr.replay()
        b.record(st)
        ev.append((a, b))
    torch.cuda.synchronize()
    del gr
    return 1e3 * float(np.median([a.elapsed_time(b) for a, b in ev]))


def measure_next_rows(tg, dev, st, flush, main, peaks, reps=10):
    """One measured figure per widened row, each on its own seeded workload:
    masked full-length attention at a sampled budget, the KV-cache row gather,
    head_dim 256 attention and four stacked gates.  Each is one C-ABI call with
    its arguments bound beforehand (device-resident inputs and index arrays);
    L2 is flushed before every rep."""
    import ctypes
    import torch
    from workloads import masked_budgets

    lib = tg.load()

    def sh_now():  # the current stream (the capture stream while a call is recorded)
        return torch.cuda.current_stream(dev).cuda_stream

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)

    def check(fn):
        def run():
            assert fn() == 0, lib.tg_last_error_string()
        return run

    tc_peak, hbm_peak = float(peaks["bf16_tflops"]), float(peaks["hbm_gbs"])
    res = {}
    # f1: masked full-length attention (training layout), N=16384, K' sampled log-uniform
    w = get_config("c3_full_budget_16k")
    kb = np.asarray(masked_budgets(w, seed=0), np.int32)
    ai = make_attention_inputs(w, w.T, layer=0)
    q, k, v = bf16(ai["q"]), bf16(ai["k"]), bf16(ai["v"])
    g, c = torch.from_numpy(ai["g"]).to(dev), torch.from_numpy(ai["c"]).to(dev)
    s = torch.from_numpy(make_scores(w.T, std=2.0, seed=w.seed)).to(dev)
    out = torch.empty((w.T, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    keep = torch.empty(w.T, dtype=torch.uint8, device=dev)
    cu, sp = w.cu_seqlens(), w.span_array()
    Mm, ck = tg.tg_kept_count(cu, sp, kb)
    maxm = int(np.max(np.diff(ck)))
    cu_d, sp_d, kb_d, ck_d = i32(cu), i32(sp), i32(kb), i32(ck)
    nws = int(lib.tg_masked_gated_attention_workspace_size(w.B, w.T, Mm, maxm, w.Hq, w.Hkv, w.d))
    mws = torch.zeros(max(nws, 256), dtype=torch.uint8, device=dev)
    fl, _ = attention_flops(ck, w.Hq, w.d)
    us = time_device_us(check(lambda: lib.tg_masked_gated_attention(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), s.data_ptr(), cu_d.data_ptr(), sp_d.data_ptr(), kb_d.data_ptr(),
        ck_d.data_ptr(), w.B, w.T, Mm, maxm, w.Hq, w.Hkv, w.d, g.data_ptr(), c.data_ptr(), 1.0 / math.sqrt(w.d),
        out.data_ptr(), keep.data_ptr(), mws.data_ptr(), mws.numel(), sh_now())), st, flush, reps)
    res["f1_masked_attention"] = {"workload": f"{w.name}: N={w.T}, K'={int(kb[0])} (log-uniform in [1, |P|/2]), M={Mm}",
                                  "us": us, "kept_pair_tflops": fl / (us * 1e-6) / 1e12,
                                  "includes": "zero fill of pruned rows + select map + Q/K/V row gather + attention "
                                              "+ scatter"}
    del q, k, v, out, s, mws
    # f2: lower-layer KV cache gathered to the kept tokens (one layer's K cache)
    wm = main["w"]
    kcache = torch.randn((wm.T, wm.Hkv, wm.d), device=dev).to(torch.bfloat16)
    kdst = torch.empty((main["M"], wm.Hkv, wm.d), dtype=torch.bfloat16, device=dev)
    row_bytes = wm.Hkv * wm.d * 2
    us = time_device_us(check(lambda: lib.tg_gather_rows(kcache.data_ptr(), wm.T, row_bytes,
                                                         main["kept_idx"].data_ptr(), main["M"], kdst.data_ptr(), sh_now())),
                        st, flush, reps)
    nbytes = 2 * main["M"] * row_bytes
    res["f2_kv_gather"] = {"workload": f"{wm.name}: K cache [{wm.T}, {wm.Hkv}, {wm.d}] bf16 -> {main['M']} rows",
                           "us": us, "bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9,
                           "frac_of_hbm": nbytes / (us * 1e-6) / 1e9 / hbm_peak}
    del kcache, kdst
    # f3: head_dim 256 attention, N=16384, K=2000
    w = get_config("c5_hd256_16k")
    cu, sp, kk = w.cu_seqlens(), w.span_array(), w.budget_array()
    M, ck = tg.tg_kept_count(cu, sp, kk)
    s = torch.from_numpy(make_scores(w.T, std=2.0, seed=w.seed)).to(dev)
    _, cmap = tg.tg_select_topk(s, cu, sp, kk, cu_kept=ck, M_total=M)
    ai = make_attention_inputs(w, M, layer=0)
    q, k, v = bf16(ai["q"]), bf16(ai["k"]), bf16(ai["v"])
    g, c = torch.from_numpy(ai["g"]).to(dev), torch.from_numpy(ai["c"]).to(dev)
    out = torch.empty((M, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    ck_d = i32(ck)
    maxM = int(np.max(np.diff(ck)))
    fl, _ = attention_flops(ck, w.Hq, w.d)
    us = time_device_us(check(lambda: lib.tg_gated_attention(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), ck_d.data_ptr(), w.B, M, maxM, w.Hq, w.Hkv, w.d,
        cmap["pos"].data_ptr(), cmap["rank"].data_ptr(), cmap["gls"].data_ptr(), g.data_ptr(), c.data_ptr(),
        1.0 / math.sqrt(w.d), out.data_ptr(), None, None, 0, sh_now())), st, flush, reps)
    res["f3_hd256_attention"] = {"workload": f"{w.name}: M={M}, Hq={w.Hq}, Hkv={w.Hkv}, d={w.d}", "us": us,
                                 "tflops": fl / (us * 1e-6) / 1e12,
                                 "frac_of_bf16_peak": fl / (us * 1e-6) / 1e12 / tc_peak}
    # f1 x f3: the backward at head_dim 256 on the same workload, from the forward's output and lse
    lse5 = torch.empty((M, w.Hq), dtype=torch.float32, device=dev)
    assert lib.tg_gated_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), ck_d.data_ptr(), w.B, M, maxM, w.Hq,
                                  w.Hkv, w.d, cmap["pos"].data_ptr(), cmap["rank"].data_ptr(), cmap["gls"].data_ptr(),
                                  g.data_ptr(), c.data_ptr(), 1.0 / math.sqrt(w.d), out.data_ptr(), lse5.data_ptr(),
                                  None, 0, sh_now()) == 0
    dout5 = torch.randn((M, w.Hq, w.d), device=dev).to(torch.bfloat16)
    gr5 = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    f5 = [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(2)] + \
         [torch.empty(w.Hq, dtype=torch.float32, device=dev) for _ in range(2)]
    nb5 = int(lib.tg_gated_attention_backward_workspace_size(M, w.Hq, w.Hkv, w.d))
    bws5 = torch.empty(nb5, dtype=torch.uint8, device=dev)
    us = time_device_us(check(lambda: lib.tg_gated_attention_backward(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout5.data_ptr(), lse5.data_ptr(), ck_d.data_ptr(),
        w.B, M, maxM, w.Hq, w.Hkv, w.d, cmap["pos"].data_ptr(), cmap["rank"].data_ptr(), cmap["gls"].data_ptr(),
        g.data_ptr(), c.data_ptr(), 1.0 / math.sqrt(w.d), gr5[0].data_ptr(), gr5[1].data_ptr(), gr5[2].data_ptr(),
        f5[0].data_ptr(), f5[1].data_ptr(), f5[2].data_ptr(), f5[3].data_ptr(), bws5.data_ptr(), bws5.numel(),
        sh_now())), st, flush, reps)
    res["f1_attention_backward_hd256"] = {"workload": f"{w.name}: M={M}, Hq={w.Hq}, Hkv={w.Hkv}, d={w.d}",
                                          "us": us, "tflops": 2.5 * fl / (us * 1e-6) / 1e12,
                                          "frac_of_bf16_peak": 2.5 * fl / (us * 1e-6) / 1e12 / tc_peak,
                                          "algorithmic": "2.5x the forward's 4*d*Hq per causal pair"}
    del lse5, dout5, gr5, f5, bws5
    # f4: four stacked gates on the main workload's attention (same inputs as the step's)
    L0, wm, bufs = main["layer"], main["w"], main["bufs"]
    rng = np.random.default_rng(5)
    extra = [torch.from_numpy(np.where(main["gls_host"] != 0, -np.abs(rng.standard_normal(main["M"])), 0.0)
                              .astype(np.float32)).to(dev) for _ in range(3)]
    gains = [L0["g"]] + [torch.from_numpy(rng.standard_normal(wm.Hq).astype(np.float32)).to(dev) for _ in range(3)]
    gls_arr = (ctypes.c_void_p * 4)(*([bufs.gls.data_ptr()] + [t.data_ptr() for t in extra]))
    g_arr = (ctypes.c_void_p * 4)(*[t.data_ptr() for t in gains])
    out = torch.empty((main["M"], wm.Hq, wm.d), dtype=torch.bfloat16, device=dev)
    ck_d = i32(main["cu_kept"])
    ws_t = main["ws"]
    ws_p, ws_n = (None, 0) if ws_t is None else (ws_t.data_ptr(), ws_t.numel())
    fl, _ = attention_flops(main["cu_kept"], wm.Hq, wm.d)
    sm = 1.0 / math.sqrt(wm.d)
    common = (L0["q"].data_ptr(), L0["k"].data_ptr(), L0["v"].data_ptr(), ck_d.data_ptr(), wm.B, main["M"],
              main["max_M"], wm.Hq, wm.Hkv, wm.d, bufs.pos.data_ptr(), bufs.rank.data_ptr())
    us = time_device_us(check(lambda: lib.tg_gated_attention_gates(*common, 4, gls_arr, g_arr, L0["c"].data_ptr(), sm,
                                                                   out.data_ptr(), None, ws_p, ws_n, sh_now())),
                        st, flush, reps)
    us1 = time_device_us(check(lambda: lib.tg_gated_attention(*common, bufs.gls.data_ptr(), L0["g"].data_ptr(),
                                                              L0["c"].data_ptr(), sm, out.data_ptr(), None, ws_p,
                                                              ws_n, sh_now())), st, flush, reps)
    res["f4_four_gates_attention"] = {"workload": f"{wm.name}: M={main['M']}, 4 gates", "us": us,
                                      "tflops": fl / (us * 1e-6) / 1e12, "one_gate_us": us1,
                                      "vs_one_gate": us / us1}
    # the key bias's cost: the same attention with gls = g = c = NULL (ordinary causal
    # attention, no bias k-step, tau = 1), against the gated call in the same kernel (the
    # persistent one, which serves both) and against the default gated call
    us_plain = time_device_us(check(lambda: lib.tg_gated_attention(*common, None, None, None, sm, out.data_ptr(),
                                                                   None, ws_p, ws_n, sh_now())), st, flush, reps)
    old_env = os.environ.get("TG_ATTENTION_KERNEL")
    os.environ["TG_ATTENTION_KERNEL"] = "persistent"
    try:
        nws = int(lib.tg_gated_attention_workspace_size(wm.B, main["max_M"], wm.Hq, wm.Hkv, wm.d))
        assert nws <= ws_n
        us_gp = time_device_us(check(lambda: lib.tg_gated_attention(*common, bufs.gls.data_ptr(), L0["g"].data_ptr(),
                                                                    L0["c"].data_ptr(), sm, out.data_ptr(), None,
                                                                    ws_p, ws_n, sh_now())), st, flush, reps)
    finally:
        if old_env is None:
            os.environ.pop("TG_ATTENTION_KERNEL", None)
        else:
            os.environ["TG_ATTENTION_KERNEL"] = old_env
    res["m6_key_bias_overhead"] = {"workload": f"{wm.name}: M={main['M']}, one gate vs none",
                                   "plain_us": us_plain, "gated_same_kernel_us": us_gp, "gated_default_us": us1,
                                   "same_kernel_ratio": us_gp / us_plain, "default_ratio": us1 / us_plain}
    # f1 (training): backward of the gated attention on the main workload, from the
    # forward's output and log-sum-exp
    lse = torch.empty((main["M"], wm.Hq), dtype=torch.float32, device=dev)
    assert lib.tg_gated_attention(*common, bufs.gls.data_ptr(), L0["g"].data_ptr(), L0["c"].data_ptr(), sm,
                                  out.data_ptr(), lse.data_ptr(), ws_p, ws_n, sh_now()) == 0
    dout = torch.randn((main["M"], wm.Hq, wm.d), device=dev).to(torch.bfloat16)
    grads = [torch.empty_like(L0["q"]), torch.empty_like(L0["k"]), torch.empty_like(L0["v"])]
    f32 = [torch.empty(main["M"], dtype=torch.float32, device=dev) for _ in range(2)] + \
          [torch.empty(wm.Hq, dtype=torch.float32, device=dev) for _ in range(2)]
    nb = int(lib.tg_gated_attention_backward_workspace_size(main["M"], wm.Hq, wm.Hkv, wm.d))
    bws = torch.empty(nb, dtype=torch.uint8, device=dev)
    us = time_device_us(check(lambda: lib.tg_gated_attention_backward(
        L0["q"].data_ptr(), L0["k"].data_ptr(), L0["v"].data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
        ck_d.data_ptr(), wm.B, main["M"], main["max_M"], wm.Hq, wm.Hkv, wm.d, bufs.pos.data_ptr(),
        bufs.rank.data_ptr(), bufs.gls.data_ptr(), L0["g"].data_ptr(), L0["c"].data_ptr(), sm, grads[0].data_ptr(),
        grads[1].data_ptr(), grads[2].data_ptr(), f32[0].data_ptr(), f32[1].data_ptr(), f32[2].data_ptr(),
        f32[3].data_ptr(), bws.data_ptr(), bws.numel(), sh_now())), st, flush, reps)
    res["f1_attention_backward"] = {"workload": f"{wm.name}: M={main['M']}, Hq={wm.Hq}, Hkv={wm.Hkv}, d={wm.d}",
                                    "us": us, "tflops": 2.5 * fl / (us * 1e-6) / 1e12,
                                    "frac_of_bf16_peak": 2.5 * fl / (us * 1e-6) / 1e12 / tc_peak,
                                    "algorithmic": "2.5x the forward's 4*d*Hq per causal pair (five products)"}
    return res


def device_gate_inputs(tg, w, dev):
    """Gate weights from the seeded workload generator; the hidden rows are drawn on the
    device from a seeded generator with the same distribution (N(0, 1), the workload's
    outlier channels x8), which keeps the largest workloads' set-up to milliseconds."""
    import torch
    from workloads import make_gate_weights
    gw = make_gate_weights(w)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7919 * (w.seed + 1) + w.T)
    hidden = torch.randn((w.T, w.D), generator=gen, device=dev, dtype=torch.float32)
    if len(gw["outlier_channels"]):
        hidden[:, torch.from_numpy(gw["outlier_channels"]).to(dev)] *= w.outlier_scale
    hidden = hidden.to(torch.bfloat16)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    Wg = tg.tg_gate_prepare(bf16(gw["gamma"]), bf16(gw["W1"]))
    return hidden, Wg, torch.from_numpy(gw["b1"]).to(dev), torch.from_numpy(gw["w2"]).to(dev), gw["b2"]


def device_attention_inputs(w, M, n_layers, dev, seed=0):
    """Per-layer q, k, v (N(0, 1) x the workload's std, bf16), g ~ N(0, 0.5), c ~ U(0, 0.5),
    drawn on the device from a seeded generator."""
    import torch
    gen = torch.Generator(device=dev)
    out = []
    for l in range(n_layers):
        gen.manual_seed(104729 * (seed + 1) + 31 * l + M)
        rnd = lambda *shape: torch.randn(shape, generator=gen, device=dev, dtype=torch.float32)  # noqa: E731
        out.append({"q": (rnd(M, w.Hq, w.d) * w.qkv_std).to(torch.bfloat16),
                    "k": (rnd(M, w.Hkv, w.d) * w.qkv_std).to(torch.bfloat16),
                    "v": (rnd(M, w.Hkv, w.d) * w.qkv_std).to(torch.bfloat16),
                    "g": rnd(w.Hq) * w.g_std,
                    "c": torch.rand((w.Hq,), generator=gen, device=dev) * w.c_high})
    return out


def measure_workload(tg, dev, st, flush, peaks, w, n_layers=1, reps=10, stages=True):
    """One gated-prefill call (score, select + compaction map, n_layers attention layers,
    row gather) on workload w, replayed as a CUDA graph after an L2 flush; median of reps.
    With `stages`, the attention and the stages 1-3 are also timed alone for their
    roofline fractions."""
    import torch
    from learned_token_pruning_rmsnorm_b200 import PrefillBuffers, PrefillCall
    lib = tg.load()
    hidden, Wg, b1, w2, b2 = device_gate_inputs(tg, w, dev)
    cu, span, k = w.cu_seqlens(), w.span_array(), w.budget_array()
    M, cu_kept = tg.tg_kept_count(cu, span, k)
    layers = device_attention_inputs(w, M, n_layers, dev, seed=w.seed)
    bufs = PrefillBuffers(w.T, w.D, M, n_layers, w.Hq, w.d, dev, with_hidden=True)
    call = PrefillCall(hidden, cu, span, k, Wg, b1, w2, b2, w.eps, layers, bufs, w.Hq, w.Hkv, w.d)
    step_us = time_device_us(call, st, flush, reps)
    flops, pairs = attention_flops(cu_kept, w.Hq, w.d)
    tc_peak, hbm_peak = float(peaks["bf16_tflops"]), float(peaks["hbm_gbs"])
    res = {"N": list(w.seqlens) if w.B > 1 else w.seqlens[0], "K": list(w.budgets) if w.B > 1 else w.budgets[0],
           "M": M, "attn_layers": n_layers, "step_us": step_us, "tokens_per_s": w.T / (step_us * 1e-6),
           "attn_flops_per_layer": flops}
    if not stages:
        return res, call
    sh = lambda: torch.cuda.current_stream(dev).cuda_stream  # noqa: E731
    L0 = layers[0]
    ws_p, ws_n = (None, 0) if call.ws is None else (call.ws.data_ptr(), call.ws.numel())
    sm = 1.0 / math.sqrt(w.d)

    def ok(rc):
        assert rc == 0, lib.tg_last_error_string()

    attn = lambda: ok(lib.tg_gated_attention(  # noqa: E731
        L0["q"].data_ptr(), L0["k"].data_ptr(), L0["v"].data_ptr(), call.ck.data_ptr(), w.B, M, call.max_M, w.Hq,
        w.Hkv, w.d, bufs.pos.data_ptr(), bufs.rank.data_ptr(), bufs.gls.data_ptr(), L0["g"].data_ptr(),
        L0["c"].data_ptr(), sm, bufs.out[0].data_ptr(), None, ws_p, ws_n, sh()))
    score = lambda: ok(lib.tg_score(  # noqa: E731
        hidden.data_ptr(), call.cu.data_ptr(), call.sp.data_ptr(), w.B, w.T, w.D, Wg.data_ptr(), b1.data_ptr(),
        w2.data_ptr(), float(b2), w.I, float(w.eps), bufs.scores.data_ptr(), sh()))
    select = lambda: ok(lib.tg_select_topk(  # noqa: E731
        bufs.scores.data_ptr(), call.cu.data_ptr(), call.sp.data_ptr(), call.kk.data_ptr(), w.B, w.T,
        bufs.keep.data_ptr(), call.ck.data_ptr(), bufs.kept_idx.data_ptr(), bufs.pos.data_ptr(),
        bufs.rank.data_ptr(), bufs.gls.data_ptr(), sh()))
    gather = lambda: ok(lib.tg_compact(  # noqa: E731
        hidden.data_ptr(), None, None, None, None, w.B, w.T, w.D, None, M, bufs.hidden_kept.data_ptr(), None, None,
        None, bufs.kept_idx.data_ptr(), sh()))
    a_us = time_device_us(attn, st, flush, reps)
    s_us = [time_device_us(f, st, flush, reps) for f in (score, select, gather)]
    sb = stage_bytes(w, M)
    s13_bytes = sb["score"] + sb["select"] + sb["gather"]
    s13_us = sum(s_us)
    res.update({"attn_us": a_us, "attn_tflops": flops / (a_us * 1e-6) / 1e12,
                "attn_frac_of_bf16_peak": flops / (a_us * 1e-6) / 1e12 / tc_peak,
                "stage_us": {"score": s_us[0], "select": s_us[1], "gather": s_us[2]},
                "score_frac_of_hbm": sb["score"] / (s_us[0] * 1e-6) / 1e9 / hbm_peak,
                "score_select_compact_gbs": s13_bytes / (s13_us * 1e-6) / 1e9,
                "score_select_compact_frac_of_hbm": s13_bytes / (s13_us * 1e-6) / 1e9 / hbm_peak})
    return res, call


def measure_workload_sweep(tg, dev, st, flush, peaks, main_step_us):
    """Every seeded workload besides the headline one, each on its own prefill call: the
    K sweep at 32k, 16k, 128k and the varlen batch; the 14-layer stack of the 32k, K=2000
    workload; and dense causal attention over all 16384 tokens (config 3's comparison:
    no pruning, bias 0 and temperature 1)."""
    import torch
    res = {}
    for name in ("c1_16k", "c2_32k_k100", "c2_32k_k500", "c2_32k_kall", "c4_128k", "c4_varlen"):
        w = get_config(name)
        r, call = measure_workload(tg, dev, st, flush, peaks, w, reps=5 if name == "c2_32k_kall" else 10)
        res[name] = r
        del call
        torch.cuda.empty_cache()
    # the stack: one call with 14 attention layers (each its own q, k, v, g, c)
    w = get_config("c2_32k_k2000")
    r14, call = measure_workload(tg, dev, st, flush, peaks, w, n_layers=14, stages=False)
    r1, call1 = measure_workload(tg, dev, st, flush, peaks, w, n_layers=1, stages=False)
    per_layer = (r14["step_us"] - r1["step_us"]) / 13.0
    r14.update({"one_layer_step_us": r1["step_us"], "marginal_attn_layer_us": per_layer,
                "marginal_attn_tflops": r14["attn_flops_per_layer"] / (per_layer * 1e-6) / 1e12,
                "marginal_attn_frac_of_bf16_peak": r14["attn_flops_per_layer"] / (per_layer * 1e-6) / 1e12
                / float(peaks["bf16_tflops"])})
    res["c2_32k_k2000_stack14"] = r14
    del call, call1
    torch.cuda.empty_cache()
    # dense causal attention over the whole 16k sequence (no compaction; gls = 0, c = 0)
    w = get_config("c3_full_budget_16k")
    lib = tg.load()
    N = w.T
    L = device_attention_inputs(w, N, 1, dev, seed=3)[0]
    zeros = torch.zeros(N, dtype=torch.float32, device=dev)
    c0 = torch.zeros(w.Hq, dtype=torch.float32, device=dev)
    ar = torch.arange(1, N + 1, dtype=torch.int32, device=dev)
    ck = torch.tensor([0, N], dtype=torch.int32, device=dev)
    out = torch.empty((N, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    ws = tg.attention_workspace(1, N, w.Hq, w.Hkv, w.d, dev)
    ws_p, ws_n = (None, 0) if ws is None else (ws.data_ptr(), ws.numel())
    flops, _ = attention_flops(np.array([0, N]), w.Hq, w.d)

    def dense():
        assert lib.tg_gated_attention(L["q"].data_ptr(), L["k"].data_ptr(), L["v"].data_ptr(), ck.data_ptr(), 1, N, N,
                                      w.Hq, w.Hkv, w.d, ar.data_ptr(), ar.data_ptr(), zeros.data_ptr(),
                                      L["g"].data_ptr(), c0.data_ptr(), 1.0 / math.sqrt(w.d), out.data_ptr(), None,
                                      ws_p, ws_n, torch.cuda.current_stream(dev).cuda_stream) == 0
    us = time_device_us(dense, st, flush, 5)
    res["c3_dense_causal_16k"] = {"N": N, "us": us, "flops": flops, "tflops": flops / (us * 1e-6) / 1e12,
                                  "frac_of_bf16_peak": flops / (us * 1e-6) / 1e12 / float(peaks["bf16_tflops"]),
                                  "note": "unpruned causal attention, N=16384, 16/8 heads, d=128 (gls = 0, c = 0)"}
    del L, out, ws
    torch.cuda.empty_cache()
    return res


def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))

    import learned_token_pruning_rmsnorm_b200 as tg
    from learned_token_pruning_rmsnorm_b200 import PrefillBuffers, PrefillCall

    peaks = load_peaks()
    gi = make_gate_inputs(w)
    cu, span, k = w.cu_seqlens(), w.span_array(), w.budget_array()
    M, cu_kept = tg.tg_kept_count(cu, span, k)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

    hidden_h = bf16(gi["hidden"]).pin_memory()
    hidden = hidden_h.to(dev)
    Wg = tg.tg_gate_prepare(bf16(gi["gamma"]).to(dev), bf16(gi["W1"]).to(dev))
    b1 = torch.from_numpy(gi["b1"]).to(dev)
    w2 = torch.from_numpy(gi["w2"]).to(dev)
    layers_np = [make_attention_inputs(w, M, layer=l) for l in range(args.layers)]
    layers_h = [{"q": bf16(a["q"]).pin_memory(), "k": bf16(a["k"]).pin_memory(), "v": bf16(a["v"]).pin_memory(),
                 "g": torch.from_numpy(a["g"]).pin_memory(), "c": torch.from_numpy(a["c"]).pin_memory()}
                for a in layers_np]
    layers = [{key: t.to(dev) for key, t in L.items()} for L in layers_h]
    bufs = PrefillBuffers(w.T, w.D, M, args.layers, w.Hq, w.d, dev, with_hidden=True)
    call = PrefillCall(hidden, cu, span, k, Wg, b1, w2, gi["b2"], w.eps, layers, bufs, w.Hq, w.Hkv, w.d)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream(dev)

    def barrier():
        if ws > 1:
            dist.barrier()

    lib = tg.load()

    def sh_now():  # the current stream (a capture stream while a stage graph is recorded)
        return torch.cuda.current_stream(dev).cuda_stream

    B, T, D, I = w.B, w.T, w.D, w.I
    sm_scale = 1.0 / math.sqrt(w.d)
    L0 = layers[0]
    _ws_ptr = None if call.ws is None else call.ws.data_ptr()
    _ws_n = 0 if call.ws is None else call.ws.numel()
    # the product's kernels, one C-ABI call each, arguments bound once (host cost ~1 us per call)
    stage_calls = {
        "score": lambda: lib.tg_score(hidden.data_ptr(), call.cu.data_ptr(), call.sp.data_ptr(), B, T, D,
                                      Wg.data_ptr(), b1.data_ptr(), w2.data_ptr(), float(gi["b2"]), I, float(w.eps),
                                      bufs.scores.data_ptr(), sh_now()),
        "select": lambda: lib.tg_select_topk(bufs.scores.data_ptr(), call.cu.data_ptr(), call.sp.data_ptr(),
                                             call.kk.data_ptr(), B, T, bufs.keep.data_ptr(), call.ck.data_ptr(),
                                             bufs.kept_idx.data_ptr(), bufs.pos.data_ptr(), bufs.rank.data_ptr(),
                                             bufs.gls.data_ptr(), sh_now()),
        "gather": lambda: lib.tg_compact(hidden.data_ptr(), None, None, None, None, B, T, D, None, M,
                                         bufs.hidden_kept.data_ptr(), None, None, None, bufs.kept_idx.data_ptr(), sh_now()),
        "attention": lambda: lib.tg_gated_attention(L0["q"].data_ptr(), L0["k"].data_ptr(), L0["v"].data_ptr(),
                                                    call.ck.data_ptr(), B, M, call.max_M, w.Hq, w.Hkv, w.d,
                                                    bufs.pos.data_ptr(), bufs.rank.data_ptr(), bufs.gls.data_ptr(),
                                                    L0["g"].data_ptr(), L0["c"].data_ptr(), sm_scale,
                                                    bufs.out[0].data_ptr(), None, _ws_ptr, _ws_n, sh_now()),
    }

    # warm-up (also sets kernel attributes before any capture)
    for _ in range(args.warmup):
        call()
        for fn in stage_calls.values():
            assert fn() == 0
    torch.cuda.synchronize(dev)

    # the step as one CUDA graph: four kernels, no host work between them
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call()
        graph.replay()
        torch.cuda.synchronize(dev)
    step = graph.replay if graph is not None else call

    # ---------------- timed region: K whole-path steps
    clocks = ClockSampler(local)
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i)
        ev[i][0].record(st)
        step()
        ev[i][1].record(st)
    torch.cuda.synchronize(dev)
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]

    # ---------------- per-stage breakdown over K more steps (same stream, same kernels); each
    # stage replays a one-call CUDA graph, so that no host work (argument checks, tensor-map
    # encoding) sits between the events around it
    names = list(stage_calls)
    stage_graphs = {}
    if not args.no_graph:
        for nm in names:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                assert stage_calls[nm]() == 0
            stage_graphs[nm] = gr
        torch.cuda.synchronize(dev)
    run_stage = {nm: (stage_graphs[nm].replay if nm in stage_graphs else stage_calls[nm]) for nm in names}
    sev = {s: [] for s in names}
    for i in range(args.steps):
        flush.fill_(i)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        e[0].record(st)
        for n_i, nm in enumerate(names):
            run_stage[nm]()
            e[n_i + 1].record(st)
        for n_i, nm in enumerate(names):
            sev[nm].append((e[n_i], e[n_i + 1]))
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    stage_us = {s: 1e3 * float(np.mean([a.elapsed_time(b) for a, b in v])) for s, v in sev.items()}

    # ---------------- end to end: pinned host inputs in, result out, every step
    out_h = torch.empty((M, w.Hq, w.d), dtype=torch.bfloat16).pin_memory()
    idx_h = torch.empty(M, dtype=torch.int32).pin_memory()
    h2d = hidden_h.numel() * 2 + sum(L[key].numel() * L[key].element_size() for L in layers_h for key in L)
    d2h = out_h.numel() * 2 + idx_h.numel() * 4
    e2e_ev = []
    for i in range(args.warmup + args.steps):
        flush.fill_(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        hidden.copy_(hidden_h, non_blocking=True)
        for L, Lh in zip(layers, layers_h):
            for key in L:
                L[key].copy_(Lh[key], non_blocking=True)
        step()
        out_h.copy_(bufs.out[-1], non_blocking=True)
        idx_h.copy_(bufs.kept_idx, non_blocking=True)
        b.record(st)
        if i >= args.warmup:
            e2e_ev.append((a, b))
    torch.cuda.synchronize(dev)
    e2e_ms = float(np.sum([a.elapsed_time(b) for a, b in e2e_ev]))

    # ---------------- max over ranks
    t_total_ms, e2e_ms = max_over_ranks([float(np.sum(step_ms)), e2e_ms], ws, dev)

    ms_per_step = t_total_ms / args.steps
    value = job_rate(ws, w.T, args.steps, t_total_ms)
    e2e_value = job_rate(ws, w.T, args.steps, e2e_ms)

    flops, pairs = attention_flops(cu_kept, w.Hq, w.d)
    attn_tflops = flops / (stage_us["attention"] * 1e-6) / 1e12
    sb = stage_bytes(w, M)
    stage_gbs = {s: sb[s] / (stage_us[s] * 1e-6) / 1e9 for s in sb}
    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak = float(peaks["bf16_tflops"])
    # dominant kernel = the stage with the largest share of the step
    dom = max(stage_us, key=stage_us.get)
    traffic_tab = read_traffic_table()
    traffic = None
    key = (dom, w.name)
    if key in traffic_tab and traffic_tab[key][0] == source_sha(KERNEL_FILES[dom]):
        traffic = traffic_tab[key][1]
    if dom == "attention":
        roof = {"bound": "tensor", "achieved": attn_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": attn_tflops / tc_peak, "traffic": traffic, "kernel": "gated_attention",
                "algorithmic": f"{flops:.4g} FLOP per launch = 4*d*Hq*{pairs} causal pairs",
                "peak_source": f"{peaks['source']} bf16_tflops (burst)"}
    else:
        roof = {"bound": "hbm", "achieved": stage_gbs[dom], "peak": hbm_peak, "unit": "GB/s",
                "frac": stage_gbs[dom] / hbm_peak, "traffic": traffic, "kernel": dom,
                "algorithmic": f"{sb[dom]} bytes per launch", "peak_source": f"{peaks['source']} hbm_gbs"}
    s13_bytes = sb["score"] + sb["select"] + sb["gather"]
    s13_us = stage_us["score"] + stage_us["select"] + stage_us["gather"]

    next_rows = None
    if rank == 0 and not args.no_next_rows:
        main_ctx = {"w": w, "M": M, "cu_kept": cu_kept, "max_M": call.max_M, "kept_idx": bufs.kept_idx,
                    "layer": L0, "bufs": bufs, "gls_host": bufs.gls.cpu().numpy(), "ws": call.ws}
        next_rows = measure_next_rows(tg, dev, st, flush, main_ctx, peaks)

    sweep = None
    if rank == 0 and not args.no_sweep:
        sweep = measure_workload_sweep(tg, dev, st, flush, peaks, ms_per_step * 1e3)

    cpu_base = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        Wg_bits = oracle.gate_fold(gi["gamma"], gi["W1"])
        cpu_base = oracle_baseline(w, gi, Wg_bits, layers_np)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; Qwen3-1.7B gate-layer shapes)",
                "config": workload_config(w, args.layers),
                "roofline": roof,
                "gated_attn": {"tflops": attn_tflops, "frac_of_bf16_peak": attn_tflops / tc_peak,
                               "us": stage_us["attention"], "flops": flops},
                "score_select_compact": {"us": s13_us, "bytes": s13_bytes, "gbs": s13_bytes / (s13_us * 1e-6) / 1e9,
                                         "frac_of_hbm": s13_bytes / (s13_us * 1e-6) / 1e9 / hbm_peak},
                "stage_us": stage_us, "stage_gbs": stage_gbs,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                        "d2h_bytes_per_step": int(d2h)},
                "gpu_launches": args.steps * (3 + args.layers), "cuda_graph": graph is not None,
                "next_rows": next_rows, "workloads": sweep,
                "cpu_baseline": cpu_base, "clocks": clk, "peaks": {"source": peaks["source"],
                                                                   "hbm_gbs": hbm_peak, "bf16_tflops": tc_peak}}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tokengate", "reference"], default="tokengate")
    ap.add_argument("--workload", default="c2_32k_k2000")
    ap.add_argument("--layers", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the measurements of masked attention, KV gather, head_dim 256 and stacked gates")
    ap.add_argument("--no-graph", action="store_true", help="launch the step directly instead of a CUDA graph")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the other workloads (K sweep, 16k, 128k, varlen, 14-layer stack, dense 16k)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = get_config(args.workload)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
