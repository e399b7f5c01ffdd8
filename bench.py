"""Benchmark of the fused-QKV + grouped-query attention path on B200.

One step = the whole attention layer over one batch of the TinyLlama-1.1B-
shaped layer (hidden 2048, 32 query heads, 4 KV heads, head_dim 64, bf16,
RoPE theta 1e4):

  1. qkv_rope_project     prompt  x [4, 2048, 2048] -> q, K/V cache slots 0..2047
  2. gqa_attn_prefill     causal, 4 x 2048 queries over their 2048 keys
  3. gqa_o_proj_residual  attention output . W_o^T + x -> y [4, 2048, 2048]
  4. qkv_rope_project     one new token per sequence at position 2048
  5. gqa_attn_decode      4 sequences x 32 heads over 2049 cached keys
                          (split-KV partials + log-sum-exp combine)
  6. gqa_o_proj_residual  the new tokens' layer output

value = tokens processed per second (8192 prompt + 4 decode tokens per step,
summed over all GPUs).  Inputs are seeded synthetic tensors resident in HBM;
4 rotating input/output sets (~0.5 GB) keep every step's data out of L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the float64 CPU oracle (the correctness reference)
on a bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill attn TFLOPS & % BF16 peak; decode KV GB/s & % HBM; tokens/s per layer"
WORKLOAD = dict(name="tinyllama-1.1b-attention-layer-prefill4x2048+decode", B=4, S=2048, hidden=2048,
                n_heads=32, n_kv_heads=4, head_dim=64, theta=10000.0, cap=2112, causal=True)
N_ROT = 4
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_traffic():
    """DRAM bytes per launch from an ncu capture (profiles/dram_traffic.txt),
    valid only while the kernel source is unchanged (sha256 prefix)."""
    out = {}
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return out
    for line in open(p):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#"):
            name, src, sha, nbytes = parts[:4]
            fp = os.path.join(ROOT, "mqa_attention_qkv_b200", "csrc", src)
            if os.path.exists(fp) and hashlib.sha256(open(fp, "rb").read()).hexdigest()[:12] == sha:
                out[name] = float(nbytes)
    return out


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]),
                                 hw=f[5], hwt=f[6], swt=f[7], swp=f[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        loaded = [r["sm"] for r in rows if r["power"] > 0.3 * max(x["power"] for x in rows)] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def max_over_ranks(v: float, world: int, device) -> float:
    """The largest of the replicas' values (each measured on its own device
    clock): the slowest replica sets the job's time."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, world: int, steps: int, ms_total: float) -> float:
    """Units that all replicas processed, per second of the (max-over-ranks)
    timed region."""
    return units_per_step_per_rank * world * steps / (ms_total / 1e3)


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import mqa_attention_qkv_b200 as gqa
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    wl = WORKLOAD
    B, S, D, nh, nkv, hd, cap = (wl[k] for k in ("B", "S", "hidden", "n_heads", "n_kv_heads", "head_dim", "cap"))
    shape = W.LayerShape(D, nh, nkv, hd, wl["theta"])
    bf = torch.bfloat16
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)

    def randn(*s, std=1.0):
        return (torch.randn(*s, generator=gen, device=dev, dtype=torch.float32) * std).to(bf)

    sets = []
    for _ in range(N_ROT):
        st = dict(
            x=randn(B, S, D), w=randn(shape.n_qkv, D, std=0.02), x_dec=randn(B, 1, D),
            w_o=randn(D, nh * hd, std=0.02),
            y=torch.empty(B, S, D, dtype=bf, device=dev), y_dec=torch.empty(B, 1, D, dtype=bf, device=dev),
            q=torch.empty(B, nh, S, hd, dtype=bf, device=dev),
            kc=torch.zeros(B, nkv, cap, hd, dtype=bf, device=dev),
            vc=torch.zeros(B, nkv, cap, hd, dtype=bf, device=dev),
            o=torch.empty(B, S, nh, hd, dtype=bf, device=dev),
            q_dec=torch.empty(B, nh, 1, hd, dtype=bf, device=dev),
            o_dec=torch.empty(B, nh, hd, dtype=bf, device=dev),
        )
        sets.append(st)
    set_mb = _set_mb(sets[0])
    pos = torch.arange(S, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    pos_dec = torch.full((B, 1), S, dtype=torch.int32, device=dev)
    lens = torch.full((B,), S, dtype=torch.int32, device=dev)
    lens_dec = torch.full((B,), S + 1, dtype=torch.int32, device=dev)
    ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    names = ("qkv_prefill", "attn_prefill", "oproj_prefill", "qkv_decode", "attn_decode", "oproj_decode")

    def step(st, evs=None):
        def mark(i):
            if evs is not None:
                evs[i].record(stream)
        mark(0)
        gqa.qkv_rope_project(st["x"], st["w"], st.get("pos", pos), nh, nkv, hd, wl["theta"], st["q"], st["kc"], st["vc"],
                             stream)
        mark(1)
        gqa.gqa_attn_prefill(st["q"], st["kc"], st["vc"], lens, True, st["o"], stream=stream)
        mark(2)
        gqa.gqa_o_proj_residual(st["o"], st["w_o"], st["y"], residual=st["x"], stream=stream)
        mark(3)
        gqa.qkv_rope_project(st["x_dec"], st["w"], pos_dec, nh, nkv, hd, wl["theta"], st["q_dec"], st["kc"], st["vc"], stream)
        mark(4)
        gqa.gqa_attn_decode(st["q_dec"].view(B, nh, hd), st["kc"], st["vc"], lens_dec, st["o_dec"], ws, stream=stream)
        mark(5)
        gqa.gqa_o_proj_residual(st["o_dec"].view(B, 1, nh, hd), st["w_o"], st["y_dec"], residual=st["x_dec"],
                                stream=stream)
        mark(6)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier(device_ids=[local])

    # warm-up
    for i in range(args.warmup):
        step(sets[i % N_ROT])
    barrier()

    # timed region: K steps between two events on the launching stream.  An
    # event recorded between two kernels costs ~2.5 us on B200 (the next
    # kernel waits for it), so the per-kernel events are not in this region:
    # the same K steps run again right after it with an event between every
    # two kernels, and the per-kernel times (the roofline figures) come from
    # that second pass.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    n0 = gqa.gqa_launch_count()
    barrier()
    t_start.record(stream)
    for i in range(args.steps):
        step(sets[i % N_ROT])
    t_end.record(stream)
    barrier()
    launches = gqa.gqa_launch_count() - n0
    for i in range(args.steps):
        step(sets[i % N_ROT], evs[i])
    barrier()
    clk = clocks.stop()
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    per_kernel = {n: [evs[i][k].elapsed_time(evs[i][k + 1]) for i in range(args.steps)]
                  for k, n in enumerate(names)}
    ms_evented = max_over_ranks(evs[0][0].elapsed_time(evs[-1][-1]), world, dev)

    tokens_per_step = B * S + B
    ms_step = ms_total / args.steps
    value = whole_job_rate(tokens_per_step, world, args.steps, ms_total)

    # algorithmic work per launch
    peaks, peak_src = load_peaks()
    flops = {
        "qkv_prefill": 2.0 * B * S * D * shape.n_qkv,
        "attn_prefill": 4.0 * B * nh * S * S * hd / 2,           # causal counted as half
        "oproj_prefill": 2.0 * B * S * nh * hd * D,
    }
    bytes_ = {
        "qkv_decode": 2.0 * (shape.n_qkv * D + B * D + B * shape.n_qkv),
        "attn_decode": 2.0 * (2 * B * nkv * (S + 1) * hd + 2 * B * nh * hd),
        "oproj_decode": 2.0 * (D * nh * hd + B * nh * hd + 2 * B * D),
    }
    mean_ms = {n: statistics.mean(v) for n, v in per_kernel.items()}
    dominant = max(mean_ms, key=mean_ms.get)
    traffic = kernel_traffic()
    bf16_peak = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])

    def roof(n):
        if n in flops:
            a = flops[n] / (mean_ms[n] / 1e3) / 1e12
            return {"bound": "tensor", "achieved": round(a, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                    "frac": round(a / bf16_peak, 4), "traffic": traffic.get(n), "kernel": n,
                    "peak_source": f"{peak_src} bf16_tflops (burst)"}
        a = bytes_[n] / (mean_ms[n] / 1e3) / 1e9
        return {"bound": "hbm", "achieved": round(a, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(a / hbm_peak, 4), "traffic": traffic.get(n), "kernel": n,
                "peak_source": f"{peak_src} hbm_gbs"}

    roofline = roof(dominant)
    kernels = {n: {"ms": round(mean_ms[n], 4), **{k: v for k, v in roof(n).items() if k in ("achieved", "unit", "frac")}}
               for n in names}

    # end to end through the public API: pinned host inputs -> device -> path -> host outputs.
    # Three streams form a pipeline over the N_ROT sets: step i's inputs are
    # copied in while step i-1 computes and step i-2's outputs are copied out.
    e2e = None
    if not args.no_e2e:
        hx = [sets[i]["x"].cpu().pin_memory() for i in range(N_ROT)]
        hxd = [sets[i]["x_dec"].cpu().pin_memory() for i in range(N_ROT)]
        ho = [torch.empty(B, S, D, dtype=bf).pin_memory() for _ in range(N_ROT)]
        hod = [torch.empty(B, 1, D, dtype=bf).pin_memory() for _ in range(N_ROT)]
        hpos = pos.cpu().pin_memory()
        for st in sets:
            st["pos"] = torch.empty_like(pos)
        in_st, out_st = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(N_ROT)]     # set's inputs landed
        ev_done = [torch.cuda.Event() for _ in range(N_ROT)]   # set's step computed
        ev_out = [torch.cuda.Event() for _ in range(N_ROT)]    # set's outputs copied out
        used = [False] * N_ROT

        def e2e_step(i):
            k = i % N_ROT
            st = sets[k]
            with torch.cuda.stream(in_st):
                if used[k]:
                    in_st.wait_event(ev_done[k])     # the previous step on this set has read its inputs
                st["x"].copy_(hx[k], non_blocking=True)
                st["x_dec"].copy_(hxd[k], non_blocking=True)
                st["pos"].copy_(hpos, non_blocking=True)
                ev_in[k].record(in_st)
            stream.wait_event(ev_in[k])
            if used[k]:
                stream.wait_event(ev_out[k])         # ... and its outputs have left the device
            step(st)
            ev_done[k].record(stream)
            with torch.cuda.stream(out_st):
                out_st.wait_event(ev_done[k])
                ho[k].copy_(st["y"], non_blocking=True)         # the layer's output
                hod[k].copy_(st["y_dec"], non_blocking=True)
                ev_out[k].record(out_st)
            used[k] = True

        for i in range(args.warmup):
            e2e_step(i)
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(in_st)                              # the first copy in opens the region
        for i in range(args.steps):
            e2e_step(i)
        b_.record(out_st)                            # the last copy out closes it
        barrier()
        ms_e2e = max_over_ranks(a.elapsed_time(b_), world, dev)
        h2d = hx[0].numel() * 2 + hxd[0].numel() * 2 + hpos.numel() * 4
        d2h = ho[0].numel() * 2 + hod[0].numel() * 2
        e2e = {"value": round(whole_job_rate(tokens_per_step, world, args.steps, ms_e2e), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(ms_e2e / args.steps, 4),
               "overlap": f"copies in, compute and copies out on three streams over {N_ROT} buffer sets"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(budget_s=args.cpu_budget)
    wls = None
    step_check = None
    if rank == 0 and world == 1 and not args.no_workloads:
        step_check = check_layer_step(sets[0], B, S, nh, nkv, hd, wl["theta"])
        del sets
        only = set(args.workloads.split(",")) if args.workloads else None
        wls = measure_workloads(dev, {"hbm_gbs": hbm_peak, "bf16_tflops": bf16_peak}, only=only)
        if only is None or "tiny" in only:
            wls["tiny_fp32_layer"] = check_tiny_fp32(dev)

    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank != 0:
        return
    attn = kernels["attn_prefill"]
    dec = kernels["attn_decode"]
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) hidden states, N(0,0.02) weights)",
        "config": {"workload": wl["name"], "global_batch": B * world, "seq_len": S, "hidden": D,
                   "n_heads": nh, "n_kv_heads": nkv, "head_dim": hd, "causal": True,
                   "decode_kv_len": S + 1, "parallelism": f"replicas x{world}",
                   "l2": f"{N_ROT} rotating input/output sets of ~{set_mb:.0f} MB (> 126 MB L2)"},
        "prefill_attn_tflops": attn["achieved"], "prefill_attn_frac_bf16_peak": attn["frac"],
        "decode_kv_gbs": dec["achieved"], "decode_frac_hbm": dec["frac"],
        "kernels": kernels,
        "kernel_timing": {"pass": "the same K steps again, right after the timed region, with a CUDA event "
                                  "between every two kernels on the launching stream",
                          "ms_per_step": round(ms_evented / args.steps, 4)},
        "roofline": roofline, "gpu_launches": int(launches), "parity": step_check,
        "clocks": clk, "e2e": e2e, "cpu_baseline": cpu, "workloads": wls,
    }
    print(json.dumps(line))


def _set_mb(st):
    return sum(t.numel() * t.element_size() for t in st.values()) / 1e6


# ---------------------------------------------------------------------------
# the other workloads of the metric, measured kernel by kernel
# ---------------------------------------------------------------------------
def measure_workloads(dev, peaks, iters=10, only=None, checks=True):
    """Llama-2-7B-shaped batched decode (B 64, 32 query heads, hd 128, ragged
    KV 512..8192, MHA/GQA/MQA caches, contiguous and in shuffled 64-key
    pages): KV GB/s; 8K-token prefill (B 2, 16
    heads, hd 128, KV heads 16/4, causal and not): TFLOP/s; the MQA generation
    loop (B 8, hidden 6144, 48 heads, 1 KV head, prompt 16 + 1024 steps):
    tokens/s; the TinyLlama layer's smaller prefill shapes (1 x 128, 8 x 512):
    projection + attention tokens/s; the MHA -> GQA mean-pool weight
    transform on the Llama-2-7B projection (32 -> 8 KV heads): GB/s.  Each
    kernel is timed alone with CUDA events, L2 flushed before every timed call
    (a 512 MB write), median of `iters`.  ``only``: a set of section names
    (decode, decode_mqa, prefill8k, generate, small, varlen, meanpool) to measure; None =
    all.  ``checks``: also compare sampled outputs of each config with the
    float64 oracle and time the oracle on the host cores (scaled linearly
    from the sample to the whole config)."""
    import numpy as np
    import torch

    import mqa_attention_qkv_b200 as gqa
    import workloads as W

    bf = torch.bfloat16
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)

    def back_to_back(fns, n=12):
        """ms per call of n calls issued back to back, cycling over ``fns``
        (each reads its own data, together larger than L2), between two
        events: the launches overlap the previous kernel's tail as in a
        decode loop over layers, and no call finds its data in L2."""
        for fn in fns:
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n):
            fns[i % len(fns)]()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / n

    def timed(fn, flush_l2=True):
        ts = []
        for i in range(iters + 2):
            if flush_l2:
                flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            if i >= 2:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    out = {}
    hbm, bf16_peak = peaks["hbm_gbs"], peaks["bf16_tflops"]

    want = (lambda name: only is None or name in only)

    # ---- batched decode
    if want("decode") or want("decode_mqa"):
        wl = W.LLAMA2_DECODE
        e = wl.extra
        B, nh, hd, cap = e["batch"], wl.shape.n_heads, wl.shape.head_dim, e["cap"]
        lens_np = W.ragged_lengths(B, e["kv_lo"], e["kv_hi"], wl.seed)
        lens = torch.from_numpy(lens_np).to(dev)
        q = torch.randn(B, nh, hd, generator=gen, device=dev).to(bf)
        dec = {}
        # "decode_mqa" alone: only the one-KV-head case (a small problem for a profiler)
        for nkv in (e["n_kv_heads_cases"] if want("decode") else (1,)):
            kc = torch.randn(B, nkv, cap, hd, generator=gen, device=dev, dtype=torch.float32).to(bf)
            vc = torch.randn(B, nkv, cap, hd, generator=gen, device=dev, dtype=torch.float32).to(bf)
            o = torch.empty(B, nh, hd, dtype=bf, device=dev)
            ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device=dev)
            ms = timed(lambda: gqa.gqa_attn_decode(q, kc, vc, lens, o, ws, stream=stream))
            nbytes = 2.0 * (2 * nkv * hd * float(lens_np.sum()) + 2 * B * nh * hd)
            gbs = nbytes / (ms / 1e3) / 1e9
            dec[f"nkv{nkv}"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                                "bytes": int(nbytes)}
            # back to back: the MQA cache (168 MB used) is close to L2's size, so two copies alternate
            sets = [(kc, vc)] if nkv > 1 else [(kc, vc), (kc.clone(), vc.clone())]
            ms_b = back_to_back([lambda kv=kv: gqa.gqa_attn_decode(q, kv[0], kv[1], lens, o, ws, stream=stream)
                                 for kv in sets])
            gbs_b = nbytes / (ms_b / 1e3) / 1e9
            dec[f"nkv{nkv}"].update({"ms_back_to_back": round(ms_b, 4), "GB/s_back_to_back": round(gbs_b, 1),
                                     "frac_hbm_back_to_back": round(gbs_b / hbm, 4)})
            del sets
            if nkv == 1:   # MQA: 143 MB of K/V fits in L2, so the warm figure differs
                ms_w = timed(lambda: gqa.gqa_attn_decode(q, kc, vc, lens, o, ws, stream=stream), flush_l2=False)
                dec["nkv1"].update({"ms_warm_l2": round(ms_w, 4),
                                    "GB/s_warm_l2": round(nbytes / (ms_w / 1e3) / 1e9, 1)})
            if checks:
                dec[f"nkv{nkv}"].update(check_decode(q, kc, vc, lens_np, o, nkv))
            # the same cache cut into 64-key pages, shuffled over the page pool
            ps, maxp = 64, cap // 64
            perm = torch.randperm(B * maxp, generator=torch.Generator().manual_seed(nkv)).to(dev)
            table = perm.view(B, maxp).to(torch.int32).contiguous()

            def paged(c):
                pool = torch.empty(B * maxp, nkv, ps, hd, dtype=bf, device=dev)
                pool[perm] = c.view(B, nkv, maxp, ps, hd).transpose(1, 2).reshape(B * maxp, nkv, ps, hd)
                return pool

            kp, vp = paged(kc), paged(vc)
            del kc, vc
            ms = timed(lambda: gqa.gqa_attn_decode_paged(q, kp, vp, table, lens, o, ws, stream=stream))
            gbs = nbytes / (ms / 1e3) / 1e9
            dec[f"nkv{nkv}_paged64"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                                        "bytes": int(nbytes)}
            sets = [(kp, vp)] if nkv > 1 else [(kp, vp), (kp.clone(), vp.clone())]
            ms_b = back_to_back([lambda kv=kv: gqa.gqa_attn_decode_paged(q, kv[0], kv[1], table, lens, o, ws,
                                                                         stream=stream) for kv in sets])
            gbs_b = nbytes / (ms_b / 1e3) / 1e9
            dec[f"nkv{nkv}_paged64"].update({"ms_back_to_back": round(ms_b, 4), "GB/s_back_to_back": round(gbs_b, 1),
                                             "frac_hbm_back_to_back": round(gbs_b / hbm, 4)})
            del sets
            del kp, vp
        out["llama2_decode_b64"] = dec

    # ---- long-context prefill
    if want("prefill8k"):
        wl = W.LONG_PREFILL
        B, S = wl.batch_seq[0]
        nh, hd = wl.shape.n_heads, wl.shape.head_dim
        lp = {}
        for nkv in wl.extra["n_kv_heads_cases"]:
            qkv = []
            for tid, H in enumerate((nh, nkv, nkv)):   # N(0,1), 0.1% of each tensor's channels x20
                t = torch.randn(B, H, S, hd, generator=gen, device=dev)
                for c in W.outlier_channels(H * hd, wl.extra["outlier_frac"], wl.seed + nkv, tid):
                    hh, d = divmod(int(c), hd)
                    t[:, hh, :, d] *= wl.extra["outlier_scale"]
                qkv.append(t.to(bf))
            q, k, v = qkv
            o = torch.empty(B, S, nh, hd, dtype=bf, device=dev)
            ln = torch.full((B,), S, dtype=torch.int32, device=dev)
            for causal in (True, False):
                ms = timed(lambda: gqa.gqa_attn_prefill(q, k, v, ln, causal, o, stream=stream))
                fl = 4.0 * B * nh * S * S * hd * (0.5 if causal else 1.0)
                tf = fl / (ms / 1e3) / 1e12
                key = f"nkv{nkv}_{'causal' if causal else 'full'}"
                lp[key] = {"ms": round(ms, 4), "TFLOP/s": round(tf, 1), "frac_bf16": round(tf / bf16_peak, 4)}
                if checks:
                    lp[key].update(check_long_prefill(q, k, v, o, causal, nkv, wl))
            # FP8 (e4m3) with incoherent processing: quantise (rotation, amax, codes), then attention
            q8 = torch.empty(B, nh, S, hd, dtype=torch.uint8, device=dev)
            k8 = torch.empty(B, nkv, S, hd, dtype=torch.uint8, device=dev)
            v8t = torch.empty(B, nkv, hd, S, dtype=torch.uint8, device=dev)
            amax = torch.empty(3, device=dev)
            signs = np.where(np.random.default_rng([wl.seed, 9]).integers(0, 2, hd) == 1, -1, 1).tolist()
            ms_q = timed(lambda: gqa.gqa_fp8_quantize_qkv(q, k, v, ln, q8, k8, v8t, amax, signs=signs, stream=stream))
            qbytes = 2.0 * 2 * (q.numel() + 2 * k.numel()) + (q.numel() + 2 * k.numel())   # two bf16 passes + codes
            fp8_peak = 2.0 * bf16_peak
            for causal in (True, False):
                ms = timed(lambda: gqa.gqa_attn_prefill_fp8(q8, k8, v8t, amax, ln, causal, o, stream=stream))
                fl = 4.0 * B * nh * S * S * hd * (0.5 if causal else 1.0)
                tf = fl / (ms / 1e3) / 1e12
                key = f"fp8_nkv{nkv}_{'causal' if causal else 'full'}"
                lp[key] = {"ms": round(ms, 4), "TFLOP/s": round(tf, 1), "frac_fp8": round(tf / fp8_peak, 4),
                           "quantize_ms": round(ms_q, 4),
                           "quantize_GB/s": round(qbytes / (ms_q / 1e3) / 1e9, 1),
                           "fp8_peak_note": "2 x the bf16 peak (the nominal fp8/bf16 ratio)"}
                if checks:
                    lp[key].update(check_fp8_error(q, k, v, o, ln, causal, nkv, signs, q8, k8, v8t, amax, stream))
        out["long_prefill_2x8192"] = lp

    # ---- MQA generation loop (prompt 16, 1024 steps), one timed region
    if want("generate"):
        wl = W.MQA_GENERATE
        sh, e = wl.shape, wl.extra
        B, P, T, cap = e["batch"], e["prompt"], e["steps"], e["cap"]
        nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
        w = (torch.randn(sh.n_qkv, sh.hidden, generator=gen, device=dev) * 0.02).to(bf)
        xp = torch.randn(B, P, sh.hidden, generator=gen, device=dev).to(bf)
        xs = torch.randn(T, B, 1, sh.hidden, generator=gen, device=dev).to(bf)
        kc = torch.zeros(B, nkv, cap, hd, dtype=bf, device=dev)
        vc = torch.zeros_like(kc)
        qp = torch.empty(B, nh, P, hd, dtype=bf, device=dev)
        op = torch.empty(B, P, nh, hd, dtype=bf, device=dev)
        qt = torch.empty(B, nh, 1, hd, dtype=bf, device=dev)
        ot = torch.empty(T, B, nh, hd, dtype=bf, device=dev)
        posp = torch.arange(P, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
        pos_steps = (P + torch.arange(T, dtype=torch.int32, device=dev)).view(T, 1, 1).expand(T, B, 1).contiguous()
        len_steps = (P + 1 + torch.arange(T, dtype=torch.int32, device=dev)).view(T, 1).expand(T, B).contiguous()
        lp_ = torch.full((B,), P, dtype=torch.int32, device=dev)
        ws = torch.zeros(gqa.gqa_attn_decode_workspace_size(B, nh, nkv, hd, cap), dtype=torch.uint8, device=dev)

        def gen_loop():
            st = torch.cuda.current_stream(dev)   # the capture stream while a graph is being recorded
            gqa.qkv_rope_project(xp, w, posp, nh, nkv, hd, sh.rope_theta, qp, kc, vc, st)
            gqa.gqa_attn_prefill(qp, kc, vc, lp_, True, op, stream=st)
            for t in range(T):
                gqa.qkv_rope_project(xs[t], w, pos_steps[t], nh, nkv, hd, sh.rope_theta, qt, kc, vc, st)
                gqa.gqa_attn_decode(qt.view(B, nh, hd), kc, vc, len_steps[t], ot[t], ws, stream=st)

        gen_loop()
        ms_direct = timed_once(gen_loop, stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            gen_loop()
        graph.replay()
        ms_graph = timed_once(graph.replay, stream)
        toks = B * (P + T)
        per_step_bytes = 2.0 * sh.n_qkv * sh.hidden
        # one step (t = 512) alone after an L2 flush: the cold counterpart of
        # the graph loop, in which W_qkv can stay L2-resident from step to step
        t_mid = T // 2

        def one_step():
            gqa.qkv_rope_project(xs[t_mid], w, pos_steps[t_mid], nh, nkv, hd, sh.rope_theta, qt, kc, vc, stream)
            gqa.gqa_attn_decode(qt.view(B, nh, hd), kc, vc, len_steps[t_mid], ot[t_mid], ws, stream=stream)

        us_cold = timed(one_step) * 1e3
        out["mqa_generate_b8_p16_g1024"] = {
            "ms_direct": round(ms_direct, 3), "ms_graph": round(ms_graph, 3),
            "tokens_per_s_direct": round(toks / (ms_direct / 1e3), 1),
            "tokens_per_s_graph": round(toks / (ms_graph / 1e3), 1),
            "us_per_step_graph_warm_l2": round(ms_graph * 1e3 / T, 2),
            "us_per_step_cold_l2": round(us_cold, 2),
            "weight_stream_GB/s_graph": round(per_step_bytes * T / (ms_graph / 1e3) / 1e9, 1),
            "note": "W_qkv (78.6 MB) is re-read every step and may stay L2-resident across steps in the graph loop"}
        del graph            # every replay and the single step recompute the same values
        torch.cuda.synchronize(dev)
        if checks:
            out["mqa_generate_b8_p16_g1024"].update(check_generation(xp, xs, w, ot, sh, P, T))

    # ---- TinyLlama layer, the smaller prefill shapes of the same config
    if want("small"):
        wl = W.TINYLLAMA_PREFILL
        sh = wl.shape
        w = (torch.randn(sh.n_qkv, sh.hidden, generator=gen, device=dev) * 0.02).to(bf)
        small = {}
        for (B, S) in wl.batch_seq:
            if B * S >= 8192:
                continue            # the 4 x 2048 shape is the bench step itself
            x = torch.randn(B, S, sh.hidden, generator=gen, device=dev).to(bf)
            pos = torch.arange(S, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
            q = torch.empty(B, sh.n_heads, S, sh.head_dim, dtype=bf, device=dev)
            kc = torch.empty(B, sh.n_kv_heads, S, sh.head_dim, dtype=bf, device=dev)
            vc = torch.empty_like(kc)
            o = torch.empty(B, S, sh.n_heads, sh.head_dim, dtype=bf, device=dev)
            ln = torch.full((B,), S, dtype=torch.int32, device=dev)
            ms_p = timed(lambda: gqa.qkv_rope_project(x, w, pos, sh.n_heads, sh.n_kv_heads, sh.head_dim,
                                                      sh.rope_theta, q, kc, vc, stream))
            ms_a = timed(lambda: gqa.gqa_attn_prefill(q, kc, vc, ln, True, o, stream=stream))
            fl_p = 2.0 * B * S * sh.hidden * sh.n_qkv
            fl_a = 4.0 * B * sh.n_heads * S * S * sh.head_dim * 0.5
            small[f"{B}x{S}"] = {"qkv_ms": round(ms_p, 4), "qkv_TFLOP/s": round(fl_p / (ms_p / 1e3) / 1e12, 1),
                                 "attn_ms": round(ms_a, 4), "attn_TFLOP/s": round(fl_a / (ms_a / 1e3) / 1e12, 1),
                                 "tokens_per_s": round(B * S / ((ms_p + ms_a) / 1e3), 1)}
        out["tinyllama_prefill_small"] = small

    # ---- packed variable-length prefill: the TinyLlama layer's attention over
    # 16 ragged causal sequences of 64..960 tokens, packed without padding
    if want("varlen"):
        sh = W.TINYLLAMA_PREFILL.shape
        nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
        seq = W.ragged_lengths(16, 64, 960, W.TINYLLAMA_PREFILL.seed)
        cu = torch.from_numpy(np.concatenate([[0], np.cumsum(seq)]).astype(np.int32)).to(dev)
        tot = int(seq.sum())
        q = torch.randn(tot, nh, hd, generator=gen, device=dev).to(bf)
        k = torch.randn(tot, nkv, hd, generator=gen, device=dev).to(bf)
        v = torch.randn(tot, nkv, hd, generator=gen, device=dev).to(bf)
        o = torch.empty_like(q)
        try:
            ms = timed(lambda: gqa.gqa_attn_prefill_varlen(q, k, v, cu, cu, int(seq.max()), True, o, stream=stream))
            # exact visible (query, key) pairs of the causal sequences
            fl = 4.0 * nh * hd * float(np.sum(seq.astype(np.float64) * (seq + 1) / 2))
            tf = fl / (ms / 1e3) / 1e12
            out["varlen_prefill_tinyllama_16_ragged"] = {
                "ms": round(ms, 4), "TFLOP/s": round(tf, 1), "frac_bf16": round(tf / bf16_peak, 4),
                "tokens": tot, "tokens_per_s": round(tot / (ms / 1e3), 1)}
        except Exception as exc:   # an auxiliary line: report it, keep the bench line
            out["varlen_prefill_tinyllama_16_ragged"] = {"error": str(exc)}

    # ---- MHA -> GQA weight transform on the Llama-2-7B projection (32 heads -> 8 KV heads)
    if want("meanpool"):
        nh, hd, D, nkv = 32, 128, 4096, 8
        w_mha = (torch.randn(3 * nh * hd, D, generator=gen, device=dev) * 0.02).to(bf)
        w_gqa = torch.empty((nh + 2 * nkv) * hd, D, dtype=bf, device=dev)
        ms = timed(lambda: gqa.gqa_meanpool_kv_heads(w_mha, nh, nkv, hd, w_gqa, stream=stream))
        nbytes = 2.0 * D * hd * (3 * nh + nh + 2 * nkv)
        gbs = nbytes / (ms / 1e3) / 1e9
        out["mha_to_gqa_meanpool_llama2_7b"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1),
                                                "frac_hbm": round(gbs / hbm, 4), "bytes": int(nbytes)}
    return out


# ---------------------------------------------------------------------------
# per-config parity against the oracle, and the oracle's own timing
# ---------------------------------------------------------------------------
def err_over_tol(got, want, dtype, col_scale=None):
    """(max |err|, max of |err| / tolerance) under the parity tests' gates:
    float32 |err| <= 1e-4 max|ref|; bf16 |err| <= 2e-2 min(1, RMS of the
    row) + half a bf16 ulp of the reference, per element (rows = last axis),
    outlier channels on their own scale."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    if dtype == "f32":
        tol = 1e-4 * max(float(np.max(np.abs(want))), 1e-30)
        return float(err.max()), float(err.max()) / tol
    sc = np.ones_like(want) if col_scale is None else np.broadcast_to(col_scale, want.shape)
    unit = want / sc
    _, ex = np.frexp(np.abs(want))
    half_ulp = np.where(want != 0, np.ldexp(1.0, ex - 9), 0.0)
    lim = 2e-2 * sc * np.minimum(1.0, np.sqrt(np.mean(unit * unit, axis=-1, keepdims=True))) + half_ulp
    return float(err.max()), float(np.max(err / np.maximum(lim, 1e-30)))


def _to64(t):
    import numpy as np
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_seconds(fn, threads=None):
    """Wall time of ``fn()`` on the host cores (``threads``: BLAS thread cap)."""
    from threadpoolctl import threadpool_limits
    if threads is None:
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0
    with threadpool_limits(limits=threads):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0


def check_tiny_fp32(dev, iters=20):
    """The tiny fp32 layer: projection, causal prefill and output projection,
    every element against the oracle; GPU microseconds (median of `iters`
    runs), oracle seconds with all host cores and with one thread."""
    import numpy as np
    import torch

    import mqa_attention_qkv_b200 as gqa
    import workloads as W
    from oracle import gqa_ref as ref
    wl = W.TINY_FP32
    sh = wl.shape
    B, S = wl.batch_seq[0]
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    x, w, pos = W.layer_inputs(sh, B, S, seed=wl.seed, dtype="f32")
    w_o = W.output_weight(sh, wl.seed, "f32")
    f32 = torch.float32
    xd, wd, wod = (torch.from_numpy(t.store).to(dev) for t in (x, w, w_o))
    posd = torch.from_numpy(pos).to(dev)
    kc = torch.zeros(B, nkv, S, hd, dtype=f32, device=dev)
    vc = torch.zeros_like(kc)
    q = torch.empty(B, nh, S, hd, dtype=f32, device=dev)
    o = torch.empty(B, S, nh, hd, dtype=f32, device=dev)
    y = torch.empty(B, S, sh.hidden, dtype=f32, device=dev)
    lens = torch.full((B,), S, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def layer():
        gqa.qkv_rope_project(xd, wd, posd, nh, nkv, hd, sh.rope_theta, q, kc, vc, stream)
        gqa.gqa_attn_prefill(q, kc, vc, lens, True, o, stream=stream)
        gqa.gqa_o_proj_residual(o, wod, y, residual=xd, stream=stream)

    layer()
    ts = []
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        layer()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)

    z = np.zeros((B, nkv, S, hd))

    def oracle():
        q_r, kc_r, vc_r = ref.qkv_rope_project(x.f64, w.f64, pos, nh, nkv, hd, sh.rope_theta, z, z)
        o_r = ref.prefill_attention(q_r, kc_r, vc_r, np.full(B, S), True)
        return o_r, ref.output_projection(o_r, w_o.f64, x.f64)

    o_r, y_r = oracle()
    e_o = err_over_tol(_to64(o), o_r, "f32")
    e_y = err_over_tol(_to64(y), y_r, "f32")
    return {"us": round(statistics.median(ts), 2), "max_err": max(e_o[0], e_y[0]),
            "err_over_tol": round(max(e_o[1], e_y[1]), 4), "checked": "every element of o and y",
            "oracle_s": round(oracle_seconds(oracle), 4), "oracle_s_1thread": round(oracle_seconds(oracle, 1), 4)}


def check_layer_step(st, B, S, nh, nkv, hd, theta, rows=48):
    """The bench step's layer output on sampled tokens of sequence 0 and the
    decode token, against the oracle's chain on the same (device-drawn)
    inputs; plus the oracle's time for the whole 4 x 2048 step, scaled
    linearly from sampled query rows (all cores and one thread)."""
    import numpy as np

    from oracle import gqa_ref as ref
    x, w, w_o, xd = _to64(st["x"][0:1]), _to64(st["w"]), _to64(st["w_o"]), _to64(st["x_dec"][0:1])
    cap = S + 1
    z = np.zeros((1, nkv, cap, hd))
    pos = np.arange(S, dtype=np.int32)[None]
    rb = ref.round_bf16

    def chain(n_rows):
        srows = np.linspace(0, S - 1, n_rows).round().astype(int)
        q, kc, vc = ref.qkv_rope_project(x, w, pos, nh, nkv, hd, theta, z, z)
        rr = [(0, h, int(s)) for s in srows for h in range(nh)]
        o = np.asarray(ref.prefill_attention(rb(q), rb(kc), rb(vc), np.array([S]), True, rows=rr))
        y = ref.output_projection(rb(o.reshape(n_rows, nh, hd)), w_o, x[0, srows])
        qd, kc, vc = ref.qkv_rope_project(xd, w, np.array([[S]], dtype=np.int32), nh, nkv, hd, theta, kc, vc)
        od = ref.decode_attention(rb(qd[:, :, 0]), rb(kc), rb(vc), np.array([S + 1]))
        yd = ref.output_projection(rb(od)[:, None], w_o, xd[:, 0:1])
        return srows, y, yd

    srows, y_r, yd_r = chain(rows)
    e1 = err_over_tol(_to64(st["y"][0])[srows], y_r, "bf16")
    e2 = err_over_tol(_to64(st["y_dec"][0:1]), yd_r, "bf16")
    out = {"max_err": max(e1[0], e2[0]), "err_over_tol": round(max(e1[1], e2[1]), 4),
           "checked": f"layer output of {rows} query rows of sequence 0 and the decode token"}
    for key, th in (("oracle_s", None), ("oracle_s_1thread", 1)):
        t16, t64 = oracle_seconds(lambda: chain(16), th), oracle_seconds(lambda: chain(64), th)
        per_row = max(0.0, (t64 - t16) / 48)
        out[key] = round(B * (t16 - 16 * per_row + S * per_row), 2)
    out["oracle_note"] = "whole 4 x 2048 step, scaled linearly from 16- and 64-row samples of one sequence"
    return out


def check_decode(q, kc, vc, lens_np, o, nkv, pairs=8):
    """Sampled (sequence, head) rows of the batched decode against the oracle
    (inputs copied from the device); oracle time for all B x 32 rows, scaled
    by the keys each row reads (all cores and one thread)."""
    import numpy as np

    from oracle import gqa_ref as ref
    B, nh, hd = q.shape
    g = nh // nkv
    r = np.random.default_rng(11)
    sel = [(int(np.argmax(lens_np)), 0), (int(np.argmin(lens_np)), nh - 1)]
    sel += [(int(r.integers(B)), int(r.integers(nh))) for _ in range(pairs - 2)]
    data = [(_to64(q[b, h]), _to64(kc[b, h // g, :int(lens_np[b])]), _to64(vc[b, h // g, :int(lens_np[b])]))
            for b, h in sel]
    got = np.stack([_to64(o[b, h]) for b, h in sel])
    rows = lambda: [ref.attend_row(qv, K, V)[0] for qv, K, V in data]   # noqa: E731
    want = np.stack(rows())
    e = err_over_tol(got, want, "bf16")
    scale = nh * float(lens_np.sum()) / sum(int(lens_np[b]) for b, _ in sel)
    return {"max_err": e[0], "err_over_tol": round(e[1], 4), "checked": f"{len(sel)} (sequence, head) rows",
            "oracle_s": round(oracle_seconds(rows) * scale, 3),
            "oracle_s_1thread": round(oracle_seconds(rows, 1) * scale, 3)}


def check_long_prefill(q, k, v, o, causal, nkv, wl, n=12):
    """Sampled query rows of the 8K prefill (outlier inputs) against the
    oracle, outlier V channels on their x20 scale; oracle time for every row,
    scaled by the keys each row sees."""
    import numpy as np

    import workloads as W
    from oracle import gqa_ref as ref
    B, nh, S, hd = q.shape
    g = nh // nkv
    r = np.random.default_rng(13)
    sel = [(0, 0, 0), (B - 1, nh - 1, S - 1)] + [(int(r.integers(B)), int(r.integers(nh)), int(r.integers(S)))
                                                  for _ in range(n - 2)]
    vis = [s + 1 if causal else S for _, _, s in sel]
    data = [(_to64(q[b, h, s]), _to64(k[b, h // g, :L]), _to64(v[b, h // g, :L])) for (b, h, s), L in zip(sel, vis)]
    rows = lambda: [ref.attend_row(qv, K, V)[0] for qv, K, V in data]   # noqa: E731
    want = np.stack(rows())
    got = np.stack([_to64(o[b, s, h]) for b, h, s in sel])
    vscale = np.ones(nkv * hd)
    vscale[W.outlier_channels(nkv * hd, wl.extra["outlier_frac"], wl.seed + nkv, 2)] = wl.extra["outlier_scale"]
    vscale = vscale.reshape(nkv, hd)
    e = err_over_tol(got, want, "bf16", np.stack([vscale[h // g] for _, h, _ in sel]))
    total = B * nh * (S * (S + 1) / 2 if causal else S * S)
    scale = total / sum(vis)
    return {"max_err": e[0], "err_over_tol": round(e[1], 4), "checked": f"{len(sel)} query rows",
            "oracle_s": round(oracle_seconds(rows) * scale, 2)}


def check_generation(xp, xs, w, ot, sh, P, T, seqs=(0, 7), steps=(0, 511, 1023)):
    """Decode outputs of sampled steps of the generation loop against the
    oracle, which projects the sequence's own tokens (inputs copied from the
    device) to rebuild its K/V cache; oracle time for the whole loop (all
    8 x 1040 tokens projected, every step's attention), scaled from one
    sequence."""
    import numpy as np

    from oracle import gqa_ref as ref
    nh, nkv, hd = sh.n_heads, sh.n_kv_heads, sh.head_dim
    W_ = _to64(w)
    rb = ref.round_bf16
    errs = []

    def one_seq(b, which, check):
        x = np.concatenate([_to64(xp[b]), _to64(xs[:, b, 0])], axis=0)[None]      # [1, P + T, hidden]
        pos = np.arange(P + T, dtype=np.int32)[None]
        z = np.zeros((1, nkv, P + T, hd))
        q, kc, vc = ref.qkv_rope_project(x, W_, pos, nh, nkv, hd, sh.rope_theta, z, z)
        for t in which:
            want = ref.decode_attention(rb(q[:, :, P + t]), rb(kc), rb(vc), np.array([P + t + 1]))
            if check:
                errs.append(err_over_tol(_to64(ot[t, b]), want[0], "bf16"))

    for b in seqs:
        one_seq(b, steps, True)
    # one sequence with every 32nd step; the steps' attention scaled to all 1024
    sample = list(range(0, T, 32))
    t_proj = oracle_seconds(lambda: one_seq(0, [], False))
    t_some = oracle_seconds(lambda: one_seq(0, sample, False))
    t_seq = t_proj + (t_some - t_proj) * T / len(sample)
    return {"max_err": max(e[0] for e in errs), "err_over_tol": round(max(e[1] for e in errs), 4),
            "checked": f"steps {list(steps)} of sequences {list(seqs)}", "oracle_s": round(t_seq * 8, 2),
            "oracle_note": "one sequence's projection and every 32nd step timed, scaled to 8 sequences x 1024 steps"}


def check_fp8_error(q, k, v, o, ln, causal, nkv, signs, q8, k8, v8t, amax, stream, n=12):
    """FP8 output on sampled rows against exact attention on the bf16 inputs
    (float64 oracle), with the random-sign Hadamard rotation (the output in
    ``o``) and without it: the error the rotation removes."""
    import numpy as np

    import mqa_attention_qkv_b200 as gqa
    from oracle import gqa_ref as ref
    B, nh, S, hd = q.shape
    g = nh // nkv
    r = np.random.default_rng(17)
    sel = [(int(r.integers(B)), int(r.integers(nh)), int(r.integers(S))) for _ in range(n)]
    vis = [s + 1 if causal else S for _, _, s in sel]
    want = np.stack([ref.attend_row(_to64(q[b, h, s]), _to64(k[b, h // g, :L]), _to64(v[b, h // g, :L]))[0]
                     for (b, h, s), L in zip(sel, vis)])

    def rms_err(out):
        got = np.stack([_to64(out[b, s, h]) for b, h, s in sel])
        return float(np.sqrt(np.mean((got - want) ** 2)))

    e_rot = rms_err(o)
    o2 = o.clone()
    gqa.gqa_fp8_quantize_qkv(q, k, v, ln, q8, k8, v8t, amax, signs=None, stream=stream)
    gqa.gqa_attn_prefill_fp8(q8, k8, v8t, amax, ln, causal, o2, stream=stream)
    e_plain = rms_err(o2)
    gqa.gqa_fp8_quantize_qkv(q, k, v, ln, q8, k8, v8t, amax, signs=signs, stream=stream)   # rotated codes again
    return {"rms_err_vs_exact": round(e_rot, 5), "rms_err_vs_exact_no_rotation": round(e_plain, 5),
            "checked": f"{n} query rows against float64 attention on the bf16 inputs"}


def timed_once(fn, stream):
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b)


# ---------------------------------------------------------------------------
# the CPU oracle (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample_step(rows_per_seq: int, seed: int = 1):
    """The float64 oracle on one of the workload's sequences: projection of its
    2048 prompt tokens, causal attention for `rows_per_seq` evenly spaced query
    rows (all 32 heads) and their output projection + residual, then the
    decode step through the same layer.  Returns tokens covered."""
    import numpy as np

    import workloads as W
    from oracle import gqa_ref as ref
    wl = WORKLOAD
    S, nh, nkv, hd, cap = wl["S"], wl["n_heads"], wl["n_kv_heads"], wl["head_dim"], wl["cap"]
    shape = W.LayerShape(wl["hidden"], nh, nkv, hd, wl["theta"])
    x, w, pos = W.layer_inputs(shape, 1, S, seed=seed, dtype="bf16")
    xd = W.hidden_states(shape, 1, 1, seed=seed, stream=1, dtype="bf16")
    zeros = np.zeros((1, nkv, cap, hd))
    q, kc, vc = ref.qkv_rope_project(x.f64, w.f64, pos, nh, nkv, hd, wl["theta"], zeros, zeros)
    srows = np.linspace(0, S - 1, rows_per_seq).round().astype(int)
    rows = [(0, h, int(s)) for h in range(nh) for s in srows]
    w_o = W.output_weight(shape, seed, "bf16")
    o = np.asarray(ref.prefill_attention(q, kc, vc, np.array([S]), True, rows=rows))
    o = o.reshape(nh, rows_per_seq, hd).transpose(1, 0, 2)                  # [tokens, heads, hd]
    ref.output_projection(o, w_o.f64, x.f64[0, srows])
    qd, kc, vc = ref.qkv_rope_project(xd.f64, w.f64, np.array([[S]], dtype=np.int32), nh, nkv, hd,
                                      wl["theta"], kc, vc)
    od = ref.decode_attention(qd[:, :, 0], kc, vc, np.array([S + 1]))
    ref.output_projection(od[:, None], w_o.f64, xd.f64[:, 0:1])
    return rows_per_seq + 1


def _cores():
    try:
        from threadpoolctl import threadpool_info
        th = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        th = 1
    return th, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def cpu_baseline(budget_s: float = 20.0, rows_per_seq: int | None = None):
    if rows_per_seq is None:
        t0 = time.perf_counter()
        oracle_sample_step(64)
        dt = time.perf_counter() - t0
        rows_per_seq = int(max(64, min(WORKLOAD["S"], 64 * budget_s / max(dt, 1e-3))))
    t0 = time.perf_counter()
    tok = oracle_sample_step(rows_per_seq)
    dt = time.perf_counter() - t0
    threads, affinity = _cores()
    return {"value": round(tok / dt, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": (f"float64 numpy oracle, 1 of 4 sequences: projection of its 2048 prompt tokens, "
                       f"causal attention of {rows_per_seq} evenly spaced query rows x 32 heads and their "
                       f"output projection, 1 decode token; {dt:.1f} s; host affinity {affinity} cores"),
            "seconds": round(dt, 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    # size each step so that warm-up + timed steps stay within ~3 minutes
    per_step_budget = max(1.0, 180.0 / max(1, args.steps + args.warmup))
    t0 = time.perf_counter()
    oracle_sample_step(16)
    dt = time.perf_counter() - t0
    rows = int(max(16, min(WORKLOAD["S"], 16 * per_step_budget / max(dt, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample_step(rows)
    times, tok = [], 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        tok += oracle_sample_step(rows)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = tok / total
    threads, affinity = _cores()
    cpu = {"value": round(value, 2), "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": (f"float64 numpy oracle per step: 1 sequence, projection of 2048 prompt tokens, "
                      f"causal attention of {rows} evenly spaced query rows x 32 heads and their output "
                      f"projection, 1 decode token; host affinity {affinity} cores")}
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / max(1, args.steps), 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD["name"], "global_batch": WORKLOAD["B"], "seq_len": WORKLOAD["S"],
                   "parallelism": "host cores"},
        "cpu_baseline": cpu,
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-kernel measurements of the decode, 8K-prefill and generation workloads")
    ap.add_argument("--workloads", default=None,
                    help="comma-separated workload sections to measure (decode, decode_mqa, prefill8k, generate, small, "
                         "varlen, meanpool, tiny); default all")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps, always
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
