"""Benchmark: committed tokens/s of the block-autoregressive denoising path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload full|tiny] [--impl reference]

A step is one denoised block per sequence: canvas initialisation, denoising
steps to the adaptive stop (a random-weight model never reaches the entropy
stop, so every block runs the 48-step cap), the causal re-encode and the KV
block commit.  The prompt prefill is outside the timed region, as in the
metric; the cache length is reset to the prompt length before every step.

Reported (one JSON line from rank 0):
  value        committed tokens/s over all ranks (each rank an independent
               replica with its own seed: the path has no data-path exchange)
  e2e          the same metric through the public API with the prompt copied
               from pinned host memory and the block's tokens copied back every
               step (prefill inside the timed region)
  roofline     the dominant kernel's achieved throughput against the measured peak
  cpu_baseline the CPU oracle on a bounded sample of the same workload
With --impl reference the CPU oracle itself is timed on that workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "committed tokens/s (B=1, 256-tok canvas); canvas-attn % of BF16 tensor peak"


def dtype_name(args):
    """The arithmetic of the path: bf16, with e4m3 parts where asked."""
    parts = [p for p, on in (("projections", args.fp8_layers), ("unembed", args.fp8_unembed)) if on]
    return "bf16" if not parts else "bf16+e4m3-" + "+".join(parts)


def metric_name(batch):
    return METRIC.replace("B=1", f"B={batch}")
UNIT = "tokens/s"
CANVAS = 256
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_env():
    from canvas_denoising_denoise_b200 import replicas
    e = replicas.rank_env()
    return e.rank, e.world, e.local


def workload_config(name, world, steps_per_block=None):
    """The `config` object of both arms' JSON lines."""
    shape, batch, prompt = workload_spec(name)
    return {"workload": name, "weights": "random-init dense stand-in", "batch": batch,
            "prompt": prompt, "canvas": CANVAS, "d": shape.d, "layers": shape.n_layers,
            "heads": [shape.n_q_heads, shape.n_kv_heads], "head_dim": shape.head_dim,
            "ffn": shape.ffn, "vocab": shape.vocab, "steps_per_block": steps_per_block,
            "parallelism": f"replicas x{world}",
            "l2": ("inputs larger than L2 (3.3 GB of weights streamed per step)"
                   if shape.vocab * shape.d * 2 > L2_BYTES else "weights fit in L2")}


def workload_spec(name):
    from canvas_denoising_denoise_b200 import synth
    w = synth.WORKLOADS[name]
    return w["model"], w["batch"], w["prompt"]


def workload_blocks(name):
    from canvas_denoising_denoise_b200 import synth
    return synth.WORKLOADS[name]["blocks"]


class L2Flush:
    """Evicts L2 by reading a buffer twice its size (a read leaves no dirty
    lines, so the timed kernel does not pay for write-backs)."""

    def __init__(self):
        import torch
        self.buf = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
        self.out = torch.empty((), dtype=torch.float32, device="cuda")

    def __call__(self):
        import torch
        torch.sum(self.buf, dim=0, out=self.out)


def time_region(fn, steps, stream):
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1000.0


def captured_traffic(profile, sources, shape):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel sources changed since the capture (hash recorded in the summary) or
    the launch is not the shape that was captured (`captured_shape`)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(path):
        return None
    h = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, "canvas_denoising_denoise_b200", "csrc", src), "rb") as f:
            h.update(f.read())
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith(("#", "|", " ")):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    if fields.get("kernel_sources_sha256_16") != h.hexdigest()[:16]:
        return None
    if fields.get("captured_shape") != ",".join(str(int(v)) for v in shape):
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


_FLUSH = None


def graph_time(fn, reps=8, prep=None, do_flush=True):
    """Median device time of fn(), captured once into a CUDA graph (after one
    ordinary warm-up call) and replayed between CUDA events, the L2 flushed
    (read-only) before each replay unless do_flush is off.  Replaying keeps
    the host's launch preparation (argument marshalling, tensor-map encoding)
    out of the timed region: timed as plain launches, a kernel shorter than
    that preparation would be measured at the host's pace.  prep() runs on
    the same stream before each replay, untimed.  fn must launch on
    torch.cuda.current_stream()."""
    import torch
    global _FLUSH
    if _FLUSH is None:
        _FLUSH = L2Flush()
    cs = torch.cuda.Stream()
    with torch.cuda.stream(cs):
        if prep:
            prep()
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        fn()
    times = []
    with torch.cuda.stream(cs):
        for i in range(reps + 2):
            if prep:
                prep()
            if do_flush:
                _FLUSH()
            st = torch.cuda.Event(enable_timing=True)
            en = torch.cuda.Event(enable_timing=True)
            st.record(cs)
            g.replay()
            en.record(cs)
            torch.cuda.synchronize()
            if i >= 2:
                times.append(st.elapsed_time(en) / 1000.0)
    del g
    torch.cuda.synchronize()
    return statistics.median(times)


def chain_time(fns, reps=5):
    """Per-call device time of a chain of calls, captured into one CUDA graph
    (after one ordinary warm-up pass) and replayed between CUDA events.  The
    calls keep the programmatic-dependent-launch edges they get in the
    denoising step, so consecutive kernels overlap as they do there, and the
    host's launch preparation stays out of the timed region.  Each fn must
    launch on torch.cuda.current_stream()."""
    import torch
    cs = torch.cuda.Stream()
    with torch.cuda.stream(cs):
        for f in fns:
            f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        for f in fns:
            f()
    times = []
    with torch.cuda.stream(cs):
        for i in range(reps + 2):
            st = torch.cuda.Event(enable_timing=True)
            en = torch.cuda.Event(enable_timing=True)
            st.record(cs)
            g.replay()
            en.record(cs)
            torch.cuda.synchronize()
            if i >= 2:
                times.append(st.elapsed_time(en) / 1000.0)
    del g
    torch.cuda.synchronize()
    return statistics.median(times) / len(fns)


def gemm_roofline(dg, model, shape, batch, peaks, stream):
    """The dominant kernel: the layer projection GEMM (gemm_kernel), on its
    largest launch of a denoising step, the MLP down projection
    (M = B*256 tokens, N = d, K = F; at B = 1 gemm_kernel<4,128>, 128 CTAs).

    Timed as in the step: the launches of all layers' MLP down weights back to
    back (805 MB of weights at the full model, far above L2, so each streams
    from HBM) on a hot activation, chained by programmatic dependent launch,
    as one CUDA-graph replay between CUDA events; the time per launch is the
    chain's over the layer count.  `alone_us` is one launch after an L2
    flush, cold and without neighbours.  FLOP-based against the burst bf16
    peak (at 256 tokens the launch sits at the ridge: 256 FLOP per weight byte).
    """
    import torch
    M, N, K = batch * CANVAS, shape.d, shape.ffn
    x = torch.randn((M, K), device="cuda").to(torch.bfloat16)
    out = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    ws = dg.Workspace()
    fns = [(lambda w=lw["w_down"]: dg.linear(x, w, out, dg.EPI_RESID_F32, ws=ws))
           for lw in model.w["layers"]]
    t = chain_time(fns)
    t_alone = graph_time(fns[-1])
    flops = 2.0 * M * N * K
    achieved = flops / t / 1e12
    peak = peaks["bf16_tflops"]
    return {"kernel": "gemm_kernel (MLP down projection launch)", "shape": [M, N, K],
            "bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": captured_traffic("gemm_mlp_down_full.md", ["gemm.cuh", "dg_common.cuh"],
                                        (M, N, K)),
            "algorithmic_bytes": int(N * K * 2 + M * K * 2 + M * N * 4 * 2),
            "hbm_frac": round((N * K * 2 + M * K * 2 + M * N * 8) / t / 1e9 / peaks["hbm_gbs"], 4),
            "peak_source": f"{peaks['source']} burst bf16",
            "launch_us": round(t * 1e6, 2), "alone_us": round(t_alone * 1e6, 2),
            "timing": f"{len(fns)} launches chained as in the step", "flops_per_launch": flops}


def sampler_step_roofline(dg, model, shape, batch, peaks, stream):
    """The unembedding fused with one sampler step (fused kernel + merge +
    commit): 2*M*V*d FLOP; the vocabulary matrix (V*d*2 bytes) is read once."""
    import torch
    M, d, V = batch * CANVAS, shape.d, shape.vocab
    h = torch.randn((M, d), device="cuda").to(torch.bfloat16)
    tok = torch.zeros((batch, CANVAS), dtype=torch.int32, device="cuda")
    com = torch.zeros((batch, CANVAS), dtype=torch.uint8, device="cuda")
    prev = torch.full((batch, CANVAS), -1, dtype=torch.int32, device="cuda")
    stat = torch.zeros(batch, dtype=torch.int32, device="cuda")
    ws = dg.Workspace()
    settings = dg.SamplerSettings()

    if model.unembed_q is not None:
        # e4m3 operands: the per-token quantisation of h is part of the step
        hq = torch.empty((M, d), dtype=torch.uint8, device="cuda")
        hs = torch.empty(M, dtype=torch.float32, device="cuda")

        def step():
            stat.zero_()
            dg.quantize_e4m3(h, hq, hs, per_row=True)
            dg.unembed_sample_commit_e4m3(hq, hs, model.unembed_q, model.unembed_scale, tok, com,
                                          prev, stat, settings, 0, 0, 5, ws=ws)
        # the recipe's nominal fp8 : bf16 dense ratio (4.5 : 2.25) times the measured bf16 peak
        peak, wbytes, kname = 2.0 * peaks["bf16_tflops"], V * d, "quantize + e4m3 fused step"
    else:
        def step():
            stat.zero_()
            dg.unembed_sample_commit(h, model.w["unembed"], tok, com, prev, stat, settings, 0,
                                     0, 5, ws=ws)
        peak, wbytes, kname = peaks["bf16_tflops"], V * d * 2, \
            "unembed_sample_kernel + merge + commit"
    t = graph_time(step)
    flops = 2.0 * M * V * d
    return {"kernel": kname, "shape": [M, V, d],
            "achieved": round(flops / t / 1e12, 1), "peak": round(peak, 1),
            "unit": "TFLOP/s", "frac": round(flops / t / 1e12 / peak, 4),
            "hbm_frac": round(wbytes / t / 1e9 / peaks["hbm_gbs"], 4),
            "us": round(t * 1e6, 1)}


def attn_roofline(dg, shape, batch, prefix, peaks, stream, st=None):
    """Achieved TFLOP/s of canvas attention (kernel + split merge) at the
    workload's prefix length.  With the workload's state `st`, timed as in the
    step: one call per layer over that layer's prefilled cache (each streams
    from HBM), back to back as one CUDA-graph replay; `alone_us` is one call
    after an L2 flush."""
    import torch
    from canvas_denoising_denoise_b200 import synth
    hq, hkv, hd = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    q, kn, vn, kc, vc = synth.make_attn_inputs(batch, hq, hkv, hd, CANVAS, prefix, seed=0,
                                               device="cuda")
    cl = torch.full((batch,), prefix, dtype=torch.int32, device="cuda")
    out = torch.empty((batch, CANVAS, hq * hd), dtype=torch.bfloat16, device="cuda")
    t_alone = graph_time(lambda: dg.canvas_attn(q, kn, vn, kc, vc, cl, prefix, out,
                                                n_q_heads=hq, n_kv_heads=hkv, head_dim=hd))
    t = t_alone
    if st is not None:
        fns = [(lambda k=k, v=v: dg.canvas_attn(q, kn, vn, k, v, cl, prefix, out, n_q_heads=hq,
                                                n_kv_heads=hkv, head_dim=hd))
               for k, v in zip(st.k_cache, st.v_cache)]
        t = chain_time(fns)
    flops = 4.0 * batch * hq * CANVAS * (prefix + CANVAS) * hd
    achieved = flops / t / 1e12
    return {"achieved": round(achieved, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(achieved / peaks["bf16_tflops"], 4), "us": round(t * 1e6, 1),
            "alone_us": round(t_alone * 1e6, 1), "prefix": prefix}


def kv_commit_roofline(dg, shape, batch, st, prefix, peaks, stream):
    """The block K/V commit of every layer (one launch): 2 x its bytes (read +
    write) over the CUDA-event time, against the measured HBM rate."""
    import torch
    nl, hq, hkv, hd = shape.n_layers, shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    nqkv = (hq + 2 * hkv) * hd
    # each layer its own QKV output, as in the re-encode (no source re-read from L2)
    qkv = [torch.randn((batch, CANVAS, nqkv), device="cuda").to(torch.bfloat16)
           for _ in range(nl)]
    k_blk = [t[:, :, hq * hd:(hq + hkv) * hd] for t in qkv]
    v_blk = [t[:, :, (hq + hkv) * hd:] for t in qkv]
    t = graph_time(lambda: dg.kv_block_commit(k_blk, v_blk, st.k_cache, st.v_cache,
                                              st.cache_len, n_kv_heads=hkv, head_dim=hd),
                   prep=lambda: st.cache_len.fill_(prefix))
    moved = 2.0 * (2 * nl * batch * hkv * CANVAS * hd * 2)
    return {"kernel": "kv_commit_kernel", "achieved": round(moved / t / 1e9, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(moved / t / 1e9 / peaks["hbm_gbs"], 4),
            "bytes": int(moved), "us": round(t * 1e6, 1)}


def step_upper_bound(shape, batch, prefix, steps, peaks):
    """tokens/s <= B*256 / ((steps + 1) * max(F_step / P_bf16, Bytes_step / BW_hbm)) for
    one block at the workload's prefix (the fused path moves no logits)."""
    d, nl, hq, hkv, hd, ffn, V = (shape.d, shape.n_layers, shape.n_q_heads, shape.n_kv_heads,
                                  shape.head_dim, shape.ffn, shape.vocab)
    M = batch * CANVAS
    params = nl * ((hq + 2 * hkv) * hd * d + d * hq * hd + 2 * ffn * d)
    flops = 2.0 * M * params + 4.0 * batch * hq * CANVAS * (prefix + CANVAS) * hd * nl \
        + 2.0 * M * V * d
    nbytes = 2.0 * (params + V * d) + 2 * nl * batch * hkv * prefix * hd * 2.0
    t = max(flops / (peaks["bf16_tflops"] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))
    return {"value": round(M / ((steps + 1) * t), 1), "unit": UNIT,
            "per_step_tflop": round(flops / 1e12, 3), "per_step_gb": round(nbytes / 1e9, 3),
            "bound": "tensor" if flops / (peaks["bf16_tflops"] * 1e12) > nbytes / (peaks["hbm_gbs"] * 1e9)
            else "hbm"}


def cpu_baseline_sample(w_cpu, shape, prefix, budget_s=30.0, w64=None):
    """The CPU oracle on one denoising step of the workload (bounded sample).

    The sample is one bidirectional forward of a 256-token canvas over a
    `prefix`-row cache plus one sampler step; the cache rows are seeded noise
    (the oracle's own prefill of a 4096-token prompt would take far longer and
    is outside the metric anyway).  Tokens/s is extrapolated to a 48-step
    block with one re-encode pass.
    """
    import numpy as np
    import torch
    from oracle import model as M
    from oracle import sampler as S
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    ocfg = M.ModelCfg(shape.d, shape.n_layers, shape.n_q_heads, shape.n_kv_heads,
                      shape.head_dim, shape.ffn, shape.vocab, shape.eps)
    if w64 is None:
        w64 = M.weights_to_f64(w_cpu)
    g = torch.Generator().manual_seed(5)
    kc = [torch.randn((shape.n_kv_heads, prefix, shape.head_dim), generator=g).double().numpy()
          for _ in range(shape.n_layers)]
    vc = [torch.randn((shape.n_kv_heads, prefix, shape.head_dim), generator=g).double().numpy()
          for _ in range(shape.n_layers)]
    tok = S.init_canvas(0, 0, 0, CANVAS, shape.vocab)
    t0 = time.perf_counter()
    logits = M.denoise_logits(ocfg, w64, tok, kc, vc, prefix)
    t_fwd = time.perf_counter() - t0
    t1 = time.perf_counter()
    S.sampler_step(S.SamplerCfg(), logits.astype(np.float32), tok, np.zeros(CANVAS, bool), None,
                   0, 0, 0, 0)
    t_smp = time.perf_counter() - t1
    block_s = 48 * (t_fwd + t_smp) + t_fwd
    return {"value": round(CANVAS / block_s, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"1 of 48 denoising steps (forward {t_fwd:.1f} s + sampler {t_smp:.1f} s) "
                       f"at prefix {prefix}, extrapolated to a 48-step block + re-encode; "
                       f"prefill excluded as in the metric")}


def run_reference(args):
    """--impl reference: the CPU oracle timed on the same workload (rank 0 only)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import torch
    from canvas_denoising_denoise_b200 import synth
    shape, batch, prompt = workload_spec(args.workload)
    if args.workload == "tiny":
        w_cpu = synth.make_weights(shape, seed=0)
    else:
        w_cpu = synth.make_weights_fast(shape, seed=0, device="cuda" if torch.cuda.is_available()
                                        else "cpu")
        w_cpu = {"embed": w_cpu["embed"].cpu(), "unembed": w_cpu["unembed"].cpu(),
                 "layers": [{k: v.cpu() for k, v in lw.items()} for lw in w_cpu["layers"]]}
    from oracle import model as M
    w64 = M.weights_to_f64(w_cpu)  # once: 4x the bf16 bytes
    vals = []
    for _ in range(max(1, args.steps)):
        vals.append(cpu_baseline_sample(w_cpu, shape, prompt, w64=w64))
    v = statistics.median([x["value"] for x in vals])
    line = {"impl": "reference", "metric": metric_name(batch), "value": v, "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(CANVAS / v * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(args.workload, world, 48),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": vals[0]["cores"],
                             "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_kernel_bench(args):
    """Single-kernel measurements (CUDA events, warm, L2 flushed between launches).

    --kernel attn     the attention microbench: B=1, Q [32, 256, 128], prefix
                      K/V [8, L, 128] for L = --prefix (default all of
                      1024, 4096, 16384, 32768), full mask.
    --kernel sampler  the sampler sweep: logits [B, 256, 262144] fp32 for
                      B = --batch, 48 scheduled steps, logits regenerated per
                      step outside the timed region.
    --kernel gemm     one projection y = x w^T for --shape M,N,K (bf16 out).
    --kernel unembed  the unembedding alone, logits to memory.
    --kernel fused    the unembedding fused with a sampler step, and unfused.
    --kernel kvcommit the block K/V commit of the full model (24 layers) at
                      prefix --prefix (default 4096), B = --batch.
    """
    import torch
    import canvas_denoising_denoise_b200 as dg
    from canvas_denoising_denoise_b200 import synth
    peaks = load_peaks()
    def timed(fn, reps, do_flush=True, prep=None):
        return graph_time(fn, reps=reps, prep=prep, do_flush=do_flush)

    out = []
    if args.kernel == "attn":
        prefixes = [args.prefix] if args.prefix else [1024, 4096, 16384, 32768]
        B, hd = 1, 128
        hq, hkv = (int(v) for v in args.heads.split(","))
        for L in prefixes:
            q, kn, vn, kc, vc = synth.make_attn_inputs(B, hq, hkv, hd, CANVAS, L, seed=0,
                                                       device="cuda")
            cl = torch.full((B,), L, dtype=torch.int32, device="cuda")
            o = torch.empty((B, CANVAS, hq * hd), dtype=torch.bfloat16, device="cuda")
            ws = dg.Workspace()
            t = timed(lambda: dg.canvas_attn(q, kn, vn, kc, vc, cl, L, o, n_q_heads=hq,
                                             n_kv_heads=hkv, head_dim=hd, ws=ws), args.steps)
            fl = 4.0 * B * hq * CANVAS * (L + CANVAS) * hd
            out.append({"kernel": "canvas_attn", "heads": [hq, hkv], "prefix": L,
                        "us": round(t * 1e6, 2),
                        "tflops": round(fl / t / 1e12, 1),
                        "frac_bf16_peak": round(fl / t / 1e12 / peaks["bf16_tflops"], 4)})
            if args.fp8_attn:
                # e4m3 codes made on the device (outside the timed region): per-token
                # Q, one scale over the cached and new K (and V), V transposed
                q8 = torch.empty((B * CANVAS, hq * hd), dtype=torch.uint8, device="cuda")
                qs = torch.empty(B * CANVAS, dtype=torch.float32, device="cuda")
                dg.quantize_e4m3(q.view(B * CANVAS, -1), q8, qs, per_row=True)
                codes = {}
                for name, cache, new in (("k", kc, kn), ("v", vc, vn)):
                    both = torch.cat([cache.reshape(-1, hd), new.reshape(-1, hd)])
                    c8 = torch.empty(both.shape, dtype=torch.uint8, device="cuda")
                    sc = torch.empty(1, dtype=torch.float32, device="cuda")
                    dg.quantize_e4m3(both, c8, sc, per_row=False)
                    nc = cache.numel() // hd
                    codes[name] = (c8[:nc].view(cache.shape), c8[nc:].view(new.shape), sc)
                kc8, kn8, ks = codes["k"]
                vc8, vn8, vs = codes["v"]
                vt_c = vc8.transpose(-1, -2).contiguous()
                vt_n = vn8.view(B, CANVAS, hkv, hd).permute(0, 2, 3, 1).contiguous()
                kn8 = kn8.contiguous()
                t8 = timed(lambda: dg.canvas_attn_e4m3(q8.view(B, CANVAS, -1), qs, kn8, vt_n,
                                                       kc8, vt_c, ks, vs, cl, L, o,
                                                       n_q_heads=hq, n_kv_heads=hkv, ws=ws),
                           args.steps)
                # e4m3 tensor peak: the measured bf16 peak times the nominal ratio 2
                out.append({"kernel": "canvas_attn_e4m3", "heads": [hq, hkv], "prefix": L,
                            "us": round(t8 * 1e6, 2), "tflops": round(fl / t8 / 1e12, 1),
                            "frac_fp8_peak": round(fl / t8 / 1e12 / (2 * peaks["bf16_tflops"]), 4),
                            "frac_bf16_peak": round(fl / t8 / 1e12 / peaks["bf16_tflops"], 4),
                            "speedup_vs_bf16": round(t / t8, 3)})
                del q8, codes, kc8, kn8, vc8, vn8, vt_c, vt_n
    elif args.kernel == "sampler":
        B, V = args.batch, 262144
        settings = dg.SamplerSettings()
        tok = torch.zeros((B, CANVAS), dtype=torch.int32, device="cuda")
        com = torch.zeros((B, CANVAS), dtype=torch.uint8, device="cuda")
        prev = torch.full((B, CANVAS), -1, dtype=torch.int32, device="cuda")
        stat = torch.zeros(B, dtype=torch.int32, device="cuda")
        ws = dg.Workspace()
        ts = []
        for s_ in range(48):
            logits = synth.make_sampler_logits(B, CANVAS, V, seed=0, step=s_, device="cuda")
            # the sweep runs all 48 scheduled steps: no sequence is left stopped
            ts.append(timed(lambda: dg.sample_commit(logits, tok, com, prev, stat, settings, 0,
                                                     0, s_, ws=ws), 1, do_flush=False,
                            prep=stat.zero_))
            del logits
        t = statistics.median(ts)
        byts = B * CANVAS * V * 4
        out.append({"kernel": "sample_commit", "batch": B, "us_per_step": round(t * 1e6, 2),
                    "gbs": round(byts / t / 1e9, 1),
                    "frac_hbm_peak": round(byts / t / 1e9 / peaks["hbm_gbs"], 4),
                    "committed_tokens_per_s": round(16 * B / t, 1)})
    elif args.kernel == "kvcommit":
        # the block K/V commit of the full model (24 layers) at the given prefix
        shape = synth.FULL
        prefix = args.prefix or 4096
        st = dg.DgState(shape, args.batch, prefix + CANVAS, CANVAS)
        out.append(kv_commit_roofline(dg, shape, args.batch, st, prefix, peaks,
                                      torch.cuda.current_stream()))
    elif args.kernel == "unembed":
        # the unembedding launch of the full workload: logits [256, 262144] fp32
        M, d, V = 256 * args.batch, 2048, 262144
        h = torch.randn((M, d), device="cuda").to(torch.bfloat16)
        w = (torch.randn((V, d), device="cuda") * 0.02).to(torch.bfloat16)
        lg = torch.empty((M, V), dtype=torch.float32, device="cuda")
        t = timed(lambda: dg.unembed(h, w, lg), args.steps)
        fl = 2.0 * M * V * d
        byts = V * d * 2 + M * V * 4 + M * d * 2
        out.append({"kernel": "unembed", "shape": [M, V, d], "us": round(t * 1e6, 2),
                    "tflops": round(fl / t / 1e12, 1),
                    "frac_bf16_peak": round(fl / t / 1e12 / peaks["bf16_tflops"], 4),
                    "gbs": round(byts / t / 1e9, 1),
                    "frac_hbm_peak": round(byts / t / 1e9 / peaks["hbm_gbs"], 4)})
    elif args.kernel == "fused":
        # the unembedding fused with one sampler step (fused kernel + merge +
        # commit) against the unfused pair (unembedding, then sample_commit)
        B, d, V = args.batch, 2048, 262144
        M = B * CANVAS
        h = torch.randn((M, d), device="cuda").to(torch.bfloat16)
        w = (torch.randn((V, d), device="cuda") * 0.02).to(torch.bfloat16)
        settings = dg.SamplerSettings()
        tok = torch.zeros((B, CANVAS), dtype=torch.int32, device="cuda")
        com = torch.zeros((B, CANVAS), dtype=torch.uint8, device="cuda")
        prev = torch.full((B, CANVAS), -1, dtype=torch.int32, device="cuda")
        stat = torch.zeros(B, dtype=torch.int32, device="cuda")
        lg = torch.empty((B, CANVAS, V), dtype=torch.float32, device="cuda")
        ws = dg.Workspace()

        def fused():
            stat.zero_()
            dg.unembed_sample_commit(h, w, tok, com, prev, stat, settings, 0, 0, 5, ws=ws)

        def unfused():
            stat.zero_()
            dg.unembed(h, w, lg.view(M, V))
            dg.sample_commit(lg, tok, com, prev, stat, settings, 0, 0, 5, ws=ws)

        hq = torch.empty((M, d), dtype=torch.uint8, device="cuda")
        hs = torch.empty(M, dtype=torch.float32, device="cuda")
        wq = torch.empty((V, d), dtype=torch.uint8, device="cuda")
        wsc = torch.empty(1, dtype=torch.float32, device="cuda")
        dg.quantize_e4m3(w, wq, wsc, per_row=False)

        def quant():
            dg.quantize_e4m3(h, hq, hs, per_row=True)

        def fused_e4m3():
            stat.zero_()
            dg.unembed_sample_commit_e4m3(hq, hs, wq, wsc, tok, com, prev, stat, settings, 0, 0,
                                          5, ws=ws)

        fl = 2.0 * M * V * d
        for name, fn, wbytes, peak in (
                ("unembed_sample_commit (fused)", fused, V * d * 2, peaks["bf16_tflops"]),
                ("unembed + sample_commit", unfused, V * d * 2, peaks["bf16_tflops"]),
                ("unembed_sample_commit_e4m3 (fused)", fused_e4m3, V * d,
                 2.0 * peaks["bf16_tflops"]),
                ("quantize_e4m3 per token", quant, M * d * 3, None)):
            t = timed(fn, args.steps)
            row = {"kernel": name, "shape": [M, V, d], "us": round(t * 1e6, 2),
                   "weight_gbs": round(wbytes / t / 1e9, 1),
                   "frac_hbm_peak": round(wbytes / t / 1e9 / peaks["hbm_gbs"], 4)}
            if peak:
                row.update(tflops=round(fl / t / 1e12, 1),
                           frac_tensor_peak=round(fl / t / 1e12 / peak, 4))
            out.append(row)
    elif args.kernel == "gemm":
        M, N, K = (int(x) for x in args.shape.split(","))
        x = torch.randn((M, K), device="cuda").to(torch.bfloat16)
        w = (torch.randn((N, K), device="cuda") * K ** -0.5).to(torch.bfloat16)
        epi = {"bf16": dg.EPI_BF16, "gelu": dg.EPI_GELU_BF16, "f32": dg.EPI_F32,
               "resid": dg.EPI_RESID_F32}[args.epi]
        y = (torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
             if args.epi in ("bf16", "gelu") else torch.zeros((M, N), dtype=torch.float32,
                                                                device="cuda"))
        ws = dg.Workspace()
        t = timed(lambda: dg.linear(x, w, y, epi, ws=ws), args.steps)
        fl = 2.0 * M * N * K
        out.append({"kernel": "linear", "epilogue": args.epi, "shape": [M, N, K],
                    "us": round(t * 1e6, 2),
                    "tflops": round(fl / t / 1e12, 1),
                    "weight_gbs": round(N * K * 2 / t / 1e9, 1)})
        if K % 128 == 0:
            # the same projection on e4m3 codes (the activation quantised per
            # token first, as the forward pass does), and the GEMM alone
            xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
            xs = torch.empty(M, dtype=torch.float32, device="cuda")
            wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
            wsc = torch.empty(1, dtype=torch.float32, device="cuda")
            dg.quantize_e4m3(w, wq, wsc, per_row=False)

            def q_and_gemm():
                dg.quantize_e4m3(x, xq, xs, per_row=True)
                dg.linear_e4m3(xq, xs, wq, wsc, y, epi)
            for name, fn in (("quantize_e4m3 + linear_e4m3", q_and_gemm),
                             ("linear_e4m3", lambda: dg.linear_e4m3(xq, xs, wq, wsc, y, epi))):
                t = timed(fn, args.steps)
                out.append({"kernel": name, "epilogue": args.epi, "shape": [M, N, K],
                            "us": round(t * 1e6, 2), "tflops": round(fl / t / 1e12, 1),
                            "frac_fp8_peak": round(fl / t / 1e12 / (2 * peaks["bf16_tflops"]), 4),
                            "weight_gbs": round(N * K / t / 1e9, 1)})
    for o in out:
        o["peaks"] = peaks["source"]
        print(json.dumps(o), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="full", choices=["full", "tiny", "long_b1", "long_b8"],
                    help="full: one canvas after a 4096-token prompt (the headline); long_b*: "
                         "8 canvases after a 2048-token prompt at B = 1 / 8")
    ap.add_argument("--impl", default="dg", choices=["dg", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["attn", "sampler", "gemm", "unembed", "fused",
                                         "kvcommit"],
                    default=None,
                    help="time one kernel alone instead of the denoising step")
    ap.add_argument("--prefix", type=int, default=0)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--shape", default="256,8192,2048")
    ap.add_argument("--epi", default="bf16", choices=["bf16", "gelu", "f32", "resid"],
                    help="epilogue for --kernel gemm")
    ap.add_argument("--heads", default="32,8", help="query,kv heads for --kernel attn")
    ap.add_argument("--fp8-attn", action="store_true",
                    help="--kernel attn: also time the e4m3 attention on the same inputs")
    ap.add_argument("--fp8-unembed", action="store_true",
                    help="run the unembedding + sampler step on e4m3 operands")
    ap.add_argument("--fp8-layers", action="store_true",
                    help="run every projection of the stack on e4m3 operands")
    args = ap.parse_args()
    if args.kernel:
        return run_kernel_bench(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch

    import canvas_denoising_denoise_b200 as dg
    from canvas_denoising_denoise_b200 import replicas, synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        replicas.init("nccl", timeout_s=120)
    seeds = replicas.replica_seeds(rank)
    lib = dg._lib.load()
    shape, batch, prompt_len = workload_spec(args.workload)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()

    # ---------------------------------------------------------------- set-up
    if args.workload == "tiny":
        w_cpu = synth.make_weights(shape, seed=0)
        weights = {"embed": w_cpu["embed"].cuda(), "unembed": w_cpu["unembed"].cuda(),
                   "layers": [{k: v.cuda() for k, v in lw.items()} for lw in w_cpu["layers"]]}
    else:
        weights = synth.make_weights_fast(shape, seed=0, device="cuda")
    model = dg.DgModel(shape, weights, fp8_unembed=args.fp8_unembed, fp8_layers=args.fp8_layers)
    blocks = workload_blocks(args.workload)
    lmax = prompt_len + CANVAS * blocks
    st = dg.DgState(shape, batch, lmax, CANVAS)
    prompt = synth.make_prompt(batch, prompt_len, shape.vocab, seed=seeds.prompt).cuda()
    ws = dg.Workspace()
    ws.get(max(dg.denoise_workspace_bytes(model, st),
               lib.dg_prefill_workspace_bytes(ctypes_ref(model.cfg), batch, prompt_len)))
    dg.prefill(model, st, prompt, ws=ws)
    torch.cuda.synchronize()
    dg.check_device_errors()
    settings = dg.SamplerSettings()
    seed = seeds.sampler
    steps_seen = []

    def block_step():
        # the generation of `blocks` canvases after the prompt
        st.cache_len.fill_(prompt_len)
        st.cache_len_host = prompt_len
        for blk in range(blocks):
            steps_seen.append(dg.denoise_block(model, st, settings, seed, blk, ws=ws))

    for _ in range(args.warmup):
        block_step()
    torch.cuda.synchronize()
    dg.check_device_errors()

    # ---------------------------------------------------------------- timed
    clocks = ClockSampler(torch.cuda.current_device())
    replicas.barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    n0 = lib.dg_launch_count()
    steps_seen.clear()
    elapsed = time_region(block_step, args.steps, stream)
    launches = lib.dg_launch_count() - n0
    clk = clocks.stop()
    elapsed = replicas.max_over_ranks(elapsed, world)
    replicas.barrier(world)
    dg.check_device_errors()
    value = replicas.whole_job_rate(batch * CANVAS * blocks * args.steps, world, elapsed)

    # ---------------------------------------------------------------- end to end
    host_prompt = synth.make_prompt(batch, prompt_len, shape.vocab, seed=seeds.prompt).pin_memory()
    host_out = torch.empty((batch, CANVAS), dtype=torch.int32).pin_memory()
    dev_prompt = torch.empty_like(prompt)

    def e2e_step():
        dev_prompt.copy_(host_prompt, non_blocking=True)
        dg.prefill(model, st, dev_prompt, ws=ws)
        for blk in range(blocks):
            dg.denoise_block(model, st, settings, seed, blk, ws=ws)
            host_out.copy_(st.tok, non_blocking=True)

    e2e_step()
    replicas.barrier(world)
    e2e_t = time_region(e2e_step, max(1, args.steps // 2), stream)
    e2e_t = replicas.max_over_ranks(e2e_t, world)
    e2e_val = replicas.whole_job_rate(batch * CANVAS * blocks * max(1, args.steps // 2), world,
                                      e2e_t)

    # ---------------------------------------------------------------- roofline
    roof = gemm_roofline(dg, model, shape, batch, peaks, stream)
    attn = attn_roofline(dg, shape, batch, prompt_len, peaks, stream, st)
    samp = (sampler_step_roofline(dg, model, shape, batch, peaks, stream)
            if shape.vocab % 256 == 0 else None)
    kvc = kv_commit_roofline(dg, shape, batch, st, prompt_len, peaks, stream)
    ub = step_upper_bound(shape, batch, prompt_len, steps_seen[-1] if steps_seen else 48, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        w_cpu = {"embed": weights["embed"].cpu(), "unembed": weights["unembed"].cpu(),
                 "layers": [{k: v.cpu() for k, v in lw.items()} for lw in weights["layers"]]}
        cpu = cpu_baseline_sample(w_cpu, shape, prompt_len)
        del w_cpu

    if rank == 0:
        line = {
            "metric": metric_name(batch), "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_name(args), "data": "synthetic",
            "config": dict(workload_config(args.workload, world,
                                           steps_seen[-1] if steps_seen else None),
                           unembed="e4m3" if args.fp8_unembed else "bf16",
                           projections="e4m3" if args.fp8_layers else "bf16"),
            "roofline": roof,
            "canvas_attn": attn,
            "unembed_sample": samp,
            "kv_commit": kvc,
            "upper_bound": ub,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_val, 2), "unit": UNIT,
                    "h2d_bytes_per_step": int(host_prompt.numel() * 4),
                    "d2h_bytes_per_step": int(host_out.numel() * 4 * blocks),
                    "includes": "prompt H2D + prefill + denoised block + tokens D2H"},
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    replicas.finish(world)
    return 0


def ctypes_ref(x):
    import ctypes
    return ctypes.byref(x)


if __name__ == "__main__":
    sys.exit(main())
