"""Benchmark of the QLoRA-linear hot path on B200.

One step = one pass of the whole path over one batch of the layer:
  nf4_quantize_dq (fp32 W0 -> NF4 codes + absmax, then the double
  quantization of the constants, in one call) ->
  nf4_dequant (materialised BF16 W', the standalone decode) ->
  qlora_linear_fwd (U = X A^T, fused NF4 GEMM + adapter) ->
  qlora_linear_bwd (G = dY B, fused dX GEMM, dA, dB).
The default workload is the prefill-shaped MLP up-projection
(W0 11008 x 4096, 2048 tokens, r = 16, s = 2), the fwd+bwd configuration of
the headline metric.  value = algorithmic fwd+bwd FLOPs of all ranks / the
slowest rank's device time for K steps (CUDA events), in TFLOP/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload prefill|large|pr1]

Under torchrun (N > 1) every rank runs its own replica with its own tokens
(weak scaling) and the data-parallel exchange, an all-reduce of dA and dB, is
part of each step.  ``--impl reference`` times the CPU oracle on the host
cores (rank 0 only) on a bounded sample of the same workload.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 (de)quant GB/s, % of B200 roofline"


def _load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# Sources of the kernels a prefill-shaped qlora_linear_fwd launches (adapter
# product + fold, fused tcgen05 GEMM) and of the dispatch that picks them.
FWD_PATH_SOURCES = ("api.cu", "lora_small.cu", "nf4_gemm_sm100.cu", "qln_common.cuh", "qln_internal.h",
                    "tc_ptx.cuh")


def _kernel_sources_sha1():
    """SHA-1 over the CUDA sources of the forward path: identifies the kernels
    a committed ncu traffic record was taken from."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "bit_nf4_quantized_07_b200", "csrc")
    for fn in FWD_PATH_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()


def _recorded_traffic(workload):
    """DRAM bytes per qlora_linear_fwd call from profiles/roofline_traffic.json,
    or None when the record is missing, for another workload, or taken from
    kernel sources other than the current ones."""
    p = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("workload") != workload or rec.get("kernel_sources_sha1") != _kernel_sources_sha1():
        return None
    return rec.get("dram_bytes_per_call")


def _workload(name):
    from bit_nf4_quantized_07_b200 import synthetic
    return {"prefill": synthetic.PREFILL, "large": synthetic.LARGE, "pr1": synthetic.PR1}[name]


def l2_note(cfg, nsets):
    """How the timed step relates to the 126 MB L2: the fp32 weight of one
    input set and whether the rotating sets defeat the cache."""
    w_mb = cfg.dout * cfg.din * 4 / 1e6
    if w_mb > 126:
        return f"{nsets} rotating input sets (W0 fp32 alone {w_mb:.0f} MB > 126 MB L2)"
    return f"{nsets} rotating input sets; W0 fp32 {w_mb:.1f} MB fits in the 126 MB L2 (launch-bound layer, not L2-defeated)"


def codec_bytes_per_param():
    """Algorithmic bytes per parameter: quantize + DQ reads fp32 W0 and writes
    codes, rhat and the group scales; dequant reads those and writes BF16."""
    q = 4.0 + 0.5 + 1.0 / 64 + 4.0 / (64 * 256)
    d = 0.5 + 1.0 / 64 + 4.0 / (64 * 256) + 2.0
    return q, d


def decode_bytes_per_call(rows, cols, n, r):
    """Algorithmic bytes of one decode-sized forward with a double-quantized
    weight: codes, rhat, group scales and mu, then X, A, B, U and Y (bf16)."""
    nb = rows * cols // 64
    wbytes = rows * cols // 2 + nb + 4 * ((nb + 255) // 256) + 4
    return wbytes + 2 * n * cols + 2 * r * cols + 2 * rows * r + 2 * n * r + 2 * n * rows


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.12)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle leg (reported baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(cfg, budget_s=15.0):
    """Time the oracle, as it stands, on a bounded sample of one step and
    extrapolate to the full step.  The sample (a row slice of W0 for the codec,
    a token slice for the fp64 linear algebra) is sized so that it takes about
    ``budget_s`` seconds.  Returns (step_seconds_estimate, info)."""
    from bit_nf4_quantized_07_b200 import synthetic
    from oracle import codec, linear
    try:
        from threadpoolctl import threadpool_info
        blas_threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        blas_threads = os.cpu_count() or 1
    # probe: 1/64 of the rows, 16 tokens; then size the real sample
    row_frac = max(64, cfg.dout // 64)
    w = synthetic.normal_f32((row_frac, cfg.din), cfg.w_sigma, 77)
    t0 = time.perf_counter()
    codec.quantize(w)
    t_probe = max(1e-4, time.perf_counter() - t0)
    row_frac = int(min(cfg.dout, max(64, row_frac * (0.3 * budget_s) / t_probe)))
    w = synthetic.normal_f32((row_frac, cfg.din), cfg.w_sigma, 77)
    t0 = time.perf_counter()
    codes, absmax = codec.quantize(w)
    qabs, scale, mu = codec.double_quant(absmax)
    wp_bits = codec.dequant(codes, w.size, qabs=qabs, scale=scale, mu=mu)
    t_codec = time.perf_counter() - t0
    codec_full = t_codec * cfg.dout / row_frac
    # fp64 forward + backward for a token slice against the full-size weight
    ntok = max(1, min(cfg.n, 16))
    g = np.random.Generator(np.random.PCG64(78))
    Wp = np.repeat(codec.bf16_bits_to_f64(wp_bits).reshape(row_frac, cfg.din), cfg.dout // row_frac + 1,
                   axis=0)[:cfg.dout]
    X = g.standard_normal((ntok, cfg.din))
    A = g.standard_normal((cfg.r, cfg.din)) * cfg.ab_sigma
    B = g.standard_normal((cfg.dout, cfg.r)) * cfg.ab_sigma
    dY = g.standard_normal((ntok, cfg.dout))
    t0 = time.perf_counter()
    linear.forward(Wp, X, A, B, cfg.s)
    linear.backward(Wp, X, A, B, cfg.s, dY)
    t_probe = max(1e-4, time.perf_counter() - t0)
    ntok = int(min(cfg.n, max(ntok, ntok * (0.7 * budget_s) / t_probe)))
    X = g.standard_normal((ntok, cfg.din))
    dY = g.standard_normal((ntok, cfg.dout))
    t0 = time.perf_counter()
    linear.forward(Wp, X, A, B, cfg.s)
    linear.backward(Wp, X, A, B, cfg.s, dY)
    t_lin = time.perf_counter() - t0
    lin_full = t_lin * cfg.n / ntok
    info = {"kind": "oracle", "cores": int(blas_threads),
            "sample": f"codec (C, 1 thread) on {row_frac}x{cfg.din} of W0 (x{cfg.dout / row_frac:.0f}); "
                      f"fp64 fwd+bwd (NumPy BLAS) on {ntok} of {cfg.n} tokens (x{cfg.n / ntok:.0f}); "
                      f"measured {t_codec + t_lin:.2f} s",
            "codec_s_full": codec_full, "linear_s_full": lin_full}
    return codec_full + lin_full, info


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = _workload(args.workload)
    flops = cfg.fwd_flops() + cfg.bwd_flops()
    # the whole run stays within about two minutes of host time
    budget = max(0.5, min(15.0, 120.0 / (args.steps + 1)))
    for _ in range(args.warmup):
        oracle_sample(cfg, budget_s=0.05)
    times, info = [], None
    for _ in range(args.steps):
        t, info = oracle_sample(cfg, budget_s=budget)
        times.append(t)
    step_s = sum(times) / len(times)
    value = flops / step_s / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": cfg.name, "dout": cfg.dout, "din": cfg.din, "n": cfg.n, "r": cfg.r,
                      "parallelism": "host cores"},
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": info["cores"], "kind": "oracle",
                            "sample": info["sample"]},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


# ---------------------------------------------------------------------------
# Secondary measurements (reported under "parts", not part of the step)
# ---------------------------------------------------------------------------
def measure_decode(api, dev, copies=64, reps=5):
    """Decode-shaped forward (4096 x 4096, r = 16, n in {1, 4, 16}) over
    `copies` distinct NF4 + DQ weights (~553 MB, far above L2): one call per
    weight, captured once as a CUDA graph and replayed `reps` times between
    CUDA events, reported per call.  GB/s counts the algorithmic bytes of a
    call: codes, DQ constants, X, A, B, U and Y."""
    import torch
    from bit_nf4_quantized_07_b200 import synthetic
    cfg = synthetic.DECODE[1]
    rows, cols, r = cfg.dout, cfg.din, cfg.r
    gen = torch.Generator(device=dev)
    weights = []
    for i in range(copies):
        gen.manual_seed(7000 + i)
        W = torch.randn(rows, cols, generator=gen, device=dev) * cfg.w_sigma
        weights.append(api.quantize_weight(W))
        del W
    A = (torch.randn(r, cols, generator=gen, device=dev) * cfg.ab_sigma).to(torch.bfloat16)
    B = (torch.randn(rows, r, generator=gen, device=dev) * cfg.ab_sigma).to(torch.bfloat16)
    out = {}
    for n in (1, 4, 16):
        X = torch.randn(n, cols, generator=gen, device=dev).to(torch.bfloat16)
        Y = torch.empty(n, rows, dtype=torch.bfloat16, device=dev)
        U = torch.empty(n, r, dtype=torch.bfloat16, device=dev)
        ws = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_FWD, rows, cols, n, r), dev)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for w in weights[:4]:
                api.qlora_linear_fwd(w, X, A, B, 2.0, Y=Y, U_out=U, ws=ws)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for w in weights:
                api.qlora_linear_fwd(w, X, A, B, 2.0, Y=Y, U_out=U, ws=ws)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        per_call = e0.elapsed_time(e1) / (reps * copies) * 1e-3
        del graph
        bytes_call = decode_bytes_per_call(rows, cols, n, r)
        out[f"n{n}"] = {"us_per_call": per_call * 1e6, "GBs": bytes_call / per_call / 1e9,
                        "TFLOPs": 2 * n * (rows * cols + r * cols + rows * r) / per_call / 1e12,
                        "timing": f"CUDA graph of {copies} calls on {copies} weight copies, {reps} replays"}
    del weights
    torch.cuda.empty_cache()
    return out


def measure_sweep(api, dev, use_graph=True):
    """Quantize + DQ and dequant of every linear of a 32-layer d=4096,
    ffn=11008 decoder (6.48 B parameters, generated on the device), one pass
    each, CUDA events around each pass.  Quantize + DQ is one
    nf4_quantize_dq_batch call over all 224 matrices; dequant is one
    nf4_dequant call per matrix.  Each pass is a CUDA graph (use_graph=False:
    enqueued from Python)."""
    import torch
    from bit_nf4_quantized_07_b200 import synthetic
    gen = torch.Generator(device=dev)
    mats = []
    for layer in range(synthetic.SWEEP_LAYERS):
        for i, (_, rr, cc) in enumerate(synthetic.SWEEP_SHAPES):
            gen.manual_seed(5000 + 7 * layer + i)
            W = torch.randn(rr, cc, generator=gen, device=dev) * synthetic.SWEEP_SIGMA
            nb = rr * cc // 64
            mats.append((W, torch.empty(rr * cc // 2, dtype=torch.uint8, device=dev),
                         torch.empty(nb, dtype=torch.float32, device=dev),
                         torch.empty(nb, dtype=torch.int8, device=dev),
                         torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev),
                         torch.empty(1, dtype=torch.float32, device=dev)))
    ws = api.alloc_workspace(api.workspace_bytes(api.OP_QUANTIZE_DQ_BATCH, len(mats)), dev)
    jobs = [(W, c, a, q, sc, mu, "int8") for (W, c, a, q, sc, mu) in mats]
    outbuf = {}
    for W, *_ in mats:
        outbuf.setdefault(tuple(W.shape), torch.empty(W.shape, dtype=torch.bfloat16, device=dev))
    wq = [api.NF4Weight(codes=c, rows=W.shape[0], cols=W.shape[1], absmax=a, qabs=q, dq_scale=sc, dq_mean=mu)
          for (W, c, a, q, sc, mu) in mats]

    def quant_pass():  # the whole model in one call
        api.nf4_quantize_dq_batch(jobs, ws=ws)

    def deq_pass():
        for w in wq:
            api.nf4_dequant(w, outbuf[(w.rows, w.cols)])

    stream = torch.cuda.current_stream()
    quant_pass()
    deq_pass()
    torch.cuda.synchronize()
    run_q, run_d = quant_pass, deq_pass
    if use_graph:
        gq, gd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gq):
            quant_pass()
        with torch.cuda.graph(gd):
            deq_pass()
        gq.replay()
        gd.replay()
        torch.cuda.synchronize()
        run_q, run_d = gq.replay, gd.replay
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    e[0].record(stream)
    run_q()
    e[1].record(stream)
    run_d()
    e[2].record(stream)
    torch.cuda.synchronize()
    if use_graph:
        del gq, gd
    params = synthetic.sweep_params()
    qb, db = codec_bytes_per_param()
    tq, td = e[0].elapsed_time(e[1]) * 1e-3, e[1].elapsed_time(e[2]) * 1e-3
    del mats, jobs, wq, outbuf
    torch.cuda.empty_cache()
    return {"params": params, "quantize_dq_ms": tq * 1e3, "quantize_dq_GBs": params * qb / tq / 1e9,
            "dequant_ms": td * 1e3, "dequant_GBs": params * db / td / 1e9}


def measure_layer(api, dev, cfg, nsets=2, reps=4):
    """One layer's rows (quantize + DQ, dequant, forward, backward) on its own
    inputs: `nsets` input sets of the layer's shapes and distributions
    (seeded torch CUDA generators), each row captured as one CUDA graph of
    `reps` calls over the rotating sets and replayed 3 times between CUDA
    events; reported per call.  Used for the large layer (28672 x 8192,
    4096 tokens, r = 64), whose fp32 weight (940 MB) alone is far above L2."""
    import torch
    numel = cfg.dout * cfg.din
    nb = numel // 64
    gen = torch.Generator(device=dev)
    sets = []
    for i in range(nsets):
        gen.manual_seed(9000 + 10 * cfg.index + i)
        W = torch.randn(cfg.dout, cfg.din, generator=gen, device=dev) * cfg.w_sigma
        if cfg.outlier_rate > 0:
            m = torch.rand(cfg.dout, cfg.din, generator=gen, device=dev) < cfg.outlier_rate
            W = torch.where(m, W * 10.0, W)
            del m
        X = torch.randn(cfg.n, cfg.din, generator=gen, device=dev).to(torch.bfloat16)
        A = (torch.randn(cfg.r, cfg.din, generator=gen, device=dev) * cfg.ab_sigma).to(torch.bfloat16)
        B = (torch.randn(cfg.dout, cfg.r, generator=gen, device=dev) * cfg.ab_sigma).to(torch.bfloat16)
        dY = torch.randn(cfg.n, cfg.dout, generator=gen, device=dev).to(torch.bfloat16)
        sets.append((W.contiguous(), X, A, B, dY))
    codes = torch.empty(numel // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    qabs = torch.empty(nb, dtype=torch.int8, device=dev)
    scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    mu = torch.empty(1, dtype=torch.float32, device=dev)
    wdq = torch.empty(cfg.dout, cfg.din, dtype=torch.bfloat16, device=dev)
    Y = torch.empty(cfg.n, cfg.dout, dtype=torch.bfloat16, device=dev)
    U = torch.empty(cfg.n, cfg.r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(cfg.n, cfg.din, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(cfg.r, cfg.din, dtype=torch.float32, device=dev)
    dB = torch.empty(cfg.dout, cfg.r, dtype=torch.float32, device=dev)
    ws_dq = api.alloc_workspace(api.workspace_bytes(api.OP_DOUBLE_QUANT, nb), dev)
    ws_f = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_FWD, cfg.dout, cfg.din, cfg.n, cfg.r), dev)
    ws_b = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_BWD, cfg.dout, cfg.din, cfg.n, cfg.r), dev)
    wq = api.NF4Weight(codes=codes, rows=cfg.dout, cols=cfg.din, absmax=absmax, qabs=qabs, dq_scale=scale, dq_mean=mu)
    api.nf4_quantize_dq(sets[0][0], codes, absmax, qabs, scale, mu, ws=ws_dq)
    rows = {
        "quantize_dq": lambda i: api.nf4_quantize_dq(sets[i % nsets][0], codes, absmax, qabs, scale, mu, ws=ws_dq),
        "dequant": lambda i: api.nf4_dequant(wq, wdq),
        "fwd": lambda i: api.qlora_linear_fwd(wq, *sets[i % nsets][1:4], cfg.s, Y=Y, U_out=U, ws=ws_f),
        "bwd": lambda i: api.qlora_linear_bwd(wq, *sets[i % nsets][1:4], cfg.s, sets[i % nsets][4], U=U, dX=dX,
                                              dA=dA, dB=dB, ws=ws_b),
    }
    stream = torch.cuda.current_stream()
    ms = {}
    for k, fn in rows.items():
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for i in range(reps):
                fn(i)
        stream.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(reps):
                fn(i)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(3):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        del g
        ms[k] = e0.elapsed_time(e1) / (3 * reps)
    qb, db = codec_bytes_per_param()
    out = {"ms": ms, "fwd_TFLOPs": cfg.fwd_flops() / (ms["fwd"] * 1e-3) / 1e12,
           "bwd_TFLOPs": cfg.bwd_flops() / (ms["bwd"] * 1e-3) / 1e12,
           "quantize_dq_GBs": numel * qb / (ms["quantize_dq"] * 1e-3) / 1e9,
           "dequant_GBs": numel * db / (ms["dequant"] * 1e-3) / 1e9,
           "timing": f"CUDA graph of {reps} calls over {nsets} input sets, 3 replays"}
    del sets
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch

    from bit_nf4_quantized_07_b200 import api, dp, synthetic

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    rank, world, local = dp.init_from_env("cuda", timeout_s=120.0)
    cfg = _workload(args.workload)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # Inputs: NSETS rotating sets resident in HBM (each larger than a third of L2),
    # so every step reads inputs last touched two steps earlier.
    NSETS = 3
    gen = torch.Generator(device=dev)
    sets = []
    for i in range(NSETS):
        gen.manual_seed(1000 * cfg.index + 100 * rank + i)
        W = torch.randn(cfg.dout, cfg.din, generator=gen, device=dev) * cfg.w_sigma
        if cfg.outlier_rate > 0:
            m = torch.rand(cfg.dout, cfg.din, generator=gen, device=dev) < cfg.outlier_rate
            W = torch.where(m, W * 10.0, W)
        X = torch.randn(cfg.n, cfg.din, generator=gen, device=dev).to(torch.bfloat16)
        A = (torch.randn(cfg.r, cfg.din, generator=gen, device=dev) * cfg.ab_sigma).to(torch.bfloat16)
        B = (torch.randn(cfg.dout, cfg.r, generator=gen, device=dev) * cfg.ab_sigma).to(torch.bfloat16)
        dY = torch.randn(cfg.n, cfg.dout, generator=gen, device=dev).to(torch.bfloat16)
        sets.append((W.contiguous(), X, A, B, dY))
    numel = cfg.dout * cfg.din
    nb = numel // 64
    codes = torch.empty(numel // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    qabs = torch.empty(nb, dtype=torch.int8, device=dev)
    scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    mu = torch.empty(1, dtype=torch.float32, device=dev)
    wdq = torch.empty(cfg.dout, cfg.din, dtype=torch.bfloat16, device=dev)
    Y = torch.empty(cfg.n, cfg.dout, dtype=torch.bfloat16, device=dev)
    U = torch.empty(cfg.n, cfg.r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(cfg.n, cfg.din, dtype=torch.bfloat16, device=dev)
    ws_dq = api.alloc_workspace(api.workspace_bytes(api.OP_DOUBLE_QUANT, nb), dev)
    ws_f = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_FWD, cfg.dout, cfg.din, cfg.n, cfg.r), dev)
    ws_b = api.alloc_workspace(api.workspace_bytes(api.OP_LINEAR_BWD, cfg.dout, cfg.din, cfg.n, cfg.r), dev)
    wq = api.NF4Weight(codes=codes, rows=cfg.dout, cols=cfg.din, absmax=absmax, qabs=qabs, dq_scale=scale,
                       dq_mean=mu)

    ev = lambda: torch.cuda.Event(enable_timing=True)

    # AdamW state of the LoRA factors (one per input set): fp32 masters, the
    # 32-bit moments and the device step counter; the update writes the BF16
    # copies the next forward of that set reads.
    # A and B live in one flat buffer per set (masters, BF16 copies, moments),
    # and dA/dB in one flat gradient buffer, so one launch updates both.
    nA, nB = cfg.r * cfg.din, cfg.dout * cfg.r
    grad_flat = torch.empty(nA + nB, dtype=torch.float32, device=dev)
    dA, dB = grad_flat[:nA].view(cfg.r, cfg.din), grad_flat[nA:].view(cfg.dout, cfg.r)
    opt = []
    for k, (W_, X_, A, B, dY_) in enumerate(sets):
        flat16 = torch.cat([A.reshape(-1), B.reshape(-1)])
        A16, B16 = flat16[:nA].view(cfg.r, cfg.din), flat16[nA:].view(cfg.dout, cfg.r)
        sets[k] = (W_, X_, A16, B16, dY_)
        opt.append({"p32": flat16.float(), "p16": flat16, "m": torch.zeros(nA + nB, device=dev),
                    "v": torch.zeros(nA + nB, device=dev), "t": torch.zeros(1, dtype=torch.int64, device=dev)})
    ADAMW = dict(lr=1e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0)

    def step_body(i):
        W, X, A, B, dYs = sets[i % NSETS]
        api.nf4_quantize_dq(W, codes, absmax, qabs, scale, mu, ws=ws_dq)
        api.nf4_dequant(wq, wdq)
        api.qlora_linear_fwd(wq, X, A, B, cfg.s, Y=Y, U_out=U, ws=ws_f)
        api.qlora_linear_bwd(wq, X, A, B, cfg.s, dYs, U=U, dX=dX, dA=dA, dB=dB, ws=ws_b)

    def optim_body(i, p16=None):
        o = opt[i % NSETS]
        o["t"].add_(1)
        api.adamw_step(o["p32"], grad_flat, o["m"], o["v"], o["t"], param_bf16=o["p16"] if p16 is None else p16,
                       **ADAMW)

    # Rows of the step, for the per-row times.
    rows = {
        "quantize_dq": lambda i: api.nf4_quantize_dq(sets[i % NSETS][0], codes, absmax, qabs, scale, mu, ws=ws_dq),
        "quantize": lambda i: api.nf4_quantize(sets[i % NSETS][0], codes, absmax),
        "double_quant": lambda i: api.nf4_double_quant(absmax, qabs, scale, mu, ws=ws_dq),
        "dequant": lambda i: api.nf4_dequant(wq, wdq),
        "fwd": lambda i: api.qlora_linear_fwd(wq, *sets[i % NSETS][1:4], cfg.s, Y=Y, U_out=U, ws=ws_f),
        "bwd": lambda i: api.qlora_linear_bwd(wq, *sets[i % NSETS][1:4], cfg.s, sets[i % NSETS][4], U=U, dX=dX,
                                              dA=dA, dB=dB, ws=ws_b),
        "adamw": lambda i: optim_body(i),
    }

    # The step runs as a CUDA graph (one per input set): the library's calls
    # are enqueued once, at capture, and every replay launches the same
    # kernels.  --no-graph enqueues each call from Python instead.
    captured = [0]

    def capture(fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        l0 = api.launch_count()
        with torch.cuda.graph(g):
            fn()
        captured[0] = api.launch_count() - l0  # kernels in the graph
        torch.cuda.synchronize()
        return g

    graphs = None
    launches_per_step = 0
    if not args.no_graph:
        graphs = []
        for i in range(NSETS):
            g_main = capture(lambda i=i: step_body(i))
            n_main = captured[0]
            g_opt = capture(lambda i=i: optim_body(i))
            graphs.append((g_main, g_opt))
            launches_per_step = n_main + captured[0]

    def step(i):
        # codec + forward + backward, the data-parallel all-reduce of dA/dB
        # (N > 1), then the optimizer
        if graphs is not None:
            dp.train_step(graphs[i % NSETS][0].replay, graphs[i % NSETS][1].replay, dA, dB, world)
        else:
            dp.train_step(lambda: step_body(i), lambda: optim_body(i), dA, dB, world)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    dp.barrier(world)
    torch.cuda.synchronize()

    start, stop = ev(), ev()
    launches0 = api.launch_count()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(i)
        stop.record(stream)
        torch.cuda.synchronize()
    launches = api.launch_count() - launches0 if graphs is None else launches_per_step * args.steps
    dp.barrier(world)
    torch.cuda.synchronize()
    elapsed_ms = start.elapsed_time(stop)
    if world > 1:
        elapsed_ms = dp.max_over_ranks(elapsed_ms, device=dev)

    # Per-row device times: each row alone, 2 * NSETS calls (rotating inputs)
    # captured in one graph, replayed 3 times between CUDA events.
    def row_ms(fn, reps=2 * NSETS):
        g = capture(lambda: [fn(i) for i in range(reps)])
        g.replay()
        a0, a1 = ev(), ev()
        a0.record(stream)
        for _ in range(3):
            g.replay()
        a1.record(stream)
        torch.cuda.synchronize()
        del g
        return a0.elapsed_time(a1) / (3 * reps)

    sec = {k: row_ms(f) for k, f in rows.items()}
    codec_split = {"quantize_ms": sec.pop("quantize"), "double_quant_ms": sec.pop("double_quant")}
    if graphs is not None:
        del graphs
        torch.cuda.synchronize()

    # End to end through the C ABI with host buffers: copies inside the timed region.
    W, X, A, B, dYs = sets[0]
    hW, hX, hA, hB, hdY = (t.cpu().pin_memory() for t in (W, X, A, B, dYs))
    dW, dXi, ddY = (torch.empty_like(t) for t in (W, X, dYs))
    dflat16 = torch.empty(nA + nB, dtype=torch.bfloat16, device=dev)
    dAi, dBi = dflat16[:nA].view(cfg.r, cfg.din), dflat16[nA:].view(cfg.dout, cfg.r)
    oY, odX, odA, odB = (torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (Y, dX, dA, dB))

    def e2e_step():
        for d, h in ((dW, hW), (dXi, hX), (dAi, hA), (dBi, hB), (ddY, hdY)):
            d.copy_(h, non_blocking=True)
        api.nf4_quantize_dq(dW, codes, absmax, qabs, scale, mu, ws=ws_dq)
        api.nf4_dequant(wq, wdq)
        api.qlora_linear_fwd(wq, dXi, dAi, dBi, cfg.s, Y=Y, U_out=U, ws=ws_f)
        api.qlora_linear_bwd(wq, dXi, dAi, dBi, cfg.s, ddY, U=U, dX=dX, dA=dA, dB=dB, ws=ws_b)
        if world > 1:
            dp.allreduce_adapter_grads(dA, dB)
        optim_body(0, p16=dflat16)
        for h, d in ((oY, Y), (odX, dX), (odA, dA), (odB, dB)):
            h.copy_(d, non_blocking=True)

    h2d = sum(t.numel() * t.element_size() for t in (hW, hX, hA, hB, hdY))
    d2h = sum(t.numel() * t.element_size() for t in (oY, odX, odA, odB))
    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    dp.barrier(world)
    e0, e1 = ev(), ev()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        e2e_ms = dp.max_over_ranks(e2e_ms, device=dev)

    flops = cfg.fwd_flops() + cfg.bwd_flops()
    ms_per_step = elapsed_ms / args.steps
    value = world * flops / (ms_per_step * 1e-3) / 1e12
    e2e_value = world * flops / (e2e_ms / e2e_steps * 1e-3) / 1e12
    peaks = _load_peaks()
    qb, db = codec_bytes_per_param()
    fwd_tflops = cfg.fwd_flops() / (sec["fwd"] * 1e-3) / 1e12
    roof = {"kernel": "qlora_linear_fwd (fused NF4 GEMM + U)", "bound": "tensor", "achieved": fwd_tflops,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": fwd_tflops / peaks["bf16_tflops"],
            "traffic": _recorded_traffic(cfg.name), "peak_source": peaks["source"] + " bf16 burst"}
    parts = {
        "quantize_dq_GBs": numel * qb / (sec["quantize_dq"] * 1e-3) / 1e9,
        "quantize_dq_split": codec_split,
        "dequant_GBs": numel * db / (sec["dequant"] * 1e-3) / 1e9,
        "fwd_TFLOPs": fwd_tflops,
        "bwd_TFLOPs": cfg.bwd_flops() / (sec["bwd"] * 1e-3) / 1e12,
        "adamw_GBs": 30 * cfg.r * (cfg.din + cfg.dout) / (sec["adamw"] * 1e-3) / 1e9,
        "ms": sec,
        "hbm_peak_GBs": peaks["hbm_gbs"],
    }
    parts["quantize_dq_frac_hbm"] = parts["quantize_dq_GBs"] / peaks["hbm_gbs"]
    parts["dequant_frac_hbm"] = parts["dequant_GBs"] / peaks["hbm_gbs"]
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": cfg.name, "dout": cfg.dout, "din": cfg.din, "n": cfg.n, "r": cfg.r, "s": cfg.s,
                      "global_batch": cfg.n * world, "parallelism": f"dp{world}",
                      "step": "nf4_quantize_dq+nf4_dequant+qlora_linear_fwd+qlora_linear_bwd"
                              "+qln_adamw_step(A,B)",
                      "l2": l2_note(cfg, NSETS),
                      "timing": "python-enqueued steps" if args.no_graph else
                      "CUDA graph replay per step (one graph per input set)"},
           "gpu_launches": launches, "roofline": roof, "parts": parts, "clocks": clk.summary(),
           "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}}
    if not args.no_extra:
        del sets
        torch.cuda.empty_cache()
        parts["decode_4096x4096_r16"] = measure_decode(api, dev)
        for k, v in parts["decode_4096x4096_r16"].items():
            v["frac_hbm"] = v["GBs"] / peaks["hbm_gbs"]
        lg = measure_layer(api, dev, synthetic.LARGE)
        lg["fwd_frac_bf16"] = lg["fwd_TFLOPs"] / peaks["bf16_tflops"]
        lg["bwd_frac_bf16"] = lg["bwd_TFLOPs"] / peaks["bf16_tflops"]
        lg["quantize_dq_frac_hbm"] = lg["quantize_dq_GBs"] / peaks["hbm_gbs"]
        lg["dequant_frac_hbm"] = lg["dequant_GBs"] / peaks["hbm_gbs"]
        lg["roofline_traffic"] = _recorded_traffic(synthetic.LARGE.name)
        parts["large_28672x8192_n4096_r64"] = lg
        sw = measure_sweep(api, dev, use_graph=not args.no_graph)
        sw["quantize_dq_frac_hbm"] = sw["quantize_dq_GBs"] / peaks["hbm_gbs"]
        sw["dequant_frac_hbm"] = sw["dequant_GBs"] / peaks["hbm_gbs"]
        parts["sweep_6.48B"] = sw
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        step_s, info = oracle_sample(cfg)
        out["cpu_baseline"] = {"value": flops / step_s / 1e12, "unit": "TFLOP/s", "cores": info["cores"],
                               "kind": "oracle", "sample": info["sample"]}
    dp.finish(world)
    if rank == 0:
        print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "large", "pr1"], default="prefill")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="enqueue every call from Python instead of replaying "
                    "CUDA graphs of the step, the rows and the sweep")
    ap.add_argument("--no-extra", action="store_true", help="skip the decode-shape and codec-sweep measurements")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode-shape measurement and print it (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.decode_only:
        import torch
        from bit_nf4_quantized_07_b200 import api
        print(json.dumps(measure_decode(api, torch.device("cuda", 0), copies=16, reps=2)))
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
