#!/usr/bin/env python
"""GDLA forward benchmark on B200: one JSON line on rank 0.

A step is one pass of the whole hot path over one batch of synthetic input:
  * prefill of B=1 x T=32768 tokens, full causal (the layer's headline workload), and
  * absorbed-form decode of B=64 sequences with 32768 cached positions, causal and SWA W=2048.
`value` is the prefill throughput of the whole layer (algorithmic FLOPs / time); decode
figures ride along under "decode".  Inputs are resident in HBM when the timed region starts;
"e2e" repeats the prefill through the C ABI with host buffers (pinned H2D of x, D2H of y).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
       (N > 1: launch under torch.distributed.run; every rank runs the same per-GPU workload.)
"""
from __future__ import annotations

import argparse
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

METRIC = "GDLA prefill TFLOP/s (% BF16 peak) at 32K; decode tok/s & KV GB/s vs HBM"
PREFILL = dict(name="prefill_b1_t32768_causal", B=1, T=32768, window=0, seed=2)
DECODE = dict(B=64, L=32768, seed=4, windows=(0, 2048), multi=(2, 3))
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- work accounting
def layer_dims():
    from differential_latent_attention_fwd_b200.synth import GdlaShape
    return GdlaShape()


def valid_pairs(T: int, window: int) -> int:
    if window <= 0 or window >= T:
        return T * (T + 1) // 2
    return window * (window + 1) // 2 + (T - window) * window


def attn_flops_per_pair(s) -> int:
    return s.n_heads * 2 * (s.d_qk + s.d_v)          # QK^T and PV over every head


def proj_flops_per_token(s) -> int:
    nqq = s.n_heads * s.d_qk
    return 2 * (s.d_model * s.q_rank + s.d_model * (s.kv_rank + s.d_rope) + s.d_model * s.n_signal
                + s.q_rank * nqq + s.q_rank * s.n_signal * s.d_v + s.kv_rank * s.n_kv_heads * (s.d_nope + s.d_v)
                + s.n_signal * s.d_v * s.d_model)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured (MEASURED_PEAKS.json)"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons, n = [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            n += 1
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        loaded = [v for v in sm if v >= 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "samples": n,
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- CPU oracle sample
def oracle_prefill_sample(inp, n_rows: int, seed: int):
    """Time the fp64 oracle on n_rows query rows of the prefill workload (it still forms the
    latent/K/V rows of every earlier token).  Returns (seconds, flops of the work done)."""
    import numpy as np
    from oracle import gdla_oracle as O
    s = inp.shape
    T = inp.x.shape[1]
    rng = np.random.default_rng(seed)
    rows = sorted(set(int(r) for r in rng.integers(0, T, n_rows)))
    cfg = O.OracleConfig.from_shape(s)
    t0 = time.perf_counter()
    O.gdla_prefill(inp.x, inp.weights, cfg, rows=rows, g_q=inp.g_q, g_kv=inp.g_kv)
    dt = time.perf_counter() - t0
    t_hi = max(rows) + 1
    kv_flops = 2 * t_hi * (s.d_model * (s.kv_rank + s.d_rope) + s.kv_rank * s.n_kv_heads * (s.d_nope + s.d_v))
    row_flops = len(rows) * (proj_flops_per_token(s) - 2 * (s.d_model * (s.kv_rank + s.d_rope)
                                                           + s.kv_rank * s.n_kv_heads * (s.d_nope + s.d_v)))
    attn = sum(min(r + 1, s.window if s.window else r + 1) for r in rows) * attn_flops_per_pair(s)
    return dt, kv_flops + row_flops + attn, rows


def threads_used() -> int:
    for v in ("OPENBLAS_NUM_THREADS", "OMP_NUM_THREADS"):
        if os.environ.get(v, "").isdigit():
            return int(os.environ[v])
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle, as it stands, on host cores: each step = a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from differential_latent_attention_fwd_b200 import synth
    s = layer_dims()
    inp = synth.make_prefill_inputs(s, PREFILL["B"], PREFILL["T"], PREFILL["seed"])
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        dt, fl, rows = oracle_prefill_sample(inp, 2, seed=100 + i)
        if i >= args.warmup:
            times.append(dt)
            flops.append(fl)
    tf = sum(flops) / sum(times) / 1e12
    sample = (f"per step: 2 uniformly drawn query rows of {PREFILL['name']} (all 80 heads), "
              "with the latent/K/V rows of every earlier token; fp64 numpy")
    line = {"impl": "reference", "metric": METRIC, "value": tf, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PREFILL["name"], "B": PREFILL["B"], "seq_len": PREFILL["T"],
                       "mask": "causal"},
            "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": threads_used(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def run_gpu(args):
    import torch
    import torch.distributed as dist

    from differential_latent_attention_fwd_b200 import binding as gb
    from differential_latent_attention_fwd_b200 import synth
    from differential_latent_attention_fwd_b200.layer import GdlaLayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))

    s = layer_dims()
    B, T = PREFILL["B"], args.T
    inp = synth.make_prefill_inputs(s, B, T, PREFILL["seed"])
    layer = GdlaLayer(s, inp.weights, inp.g_q, inp.g_kv, device=dev)
    x_host = inp.x.pin_memory()
    x = x_host.to(dev, non_blocking=True)
    y = torch.empty_like(x)
    ws = layer.workspace(B, T, gb.GDLA_MODE_PREFILL)
    windows = () if args.skip_decode else DECODE["windows"]
    dec_L = 1 if args.skip_decode else args.decode_L
    qmax = max(DECODE["multi"])
    # cache capacity: the cached positions plus room for up to qmax new tokens per sequence
    dinp = synth.make_decode_inputs(synth.GdlaShape(), DECODE["B"], dec_L, dec_L + qmax, DECODE["seed"])
    cache = dinp.cache.to(dev)
    lens = dinp.cache_len.to(dev)
    x_new = dinp.x_new.to(dev)
    y_new = torch.empty_like(x_new)
    multis = () if args.skip_decode else DECODE["multi"]
    x_multi = {q: torch.randn((DECODE["B"], q, s.d_model), generator=torch.Generator().manual_seed(6 + q))
               .bfloat16().to(dev) for q in multis}
    y_multi = {q: torch.empty_like(x_multi[q]) for q in multis}
    # the same cache stored as MXFP8 rows (608 bytes a position instead of 1152)
    cache8 = layer.quantize_latent_fp8(cache) if windows else None
    y_new8 = torch.empty_like(x_new)
    absorbed = layer.absorbed()
    dcfg = {w: gb.make_config(s.with_window(w)) for w in (0, 2048)}
    dws = torch.empty(max(gb.gdla_workspace_size(dcfg[w], DECODE["B"] * qmax, cache.shape[1],
                                                 gb.GDLA_MODE_DECODE) for w in (0, 2048)),
                      dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream(dev)
    pev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    dev_ev = {k: [torch.cuda.Event(enable_timing=True) for _ in range(5)]
              for k in ["c", "w2048", "c_q2", "c_q3", "c_fp8"]}

    def prefill_once():
        gb.gdla_set_stage_events(pev)
        gb.gdla_prefill_fwd(layer.cfg, layer.cw, x, y, ws, stream=stream)

    # A decode step is ~20 short kernels: it is replayed as a CUDA graph (one capture per
    # configuration), as a serving loop runs it; the eager time is reported beside it.  Decode
    # is timed as its own run of back-to-back replays (continuous decoding), not right after a
    # prefill, whose power draw would leave the decode at the prefill's reduced clocks; the
    # caches (2.4 GB causal, 151 MB for the 2048 window) exceed the 126 MB L2, so no flush.
    dec_keys = [("c" if w == 0 else f"w{w}", w, 1) for w in windows] + [(f"c_q{q}", 0, q) for q in multis]
    if windows:
        dec_keys.append(("c_fp8", 0, 1))

    def decode_call(key, st):
        _, w, q = next(d for d in dec_keys if d[0] == key)
        if key == "c_fp8":
            gb.gdla_decode_fp8_fwd(dcfg[0], absorbed, x_new, cache8, lens, y_new8, dws, stream=st)
        elif q == 1:
            gb.gdla_decode_fwd(dcfg[w], absorbed, x_new, cache, lens, y_new, dws, stream=st)
        else:
            gb.gdla_decode_multi_fwd(dcfg[w], absorbed, x_multi[q], cache, lens, y_multi[q], dws, stream=st)

    graphs = {}
    ev_pairs = {k: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)] for k, _, _ in dec_keys}

    def prefill_step():
        flush.fill_(1)
        prefill_once()
        torch.cuda.synchronize(dev)
        return {"prefill_ms": pev[0].elapsed_time(pev[5]), "attn_ms": pev[3].elapsed_time(pev[4]),
                "down_ms": pev[0].elapsed_time(pev[1]), "norm_ms": pev[1].elapsed_time(pev[2]),
                "up_ms": pev[2].elapsed_time(pev[3]), "out_ms": pev[4].elapsed_time(pev[5])}

    def decode_run(key, n, record=True):
        for i in range(n):
            if record:
                ev_pairs[key][i][0].record(stream)
            graphs[key].replay()
            if record:
                ev_pairs[key][i][1].record(stream)
        torch.cuda.synchronize(dev)
        return [a.elapsed_time(b) for a, b in ev_pairs[key][:n]] if record else []

    for _ in range(0 if args.skip_prefill else max(3, args.warmup)):
        prefill_step()
    assert gb.gdla_device_error(stream) == 0, "device error during warm-up"
    gb.gdla_set_stage_events([])     # no event nodes inside the captured graphs
    for k, _, _ in dec_keys:         # one eager call each before capture (first-use set-up)
        decode_call(k, stream)
    torch.cuda.synchronize(dev)
    for k, _, _ in dec_keys:
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(dev)
        cs.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                decode_call(k, cs)
        torch.cuda.current_stream(dev).wait_stream(cs)
        graphs[k] = g
    for k, _, _ in dec_keys:
        decode_run(k, max(3, args.warmup), record=False)
    torch.cuda.synchronize(dev)
    assert gb.gdla_device_error(stream) == 0, "device error in graph warm-up"
    # the per-stage split of a decode call comes from eager calls with stage events, made after
    # the graph warm-up (so at the decode's clocks, not the prefill's); the L2 is flushed first
    eager_dec = {k: [] for k, _, _ in dec_keys}
    eager_stage = {k: {"attn": [], "q": [], "comb": []} for k, _, _ in dec_keys}
    kernels_per_decode = {}
    for _ in range(5):
        for k, _, _ in dec_keys:
            flush.fill_(1)
            n0 = gb.gdla_kernel_launches()
            gb.gdla_set_stage_events(dev_ev[k])
            decode_call(k, stream)
            kernels_per_decode[k] = gb.gdla_kernel_launches() - n0
            torch.cuda.synchronize(dev)
            e = dev_ev[k]
            eager_dec[k].append(e[0].elapsed_time(e[4]))
            eager_stage[k]["attn"].append(e[1].elapsed_time(e[2]))
            eager_stage[k]["q"].append(e[0].elapsed_time(e[1]))
            eager_stage[k]["comb"].append(e[2].elapsed_time(e[3]))
    gb.gdla_set_stage_events([])

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    barrier()
    launches0 = gb.gdla_kernel_launches()
    recs = []
    dec_ms = {}
    # decode first (its graph warm-up just ran: the GPU is in its decode state), then prefill;
    # clocks are sampled over each part and over the whole timed region
    with ClockSampler(local) as clk:
        with ClockSampler(local) as clk_dec:
            for k, _, _ in dec_keys:
                dec_ms[k] = decode_run(k, args.steps)
            barrier()
        with ClockSampler(local) as clk_pre:
            for _ in range(0 if args.skip_prefill else args.steps):
                recs.append(prefill_step())
            barrier()
    # graph replays launch the captured kernels without passing through the library's counter
    launches = gb.gdla_kernel_launches() - launches0 + args.steps * sum(kernels_per_decode.values())
    gb.gdla_set_stage_events([])
    site = gb.gdla_device_error(stream)
    assert site == 0, f"device error site {site:#x} in the timed region"
    if not recs:
        recs = [{"prefill_ms": 0.0, "attn_ms": float("nan"), "down_ms": 0.0, "norm_ms": 0.0, "up_ms": 0.0,
                 "out_ms": 0.0}]
    for r in recs:
        for k in dec_ms:
            r[f"dec_{k}_ms"] = statistics.mean(dec_ms[k])

    def mean(k):
        return statistics.mean(r[k] for r in recs)

    keys = list(recs[0].keys())
    local_stats = torch.tensor([mean(k) for k in keys], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(local_stats, op=dist.ReduceOp.MAX)
    st = dict(zip(keys, local_stats.tolist()))

    # ---- end to end through the C ABI with host buffers: gdla_prefill_host_fwd takes x from and
    # writes y to pinned host memory, its copies overlapping the row-separable stages
    y_host = torch.empty_like(x_host).pin_memory()
    ws_host = torch.empty(gb.gdla_workspace_size(layer.cfg, B, T, gb.GDLA_MODE_HOST) if not
                          (args.skip_e2e or args.skip_prefill) else 1, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = []
    for i in range(0 if (args.skip_e2e or args.skip_prefill) else max(2, min(args.steps, 5)) + 1):
        flush.fill_(1)
        barrier()
        e0.record(stream)
        gb.gdla_prefill_host_fwd(layer.cfg, layer.cw, x_host, y_host, ws_host, n_pieces=16, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if i > 0:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e_t = torch.tensor([statistics.mean(e2e_ms) if e2e_ms else float("nan")], dtype=torch.float64,
                         device=dev)
    if world > 1:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)

    # ---- context parallelism: per-rank compute of an 8-way split of the same sequence (its
    # latent pass + its tokens after the latent rows of every earlier token); the exchange of
    # latent rows between ranks needs several GPUs and is reported as bytes only
    cp = None
    if not (args.skip_prefill or args.skip_cp) and world == 1:
        P = 8
        Tr = T // P
        lat_all = layer.latent(x[0], 0)
        lat_r = torch.empty((Tr, s.latent_row), dtype=torch.bfloat16, device=dev)
        y_r = torch.empty((Tr, s.d_model), dtype=torch.bfloat16, device=dev)
        cp_ms = {}
        for r in (0, P - 1):
            xr = x[0, r * Tr:(r + 1) * Tr]
            prefix = lat_all[: r * Tr] if r else None
            times = []
            for i in range(4):
                flush.fill_(1)
                e0.record(stream)
                layer.latent(xr, r * Tr, out=lat_r, stream=stream)
                layer.prefill_context(xr, r * Tr, prefix, y=y_r, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize(dev)
                if i:
                    times.append(e0.elapsed_time(e1))
            cp_ms[r] = statistics.median(times)
        last_pairs = Tr * (P - 1) * Tr + Tr * (Tr + 1) // 2
        last_flop = (last_pairs * attn_flops_per_pair(s) + Tr * proj_flops_per_token(s)
                     + (P - 1) * Tr * 2 * s.kv_rank * s.n_kv_heads * (s.d_nope + s.d_v))
        cp = {"ranks": P, "tokens_per_rank": Tr, "first_rank_ms": cp_ms[0],
              "last_rank_ms": cp_ms[P - 1], "last_rank_tflops": last_flop / (cp_ms[P - 1] * 1e-3) / 1e12,
              "exchanged_bytes_per_token": s.latent_row * 2,
              "last_rank_receives_bytes": (P - 1) * Tr * s.latent_row * 2,
              "timing": "one GPU, each rank's two calls back to back (L2 flushed); no communication"}

    # ---- training: the attention stage's saving forward and its backward on the projected
    # inputs the prefill left in its workspace (dL/dDg synthetic, seeded)
    bwd = None
    if not (args.skip_prefill or args.skip_bwd) and world == 1 and B == 1:
        def slot(which, dtype, shape):
            o = gb.gdla_workspace_offset(layer.cfg, B, T, gb.GDLA_MODE_PREFILL, which)
            n = int(math.prod(shape)) * torch.empty((), dtype=dtype).element_size()
            return ws[o: o + n].view(dtype).view(*shape)
        M = B * T
        nH = s.n_signal + s.n_noise
        qq = slot(4, torch.float16, (M, nH * 192)); kvs = slot(6, torch.float16, (M, s.n_kv_heads * 256))
        kr = slot(9, torch.float16, (M, 64)); lam_t = slot(3, torch.float32, (M, s.n_signal))
        gate = slot(5, torch.bfloat16, (M, s.n_signal * 128))
        fb, bb = gb.gdla_attn_train_workspace_size(layer.cfg, B, T)
        wsf = torch.empty(fb, dtype=torch.uint8, device=dev)
        wsb = torch.empty(bb, dtype=torch.uint8, device=dev)
        dg_t = torch.empty((M, s.n_signal * 128), dtype=torch.bfloat16, device=dev)
        h_t = torch.empty((M, nH, 128), dtype=torch.bfloat16, device=dev)
        lse_t = torch.empty((M, nH), dtype=torch.float32, device=dev)
        ddg = torch.randn((M, s.n_signal * 128), generator=torch.Generator(device=dev).manual_seed(9),
                          device=dev).bfloat16()
        grads = [torch.empty((M, nH * 192), device=dev), torch.empty((M, s.n_kv_heads * 256), device=dev),
                 torch.empty((M, 64), device=dev), torch.empty((M, s.n_signal), device=dev),
                 torch.empty((M, s.n_signal * 128), device=dev)]
        e2 = torch.cuda.Event(enable_timing=True)
        tf_ms, tb_ms = [], []
        for i in range(3):
            e0.record(stream)
            gb.gdla_attn_train_fwd(layer.cfg, qq, kvs, kr, lam_t, gate, B, T, dg_t, h_t, lse_t, wsf, stream=stream)
            e1.record(stream)
            gb.gdla_attn_bwd(layer.cfg, qq, kvs, kr, lam_t, gate, h_t, lse_t, ddg, B, T, *grads, wsb, stream=stream)
            e2.record(stream)
            torch.cuda.synchronize(dev)
            if i:
                tf_ms.append(e0.elapsed_time(e1))
                tb_ms.append(e1.elapsed_time(e2))
        bwd_flop = B * valid_pairs(T, 0) * nH * 2 * (192 + 128 + 192 + 192 + 128)
        bwd = {"seq_len": T, "train_fwd_ms": statistics.median(tf_ms), "bwd_ms": statistics.median(tb_ms),
               "bwd_flop": bwd_flop, "bwd_tflops": bwd_flop / (statistics.median(tb_ms) * 1e-3) / 1e12,
               "bwd_frac_of_bf16_peak": bwd_flop / (statistics.median(tb_ms) * 1e-3) / 1e12
               / load_peaks()[0]["bf16_tflops_sustained"],
               "method": "tcgen05 kernels (fp16 operands, fp32 accumulators in TMEM): keys-stationary dK/dV "
                         "per (KV group, 128 keys) over 64-query tiles x 5 heads, queries-stationary dq per "
                         "(head, 128 queries) over 64-key tiles; P recomputed from the saved log-sum-exp; "
                         "plus dH/Delta/dlambda/dG, gathers and the dk^R sum"}
        del wsb, grads, h_t

    peaks, peak_src = load_peaks()
    pairs = valid_pairs(T, 0)
    attn_flop = B * pairs * attn_flops_per_pair(s)
    layer_flop = attn_flop + B * T * proj_flops_per_token(s)
    def tflops(flop, ms):
        return flop / (ms * 1e-3) / 1e12 if ms and ms == ms and ms > 0 else float("nan")

    value = world * tflops(layer_flop, st["prefill_ms"])
    attn_tf = tflops(attn_flop, st["attn_ms"])
    e2e_val = world * tflops(layer_flop, e2e_t.item())

    decode = {}
    for k, w, q in dec_keys:
        keys_read = dec_L + q if w == 0 else min(w, dec_L + q)
        row_bytes = gb.FP8_ROW_BYTES if k == "c_fp8" else s.latent_row * 2
        kv_bytes = DECODE["B"] * keys_read * row_bytes                # each sequence's rows, once
        t_att = statistics.median(eager_stage[k]["attn"]) * 1e-3
        t_all = st[f"dec_{k}_ms"] * 1e-3
        name = ("causal" if w == 0 else f"swa{w}") + ("" if q == 1 else f"_q{q}") + ("_fp8" if k == "c_fp8" else "")
        decode[name] = {
            "B": DECODE["B"], "cache_len": dec_L, "window": w, "q_len": q,
            "tok_per_s": world * DECODE["B"] * q / t_all, "ms": st[f"dec_{k}_ms"],
            "timing": f"{args.steps} back-to-back CUDA graph replays of one decode call (mean)",
            "ms_eager": statistics.median(eager_dec[k]),
            "latent_attention_ms": statistics.median(eager_stage[k]["attn"]),
            "query_path_ms": statistics.median(eager_stage[k]["q"]),
            "combine_ms": statistics.median(eager_stage[k]["comb"]),
            "kv_bytes": kv_bytes, "kv_gbs": kv_bytes / t_att / 1e9,
            "kv_frac_of_hbm": kv_bytes / t_att / 1e9 / peaks["hbm_gbs"],
        }
        if k == "c_fp8":
            decode[name]["kv_note"] = ("MXFP8 latent cache: 608 bytes per cached position (576 E4M3 "
                                       "values, 18 block scales, padding) against 1152 in bf16")
        if q > 1:
            decode[name]["kv_note"] = ("kv_bytes counts each sequence's cache rows once: the rows of its "
                                       f"{q} new tokens are consecutive query rows, whose CTAs read the same "
                                       "tiles at about the same time (shared in L2)")

    traffic = None
    tf_path = os.path.join(ROOT, "profiles", "attn_prefill_t32768_causal.traffic.json")
    try:
        with open(tf_path) as f:
            tr = json.load(f)
        if tr.get("kernel_source_sha256") == kernel_source_digest():
            traffic = tr.get("dram_bytes_per_launch")
    except Exception:
        traffic = None

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": st["prefill_ms"] + sum(
            st[f"dec_{k}_ms"] for k, _, q in dec_keys if q == 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": (f"prefill_b1_t{T}_causal" + ("" if args.skip_decode else
                                " (+ decode_b64_l32768 causal and swa2048)")),
                   "B": B, "seq_len": T, "mask": "causal", "d_model": s.d_model,
                   "heads": f"{s.n_signal} signal + {s.n_noise} noise, {s.n_kv_heads} KV",
                   "attn_operands": "fp16 (q, K^C, V, k^R, P); projections bf16; fp32 accumulate",
                   "l2": "flushed (256 MiB write) before every timed prefill call; decode caches exceed L2",
                   "parallelism": f"replicas x{world}"},
        "prefill": {"layer_ms": st["prefill_ms"], "attention_ms": st["attn_ms"],
                    "down_proj_ms": st["down_ms"], "norm_rope_ms": st["norm_ms"],
                    "up_proj_ms": st["up_ms"], "out_proj_ms": st["out_ms"],
                    "layer_flop": layer_flop, "attention_flop": attn_flop,
                    "attention_tflops": attn_tf, "tok_per_s": world * B * T / max(st["prefill_ms"] * 1e-3, 1e-12),
                    "layer_frac_of_bf16_peak": value / world / peaks["bf16_tflops_sustained"]},
        "decode": decode,
        "context_parallel": cp,
        "backward": bwd,
        # the attention kernel is timed per call, on its own (L2 flushed, events around the one
        # launch): the burst GEMM peak is its denominator; the sustained one rides along
        "roofline": {"kernel": "attn_prefill_kernel", "bound": "tensor", "achieved": attn_tf,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": attn_tf / peaks["bf16_tflops"],
                     "frac_of_sustained_peak": attn_tf / peaks["bf16_tflops_sustained"],
                     "peak_source": peak_src + ", burst bf16 (fp16 has the same dense rate)",
                     "traffic": traffic},
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": x.numel() * 2,
                "d2h_bytes_per_step": y.numel() * 2, "ms": e2e_t.item()},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "clocks_decode_part": clk_dec.summary(),
        "clocks_prefill_part": clk_pre.summary(),
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.skip_prefill:
        dt, fl, rows = oracle_prefill_sample(inp, 8, seed=7)
        line["cpu_baseline"] = {
            "value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads_used(), "kind": "oracle",
            "sample": f"{len(rows)} uniformly drawn query rows of {PREFILL['name']} (all 80 heads) "
                      f"plus the latent/K/V rows of tokens 0..{max(rows)}; fp64 numpy; {dt:.1f} s"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def kernel_source_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ("attn_prefill.cu", "gdla_common.cuh"):
        with open(os.path.join(ROOT, "differential_latent_attention_fwd_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="gdla", choices=["gdla", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--T", type=int, default=PREFILL["T"], help="prefill length (profiling runs)")
    ap.add_argument("--skip-decode", action="store_true", help="profiling runs: prefill only")
    ap.add_argument("--skip-prefill", action="store_true", help="profiling runs: decode only")
    ap.add_argument("--skip-e2e", action="store_true", help="profiling runs: no host-buffer pass")
    ap.add_argument("--decode-L", type=int, default=DECODE["L"], help="cached positions (profiling runs)")
    ap.add_argument("--skip-cp", action="store_true", help="profiling runs: no context-parallel split")
    ap.add_argument("--skip-bwd", action="store_true", help="profiling runs: no backward pass")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
