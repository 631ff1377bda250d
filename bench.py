"""Benchmark of the DCA hot path on B200.

One step = one pass of the whole path on synthetic data:
  prefill  (the 100k-token workload: L=100000, 64 query / 8 kv heads, D=128,
            c=4096, s=3072, ragged last chunk): fused RoPE, then DCA attention;
  decode   (16 sequences, 64/8 heads, D=128, t ~ U[32768, 65536), cache
            pre-rotated at j mod s): split-KV kernel, then LSE merge.
`value` is prefill TFLOP/s (algorithmic causal FLOPs 4*D*Hq*B*L(L+1)/2 over
the device time of RoPE + attention); decode KV GB/s is reported beside it.
The other prefill workloads (Llama-2 70B-shaped GQA at 32k tokens with K
doubled on 1% of positions, Llama-2 7B-shaped at 16k, and the tiny one) are
timed after the step, each on its own inputs, and reported under `configs`.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: one process per GPU; every rank runs its own replica (the path has
no exchange step), times are max-reduced over ranks.  Under torchrun
WORLD_SIZE must equal --gpus; without torchrun, --gpus N > 1 starts N local
ranks itself through torch.distributed.run.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_attention_dca_b200 import workloads as W  # noqa: E402

PREFILL = "prefill_100k"
# prefill workloads timed after the step, each reported on its own
SUB_CONFIGS = ("llama2_70b_32k", "llama2_7b_16k", "tiny")
# workload of the calls beyond the step (chunked, packed, three passes, ...)
NEXT_ROWS_WORKLOAD = "llama2_7b_16k"
DECODE = "decode_b16"
METRIC = "DCA prefill TFLOP/s (bf16, % of TC peak); decode KV GB/s (% of HBM peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic():
    """Per-launch DRAM bytes of the dominant kernels from the committed ncu
    summary (profiles/traffic.json), or {} when none was captured."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return {}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the prefill workload
# ---------------------------------------------------------------------------
class _F64:
    """float64 numpy view of a CPU torch tensor, converted per index."""

    def __init__(self, t):
        self.t, self.shape = t, tuple(t.shape)

    def __getitem__(self, idx):
        return self.t[idx].to(torch.float64).numpy()


_CPU_INPUTS = {}


def oracle_sample(budget_s: float, seed: int = 0, name: str = PREFILL):
    """Time the oracle on random (row, head) outputs of a prefill workload
    until `budget_s` seconds have passed; returns (TFLOP/s, rows, heads, s)."""
    import numpy as np
    from oracle import dca_oracle as orc
    cfg = W.CONFIGS[name]
    if name not in _CPU_INPUTS:
        _CPU_INPUTS[name] = W.make_prefill_inputs(cfg)
    Q, K, V = _CPU_INPUTS[name]
    rng = np.random.default_rng(seed)
    flops = 0.0
    n_rows = 0
    heads = [0]
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        rows = sorted(int(x) for x in rng.integers(0, cfg["L"], size=8))
        orc.dca_prefill_rows(_F64(Q), _F64(K), _F64(V), cfg["s"], cfg["c"],
                             cfg["base"], rows=rows, heads=heads)
        flops += sum(4.0 * cfg["D"] * (i + 1) for i in rows) * len(heads)
        n_rows += len(rows)
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, n_rows, len(heads), dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle as it stands, on the host cores."""
    if rank != 0:
        return
    per_step = []
    rows_total = 0
    budget = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for k in range(args.warmup + args.steps):
        tf, n_rows, _, dt = oracle_sample(budget, seed=k)
        if k >= args.warmup:
            per_step.append((tf, dt))
            rows_total += n_rows
    value = statistics.mean(x[0] for x in per_step)
    ms = statistics.mean(x[1] for x in per_step) * 1e3
    cores = blas_threads()
    sample = (f"{rows_total} random query rows x 1 head of the {PREFILL} prefill workload, "
              f"fp64 oracle, ~{budget:.0f} s per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PREFILL, **_cfg_summary(W.CONFIGS[PREFILL])},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _cfg_summary(cfg):
    keys = ("B", "L", "Hq", "Hkv", "D", "c", "s", "Tcap")
    return {k: cfg[k] for k in keys if k in cfg}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, dev):
    import long_context_attention_dca_b200 as dca
    from long_context_attention_dca_b200 import build
    if rank == 0:
        build.build()  # (re)built once; the other ranks load it after the barrier
    _barrier(world)
    lib = dca.lib()
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    import ctypes
    P = ctypes.c_void_p

    pc = W.CONFIGS[args.workload]
    if args.override_s:  # profiling runs of the straddling-tile kernel
        pc = dict(pc, s=args.override_s)
    if args.override_d:  # profiling runs of the D = 64 instantiation
        pc = dict(pc, D=args.override_d)
    dc = W.CONFIGS[DECODE]
    Q, K, V = W.make_prefill_inputs(pc, device=dev)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    s, c, base = pc["s"], pc["c"], pc["base"]
    ws_bytes = dca.dca_attn_prefill_workspace(B, L, Hq, Hkv, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    O = torch.empty_like(Q)
    LSE = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)
    path = dca.dca_prefill_path(L, D, s, c)

    do_pre = args.only in ("all", "prefill")
    do_dec = args.only in ("all", "decode")
    if not do_dec:  # profiling run: a 1-sequence, 1k-token stand-in keeps memory small
        dc = W.scaled(dc, B=1, Tcap=1024, t_lo=1000, t_hi=1001)
    elif args.decode_seqs:
        dc = W.scaled(dc, B=args.decode_seqs)
    t_dec, q_dec, Kc, Vc = W.make_decode_inputs(dc, device=dev)
    Bd, Hqd, Dd = q_dec.shape
    Tcap, Hkvd = Kc.shape[1], Kc.shape[2]
    dws_bytes = dca.dca_attn_decode_workspace(Bd, Hqd, Dd, Tcap)
    dws = torch.empty(dws_bytes, dtype=torch.uint8, device=dev)
    Od = torch.empty_like(q_dec)
    LSEd = torch.empty(Bd, Hqd, dtype=torch.float32, device=dev)
    t_host = t_dec.cpu()

    def chk(st):
        if st != 0:
            raise dca.DcaError(st, dca.dca_last_error_string())

    def rope():
        chk(lib.dca_prefill_rope(P(Q.data_ptr()), P(K.data_ptr()), B, L, Hq, Hkv, D, s, c,
                                 base, P(ws.data_ptr()), ws_bytes, P(sptr)))

    def attn():
        chk(lib.dca_prefill_attention(P(V.data_ptr()), P(O.data_ptr()), P(LSE.data_ptr()), B, L,
                                      Hq, Hkv, D, s, c, 0.0, 0, P(ws.data_ptr()), ws_bytes,
                                      P(sptr)))

    def decode():
        chk(lib.dca_attn_decode(P(q_dec.data_ptr()), P(Kc.data_ptr()), P(Vc.data_ptr()),
                                P(t_dec.data_ptr()), P(Od.data_ptr()), P(LSEd.data_ptr()), Bd,
                                Hqd, Hkvd, Dd, Tcap, dc["s"], dc["c"], dc["base"], 0.0,
                                P(dws.data_ptr()), dws_bytes, P(sptr)))

    for _ in range(args.warmup):
        if do_pre:
            rope(); attn()
        if do_dec:
            decode()
    torch.cuda.synchronize(dev)
    dca.dca_sync_status(dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    _barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.15)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        e = ev[k]
        e[0].record(stream)
        if do_pre:
            rope()
        e[1].record(stream)
        if do_pre:
            attn()
        e[2].record(stream)
        if do_dec:
            decode()
        e[3].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    _barrier(world)
    dca.dca_sync_status(dev)

    total_ms = t_start.elapsed_time(t_end)
    rope_ms = [e[0].elapsed_time(e[1]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    dec_ms = [e[2].elapsed_time(e[3]) for e in ev]
    total_ms = _max_over_ranks(total_ms, world, dev)
    prefill_ms = _max_over_ranks(sum(rope_ms) + sum(attn_ms), world, dev)
    attn_sum = _max_over_ranks(sum(attn_ms), world, dev)
    rope_sum = _max_over_ranks(sum(rope_ms), world, dev)
    dec_sum = _max_over_ranks(sum(dec_ms), world, dev)

    flops = W.prefill_flops(pc)
    dec_bytes = W.decode_bytes(dc, t_host.tolist())
    rope_bytes = float(B * L * (Hq + Hkv) * D * 2 + B * L * (3 * Hq + Hkv) * D * 2)
    rate = lambda work, ms: work * args.steps / (ms * 1e-3) if ms > 1e-6 else 0.0
    value = world * rate(flops, prefill_ms) / 1e12
    attn_tflops = rate(flops, attn_sum) / 1e12
    dec_gbs = world * rate(dec_bytes, dec_sum) / 1e9
    rope_gbs = rate(rope_bytes, rope_sum) / 1e9

    peaks, peak_kind = load_peaks()
    traffic = load_traffic()
    tpk = peaks["bf16_tflops"]  # burst: kernels timed alone for a fraction of a second
    hbm = peaks["hbm_gbs"]
    # The step's attention kernel runs for seconds back to back inside the
    # timed region (the GPU settles at its power cap), so its roofline takes
    # the sustained bf16 figure; a short region takes the burst figure.
    long_region = total_ms > 1000.0
    tpk_step = peaks.get("bf16_tflops_sustained", tpk) if long_region else tpk
    step_peak_kind = f"{peak_kind} {'sustained' if long_region else 'burst'}"

    # ---- e2e through the public API with host buffers ----
    e2e = None if (args.no_e2e or args.only != "all") else run_e2e(dca, pc, dc, dev, args, world, Q, K, V, q_dec,
                                           t_dec, Kc, Vc)

    configs = None
    if args.configs and args.only == "all":
        configs = {name: run_config(dca, lib, name, dev, stream, world, tpk)
                   for name in SUB_CONFIGS if name != args.workload}

    next_rows = None
    select = set(args.next_rows_select.split(",")) if args.next_rows_select else None
    if args.next_rows and (args.only == "all" or select):
        nc = W.CONFIGS[NEXT_ROWS_WORKLOAD]
        if args.workload == NEXT_ROWS_WORKLOAD:
            nQ, nK, nV = Q, K, V
        else:
            nQ, nK, nV = W.make_prefill_inputs(nc, device=dev)
        next_rows = run_next_rows(dca, lib, nc, dc, dev, stream, nQ, nK, nV, t_dec, Kc, Vc,
                                  select=select)
        next_rows["workload"] = NEXT_ROWS_WORKLOAD
        del nQ, nK, nV

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            tf, n_rows, n_heads, dt = oracle_sample(args.cpu_seconds, name=args.workload)
            cpu = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                   "sample": f"{n_rows} random query rows x {n_heads} head of the {args.workload} "
                             f"prefill workload, fp64 oracle, {dt:.1f} s",
                   "rows_per_s": n_rows * n_heads / dt,
                   "extrapolated_full_prefill_s": flops / (tf * 1e12) if tf > 0 else None}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16, Llama-2 attention shapes)",
            "config": {"workload": args.workload, **_cfg_summary(pc),
                       "decode_workload": DECODE, "decode": _cfg_summary(dc),
                       "prefill_path": {1: "general (warp MMA)",
                                        2: "tcgen05/TMEM/TMA"}.get(path, str(path)),
                       "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2 (prefill Q,K,V "
                             f"{(Q.numel() + K.numel() + V.numel()) * 2 / 1e6:.0f} MB; decode "
                             f"KV {dec_bytes / 1e9:.1f} GB); no flush"},
            "prefill": {"tflops_rope_plus_attn": value / world, "attn_tflops": attn_tflops,
                        "attn_ms": attn_sum / args.steps, "rope_ms": rope_sum / args.steps,
                        "attn_ms_median": statistics.median(attn_ms),
                        "rope_ms_median": statistics.median(rope_ms),
                        "rope_gbs": rope_gbs, "frac_of_peak": attn_tflops / tpk_step,
                        "frac_of_burst_peak": attn_tflops / tpk},
            "decode": {"value": dec_gbs, "unit": "GB/s", "ms": dec_sum / args.steps,
                       "ms_median": statistics.median(dec_ms),
                       "bytes_per_step": dec_bytes, "frac_of_hbm_peak": dec_gbs / world / hbm},
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": tpk_step,
                         "unit": "TFLOP/s", "frac": attn_tflops / tpk_step,
                         "traffic": traffic.get(f"prefill_attn/{args.workload}"),
                         "kernel": "prefill attention", "peak_source": step_peak_kind,
                         "timed_region_ms": total_ms},
            "rooflines": {
                "decode_split_kv+merge": {"bound": "hbm", "achieved": dec_gbs / world,
                                          "peak": hbm, "unit": "GB/s",
                                          "frac": dec_gbs / world / hbm,
                                          "traffic": traffic.get(f"decode/{DECODE}")}
                if do_dec else None,
                "prefill_rope": {"bound": "hbm", "achieved": rope_gbs, "peak": hbm,
                                 "unit": "GB/s", "frac": rope_gbs / hbm,
                                 "traffic": traffic.get(f"prefill_rope/{args.workload}")}
                if do_pre else None},
            "e2e": e2e,
            "configs": configs,
            "next_rows": next_rows,
            "gpu_launches": (2 * do_pre + 2 * do_dec) * args.steps,
            "clocks": clocks,
            "env": _env(dev),
            "cpu_baseline": cpu,
        }
    return line


def run_config(dca, lib, name, dev, stream, world, tpk):
    """One prefill workload on its own seeded inputs: fused RoPE then DCA
    attention through the C ABI, three untimed calls, then `reps` calls timed
    with CUDA events on the launching stream (RoPE and attention separately).
    Reports device time, TFLOP/s of RoPE + attention and of the attention
    kernel alone, and the attention kernel's fraction of the bf16 peak."""
    import ctypes
    P = ctypes.c_void_p
    cfg = W.CONFIGS[name]
    Q, K, V = W.make_prefill_inputs(cfg, device=dev)
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    s, c, base = cfg["s"], cfg["c"], cfg["base"]
    wsb = dca.dca_attn_prefill_workspace(B, L, Hq, Hkv, D)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    O = torch.empty_like(Q)
    LSE = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)
    sp = P(stream.cuda_stream)

    def chk(st):
        if st != 0:
            raise dca.DcaError(st, dca.dca_last_error_string())

    def rope():
        chk(lib.dca_prefill_rope(P(Q.data_ptr()), P(K.data_ptr()), B, L, Hq, Hkv, D, s, c, base,
                                 P(ws.data_ptr()), wsb, sp))

    def attn():
        chk(lib.dca_prefill_attention(P(V.data_ptr()), P(O.data_ptr()), P(LSE.data_ptr()), B, L,
                                      Hq, Hkv, D, s, c, 0.0, 0, P(ws.data_ptr()), wsb, sp))

    flops = W.prefill_flops(cfg)
    reps = int(min(50, max(5, 0.2 / max(flops / 1e15, 1e-6))))
    for _ in range(3):
        rope(); attn()
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    _barrier(world)
    for e in ev:
        e[0].record(stream)
        rope()
        e[1].record(stream)
        attn()
        e[2].record(stream)
    torch.cuda.synchronize(dev)
    dca.dca_sync_status(dev)
    rope_ms = _max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / reps, world, dev)
    attn_ms = _max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / reps, world, dev)
    path = dca.dca_prefill_path(L, D, s, c)
    attn_tf = flops / (attn_ms * 1e-3) / 1e12
    out = {"tflops_rope_plus_attn": flops / ((rope_ms + attn_ms) * 1e-3) / 1e12,
           "attn_tflops": attn_tf, "frac_of_peak": attn_tf / tpk,
           "attn_ms": attn_ms, "rope_ms": rope_ms, "reps": reps, "flops": flops,
           **_cfg_summary(cfg), "k_boost_frac": cfg.get("k_boost_frac", 0.0),
           "attn_kernel": {1: "general (warp MMA)", 2: "tcgen05 " + (
               "two-tile" if D == 128 and s % 256 == 0 else "per-row intervals")}.get(path),
           "launches_per_call": 2}
    del Q, K, V, ws, O, LSE
    return out


def run_e2e(dca, pc, dc, dev, args, world, Q, K, V, q_dec, t_dec, Kc, Vc):
    """The step through the public API with host buffers: dca_attn_prefill_host
    reads Q, K, V from pinned host memory and writes O and LSE back (PCIe copies
    overlapped with the chunked kernels inside the call); decode copies q and t
    in and O, LSE out around dca_attn_decode (the KV cache is device-resident
    state, as in serving).  Every byte of the step's inputs crosses PCIe inside
    the timed region."""
    hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
    hO = torch.empty(Q.shape, dtype=torch.bfloat16).pin_memory()
    hL = torch.empty(Q.shape[0], Q.shape[2], Q.shape[1], dtype=torch.float32).pin_memory()
    hq, ht = q_dec.cpu().pin_memory(), t_dec.cpu().pin_memory()
    dq, dt_ = torch.empty_like(q_dec), torch.empty_like(t_dec)
    hOd = torch.empty(q_dec.shape, dtype=torch.bfloat16).pin_memory()
    hLd = torch.empty(q_dec.shape[:2], dtype=torch.float32).pin_memory()
    s, c = pc["s"], pc["c"]
    # long prompts in 8192-row chunks (2048 CTAs per chunk launch, several
    # waves of the 148 SMs), shorter ones in 2048-row chunks
    chunk = args.e2e_chunk or (8192 if pc["L"] > 32768 else 2048)
    ws = torch.empty(dca.dca_attn_prefill_host_workspace(*Q.shape[:3], K.shape[2], Q.shape[3],
                                                         chunk), dtype=torch.uint8, device=dev)
    dws = torch.empty(dca.dca_attn_decode_workspace(*q_dec.shape[:2], q_dec.shape[2],
                                                    Kc.shape[1]), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        dca.dca_attn_prefill_host(hQ, hK, hV, s, c, pc["base"], chunk_rows=chunk, workspace=ws,
                                  O=hO, LSE=hL, device=dev)
        dq.copy_(hq, non_blocking=True); dt_.copy_(ht, non_blocking=True)
        Od, LSEd = dca.dca_attn_decode(dq, Kc, Vc, dt_, dc["s"], dc["c"], dc["base"],
                                       workspace=dws)
        hOd.copy_(Od, non_blocking=True); hLd.copy_(LSEd, non_blocking=True)

    n = max(1, min(args.steps, 10))
    for _ in range(2):
        step()
    torch.cuda.synchronize(dev)
    _barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    dca.dca_sync_status(dev)
    ms = _max_over_ranks(a.elapsed_time(b), world, dev) / n
    flops = W.prefill_flops(pc)
    h2d = sum(x.numel() * x.element_size() for x in (hQ, hK, hV, hq, ht))
    d2h = sum(x.numel() * x.element_size() for x in (hO, hL, hOd, hLd))
    return {"value": world * flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "api": f"dca_attn_prefill_host (chunks of {chunk} rows, copies overlapped) + "
                   "dca_attn_decode (decode KV cache device-resident)"}


def run_next_rows(dca, lib, pc, dc, dev, stream, Q, K, V, t_dec, Kc, Vc, reps=3, select=None):
    """Device time of the calls beyond the step, each on the launching stream
    with CUDA events, after one untimed call:
      prefill_chunk  the prefill workload as four equal chunks against a cache
                     (dca_attn_prefill_chunk, chunk starts 0, L/4, L/2, 3L/4);
      prefill_general_path  the attention of the prefill workload forced onto
                     the general warp-MMA kernel (dca_prefill_attention);
      prefill_unaligned_s  the prefill workload's attention with s = 3000 (tiles
                     straddle chunk boundaries; dca_prefill_attention, auto path);
      prefill_3pass  the prefill workload as three single-piece passes merged
                     by LSE (dca_attn_prefill_3pass);
      prefill_selfextend  the prefill workload under the SelfExtend position
                     map, G = 8, W = 1024 (dca_attn_prefill_selfextend);
      prefill_varlen a packed batch of eight Llama-2 7B prompts of mixed length
                     (dca_attn_prefill_varlen, RoPE included);
      prefill_varlen_chunk  the next chunks (256 .. 2048 tokens) of eight
                     sequences with 0 .. 14000 cached tokens, packed
                     (dca_attn_prefill_varlen_chunk), and the same batch with
                     the caller's fp16 key mirror
                     (dca_attn_prefill_varlen_chunk_mirror);
      decode_paged   the decode workload over a paged copy of its caches
                     (dca_attn_decode_paged, 256-row blocks in random order);
      kv_append      one decoded token appended per sequence of the decode
                     batch (dca_kv_append), 100 calls back to back."""
    import ctypes
    import numpy as np
    P = ctypes.c_void_p
    B, L, Hq, D = Q.shape
    Hkv = K.shape[2]
    s, c, base = pc["s"], pc["c"], pc["base"]
    flops = W.prefill_flops(pc)
    out = {}

    def want(name):
        return select is None or name in select

    def timed(fn, n=reps):
        fn()
        torch.cuda.synchronize(dev)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        dca.dca_sync_status(dev)
        return a.elapsed_time(b) / n

    # chunked prefill
    if want("prefill_chunk"):
        n_chunks = 4
        bounds = [L * k // n_chunks for k in range(n_chunks + 1)]
        Kcache = torch.empty(B, L, Hkv, D, dtype=torch.bfloat16, device=dev)
        Vcache = torch.empty_like(Kcache)
        Qs = [Q[:, a:e].contiguous() for a, e in zip(bounds[:-1], bounds[1:])]
        Ks = [K[:, a:e].contiguous() for a, e in zip(bounds[:-1], bounds[1:])]
        Vs = [V[:, a:e].contiguous() for a, e in zip(bounds[:-1], bounds[1:])]
        wsz = max(dca.dca_attn_prefill_chunk_workspace(B, e - a, Hq, Hkv, D, a)
                  for a, e in zip(bounds[:-1], bounds[1:]))
        cws = torch.empty(wsz, dtype=torch.uint8, device=dev)
        Oc = torch.empty_like(Q)
        Lc = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)
        Ob = [torch.empty_like(q) for q in Qs]
        Lb = [torch.empty(B, Hq, q.shape[1], dtype=torch.float32, device=dev) for q in Qs]

        def chunks():
            for k, (a, e) in enumerate(zip(bounds[:-1], bounds[1:])):
                st = lib.dca_attn_prefill_chunk(
                    P(Qs[k].data_ptr()), P(Ks[k].data_ptr()), P(Vs[k].data_ptr()),
                    P(Kcache.data_ptr()), P(Vcache.data_ptr()), P(Ob[k].data_ptr()),
                    P(Lb[k].data_ptr()), B, e - a, Hq, Hkv, D, a, L, s, c, base, 0.0,
                    P(cws.data_ptr()), wsz, P(stream.cuda_stream))
                if st != 0:
                    raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(chunks)
        tc = all(a % 256 == 0 for a in bounds[:-1]) and s % 256 == 0 and D == 128
        out["prefill_chunk"] = {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                                "ms": ms, "chunks": n_chunks,
                                "path": "tcgen05/TMEM/TMA" if tc else "general (warp MMA)",
                                "launches_per_call": 3 if tc else 2}
        del Kcache, Vcache, cws, Oc, Lc, Ob, Lb, Qs, Ks, Vs

    # the general (warp-MMA) kernel on the same workload: the path of every
    # chunking the tcgen05 kernels do not cover (straddling tiles, per-element
    # piece selection)
    if want("prefill_general_path") or want("prefill_unaligned_s"):
        gws = dca.dca_attn_prefill_workspace(B, L, Hq, Hkv, D)
        gbuf = torch.empty(gws, dtype=torch.uint8, device=dev)
        Og = torch.empty_like(Q)
        Lg = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)
        st = lib.dca_prefill_rope(P(Q.data_ptr()), P(K.data_ptr()), B, L, Hq, Hkv, D, s, c, base,
                                  P(gbuf.data_ptr()), gws, P(stream.cuda_stream))
        if st != 0:
            raise dca.DcaError(st, dca.dca_last_error_string())

        def general():
            st = lib.dca_prefill_attention(P(V.data_ptr()), P(Og.data_ptr()), P(Lg.data_ptr()), B, L,
                                           Hq, Hkv, D, s, c, 0.0, dca.DCA_PATH_GENERAL,
                                           P(gbuf.data_ptr()), gws, P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(general)
        out["prefill_general_path"] = {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                                       "ms": ms, "path": "general (warp MMA), attention only",
                                       "launches_per_call": 1}

        # a chunk size that is not a multiple of the 128-row tiles (s = 3000):
        # tiles straddle chunk boundaries, the per-row-interval tcgen05 kernel
        s_u = 3000
        st = lib.dca_prefill_rope(P(Q.data_ptr()), P(K.data_ptr()), B, L, Hq, Hkv, D, s_u, c, base,
                                  P(gbuf.data_ptr()), gws, P(stream.cuda_stream))
        if st != 0:
            raise dca.DcaError(st, dca.dca_last_error_string())

        def unaligned():
            st = lib.dca_prefill_attention(P(V.data_ptr()), P(Og.data_ptr()), P(Lg.data_ptr()), B, L,
                                           Hq, Hkv, D, s_u, c, 0.0, dca.DCA_PATH_AUTO,
                                           P(gbuf.data_ptr()), gws, P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(unaligned)
        out["prefill_unaligned_s"] = {
            "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms": ms, "s": s_u, "c": c,
            "path": {1: "general (warp MMA)", 2: "tcgen05 per-row intervals"}.get(
                dca.dca_prefill_path(L, D, s_u, c)), "launches_per_call": 1}
        del gbuf, Og, Lg

    # three passes + LSE merge
    if want("prefill_3pass"):
        wsz = dca.dca_attn_prefill_3pass_workspace(B, L, Hq, Hkv, D)
        pws = torch.empty(wsz, dtype=torch.uint8, device=dev)
        O3 = torch.empty_like(Q)
        L3 = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)

        def three():
            st = lib.dca_attn_prefill_3pass(P(Q.data_ptr()), P(K.data_ptr()), P(V.data_ptr()),
                                            P(O3.data_ptr()), P(L3.data_ptr()), B, L, Hq, Hkv, D, s,
                                            c, base, 0.0, P(pws.data_ptr()), wsz,
                                            P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(three)
        out["prefill_3pass"] = {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms": ms,
                                "path": "general (warp MMA) x3 + merge", "launches_per_call": 5}
        del pws, O3, L3

    # SelfExtend position map on the general kernel (group 8, window 1024)
    if want("prefill_selfextend"):
        G_se, W_se = 8, 1024
        wsz = dca.dca_selfextend_workspace(B, L, Hq, Hkv, D)
        sws = torch.empty(wsz, dtype=torch.uint8, device=dev)
        Ose = torch.empty_like(Q)
        Lse = torch.empty(B, Hq, L, dtype=torch.float32, device=dev)

        def selfextend():
            st = lib.dca_attn_prefill_selfextend(P(Q.data_ptr()), P(K.data_ptr()), P(V.data_ptr()),
                                                 P(Ose.data_ptr()), P(Lse.data_ptr()), B, L, Hq, Hkv,
                                                 D, G_se, W_se, base, 0.0, P(sws.data_ptr()), wsz,
                                                 P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(selfextend)
        out["prefill_selfextend"] = {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                                     "ms": ms, "G": G_se, "W": W_se,
                                     "path": "RoPE (2 planes) + tcgen05 per-row intervals",
                                     "launches_per_call": 2}
        del sws, Ose, Lse

    # packed variable-length batch: Llama-2 7B heads, eight prompts of seeded
    # lengths in [512, 16384] back to back (RoPE + attention in one call)
    vc = W.CONFIGS["varlen_7b_mix"]
    Hqv, Hkvv, Dv = vc["Hq"], vc["Hkv"], vc["D"]
    if want("prefill_varlen"):
        Qv, Kv, Vv, cu, lens = W.make_varlen_inputs(vc, device=dev)
        cu_d = cu.to(dev)
        Tv = Qv.shape[0]
        wsz = dca.dca_attn_prefill_varlen_workspace(Tv, Hqv, Hkvv, Dv)
        vws = torch.empty(wsz, dtype=torch.uint8, device=dev)
        Ov = torch.empty_like(Qv)
        Lv = torch.empty(Hqv, Tv, dtype=torch.float32, device=dev)

        def varlen():
            st = lib.dca_attn_prefill_varlen(P(Qv.data_ptr()), P(Kv.data_ptr()), P(Vv.data_ptr()),
                                             P(Ov.data_ptr()), P(Lv.data_ptr()), P(cu_d.data_ptr()),
                                             len(lens), max(lens), Tv, Hqv, Hkvv, Dv, vc["s"],
                                             vc["c"], vc["base"], 0.0, P(vws.data_ptr()), wsz,
                                             P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(varlen)
        out["prefill_varlen"] = {
            "value": W.varlen_flops(lens, Hqv, Dv) / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms": ms, "workload": "varlen_7b_mix", "lens": lens, "T": Tv,
            "path": "RoPE + tcgen05 " + ("two-tile" if Dv == 128 and vc["s"] % 256 == 0
                                         else "per-row intervals"),
            "launches_per_call": 2}
        del Qv, Kv, Vv, vws, Ov, Lv

    # packed chunks over per-sequence caches: Llama-2 7B heads, eight
    # sequences with seeded 0 .. 14000 cached tokens and new chunks of
    # 256 .. 2048 tokens (RoPE, cache writes, key conversion and attention)
    if want("prefill_varlen_chunk"):
        rng = np.random.default_rng(7)
        t0c = [int(x) for x in rng.integers(0, 14001, 8)]
        lensc = [int(x) for x in rng.integers(256, 2049, 8)]
        Tc, Tcap_c = sum(lensc), 16384
        gen_c = torch.Generator(device=dev)
        gen_c.manual_seed(7)
        Qc = torch.randn(Tc, Hqv, Dv, generator=gen_c, device=dev).to(torch.bfloat16)
        Kn = torch.randn(Tc, Hkvv, Dv, generator=gen_c, device=dev).to(torch.bfloat16)
        Vn = torch.randn(Tc, Hkvv, Dv, generator=gen_c, device=dev).to(torch.bfloat16)
        Kcc = torch.randn(8, Tcap_c, Hkvv, Dv, generator=gen_c, device=dev).to(torch.bfloat16)
        Vcc = torch.randn(8, Tcap_c, Hkvv, Dv, generator=gen_c, device=dev).to(torch.bfloat16)
        cu_c = torch.zeros(9, dtype=torch.int32)
        cu_c[1:] = torch.cumsum(torch.tensor(lensc), 0).to(torch.int32)
        cu_c, t0_d = cu_c.to(dev), torch.tensor(t0c, dtype=torch.int32, device=dev)
        max_kv = max(a + n for a, n in zip(t0c, lensc))
        wsz = dca.dca_attn_prefill_varlen_chunk_workspace(8, Tc, max_kv, Hqv, Hkvv, Dv)
        cws = torch.empty(wsz, dtype=torch.uint8, device=dev)
        Occ = torch.empty_like(Qc)
        Lcc = torch.empty(Hqv, Tc, dtype=torch.float32, device=dev)

        def varlen_chunk():
            st = lib.dca_attn_prefill_varlen_chunk(
                P(Qc.data_ptr()), P(Kn.data_ptr()), P(Vn.data_ptr()), P(Kcc.data_ptr()),
                P(Vcc.data_ptr()), P(Occ.data_ptr()), P(Lcc.data_ptr()), P(cu_c.data_ptr()),
                P(t0_d.data_ptr()), 8, max(lensc), Tc, max_kv, Hqv, Hkvv, Dv, Tcap_c, vc["s"],
                vc["c"], vc["base"], 0.0, P(cws.data_ptr()), wsz, P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(varlen_chunk)
        out["prefill_varlen_chunk"] = {
            "value": W.varlen_chunk_flops(t0c, lensc, Hqv, Dv) / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s", "ms": ms, "t0": t0c, "lens": lensc,
            "path": "chunk RoPE + key conversion + work order + tcgen05 per-row intervals",
            "launches_per_call": 4}
        # the same batch with the caller's fp16 key mirror: the cached prefix
        # is read as kept from earlier calls instead of converted again (the
        # mirror is filled once here, outside the timing)
        Kf = Kcc.to(torch.float16)
        wsm = dca.dca_attn_prefill_varlen_chunk_mirror_workspace(8, Tc, Hqv, Hkvv, Dv)
        mws = torch.empty(wsm, dtype=torch.uint8, device=dev)

        def varlen_chunk_mirror():
            st = lib.dca_attn_prefill_varlen_chunk_mirror(
                P(Qc.data_ptr()), P(Kn.data_ptr()), P(Vn.data_ptr()), P(Kcc.data_ptr()),
                P(Vcc.data_ptr()), P(Kf.data_ptr()), P(Occ.data_ptr()), P(Lcc.data_ptr()),
                P(cu_c.data_ptr()), P(t0_d.data_ptr()), 8, max(lensc), Tc, max_kv, Hqv, Hkvv, Dv,
                Tcap_c, vc["s"], vc["c"], vc["base"], 0.0, P(mws.data_ptr()), wsm,
                P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(varlen_chunk_mirror)
        out["prefill_varlen_chunk_mirror"] = {
            "value": W.varlen_chunk_flops(t0c, lensc, Hqv, Dv) / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s", "ms": ms, "t0": t0c, "lens": lensc,
            "path": "chunk RoPE (fp16 keys to the caller's mirror) + value tail + tcgen05 "
                    "per-row intervals",
            "launches_per_call": 4}
        del Qc, Kn, Vn, Kcc, Vcc, cws, Occ, Lcc, Kf, mws

    # decode over a paged cache: the decode workload's caches scattered into
    # 256-row blocks in a seeded random physical order
    if want("decode_paged"):
        Bd, Tcap, Hkvd, Dd = Kc.shape
        rows = 256
        nb = Tcap // rows
        gperm = torch.Generator().manual_seed(0)
        perm = torch.randperm(Bd * nb, generator=gperm).to(dev)
        Kp = torch.empty(Bd * nb, rows, Hkvd, Dd, dtype=Kc.dtype, device=dev)
        Vp = torch.empty_like(Kp)
        Kp[perm] = Kc.view(Bd * nb, rows, Hkvd, Dd)
        Vp[perm] = Vc.view(Bd * nb, rows, Hkvd, Dd)
        table = perm.view(Bd, nb).to(torch.int32)
        qd = torch.randn(Bd, dc["Hq"], Dd, device=dev).to(torch.bfloat16)
        pws = torch.empty(dca.dca_attn_decode_workspace(Bd, dc["Hq"], Dd, Tcap), dtype=torch.uint8,
                          device=dev)
        Opg = torch.empty_like(qd)
        Lpg = torch.empty(Bd, dc["Hq"], dtype=torch.float32, device=dev)

        def paged():
            st = lib.dca_attn_decode_paged(P(qd.data_ptr()), P(Kp.data_ptr()), P(Vp.data_ptr()),
                                           P(table.data_ptr()), nb, rows, Bd * nb,
                                           P(t_dec.data_ptr()), P(Opg.data_ptr()), P(Lpg.data_ptr()),
                                           Bd, dc["Hq"], Hkvd, Dd, dc["s"], dc["c"], dc["base"], 0.0,
                                           P(pws.data_ptr()), pws.numel(), P(stream.cuda_stream))
            if st != 0:
                raise dca.DcaError(st, dca.dca_last_error_string())
        ms = timed(paged, 10)
        dbytes = W.decode_bytes(dc, t_dec.cpu().tolist())
        out["decode_paged"] = {"value": dbytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms": ms,
                               "block_rows": rows, "launches_per_call": 2}
        del Kp, Vp, pws

    # decode-time append of one token per sequence (positions t_dec + 1 < Tcap)
    if want("kv_append"):
        Bd, Tcap, Hkvd, Dd = Kc.shape
        kn = torch.randn(Bd, Hkvd, Dd, device=dev).to(torch.bfloat16)
        vn = torch.randn(Bd, Hkvd, Dd, device=dev).to(torch.bfloat16)
        t_app = torch.clamp(t_dec + 1, max=Tcap - 1).to(torch.int32)
        Kc2, Vc2 = Kc.clone(), Vc.clone()  # the step's caches stay as they are

        def append(strm):
            for _ in range(100):
                st = lib.dca_kv_append(P(kn.data_ptr()), P(vn.data_ptr()), P(Kc2.data_ptr()),
                                       P(Vc2.data_ptr()), P(t_app.data_ptr()), Bd, Hkvd, Dd, Tcap,
                                       dc["s"], dc["c"], dc["base"], P(strm.cuda_stream))
                if st != 0:
                    raise dca.DcaError(st, dca.dca_last_error_string())
        ms_stream = timed(lambda: append(stream), 1) / 100
        # the same 100 appends replayed from a CUDA graph (no host launch overhead)
        side = torch.cuda.Stream(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            append(side)
        ms_graph = timed(graph.replay, 1) / 100
        del graph
        nbytes = Bd * Hkvd * Dd * 2 * 4  # read k, v; write the two cache rows
        out["kv_append"] = {"us_per_call": ms_graph * 1e3, "us_per_call_stream": ms_stream * 1e3,
                            "bytes_per_call": nbytes, "timing": "100 appends in a CUDA graph",
                            "bound": "launch latency (a few hundred KB per call)",
                            "launches_per_call": 1}
        del Kc2, Vc2
    return out


def _env(dev):
    """GPU, driver and host-core facts of the run."""
    drv = None
    try:
        out = subprocess.run(["nvidia-smi", "--query-gpu=driver_version", "--format=csv,noheader",
                              "-i", str(dev.index or 0)], capture_output=True, text=True,
                             timeout=20)
        drv = out.stdout.strip() or None
    except (OSError, subprocess.SubprocessError):
        pass
    return {"gpu": torch.cuda.get_device_name(dev), "driver": drv,
            "torch_cuda": torch.version.cuda, "torch": torch.__version__,
            "host_cores": os.cpu_count(), "affinity_cores": len(os.sched_getaffinity(0))}


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _max_over_ranks(x, world, dev):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--decode-seqs", type=int, default=0,
                    help="profiling runs: decode this many sequences instead of 16")
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                    help="profiling runs: time only one half of the step")
    ap.add_argument("--next-rows", action=argparse.BooleanOptionalAction, default=True,
                    help="also time chunked prefill, the 3-pass variant and KV append "
                         "(outside the timed step)")
    ap.add_argument("--next-rows-select", default="",
                    help="profiling runs: comma-separated names of the calls beyond the step "
                         "to time (e.g. prefill_varlen_chunk); runs them with --only prefill too")
    ap.add_argument("--override-s", type=int, default=0,
                    help="profiling runs: chunk size s of the prefill workload (e.g. 3000, "
                         "whose tiles straddle chunk boundaries)")
    ap.add_argument("--override-d", type=int, default=0, choices=[0, 64, 128],
                    help="profiling runs: head dim of the prefill workload (64 runs the "
                         "interval kernel's D = 64 instantiation)")
    ap.add_argument("--e2e-chunk", type=int, default=0,
                    help="rows per chunk of the host-buffer prefill in the e2e leg "
                         "(0: 8192 above 32k tokens, else 2048)")
    ap.add_argument("--configs", action=argparse.BooleanOptionalAction, default=True,
                    help="also time the other prefill workloads (70B-, 7B-shaped, tiny)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (profiling runs)")
    ap.add_argument("--workload", default=PREFILL, choices=sorted(
        k for k, v in W.CONFIGS.items() if v["kind"] == "prefill" and v["D"] == 128),
                    help="prefill workload of the step (default: the 100k-token one)")
    ap.add_argument("--dry-run", action="store_true",
                    help="launcher and rank plumbing only: gloo process group, barrier and "
                         "max over ranks, no GPU work (checks --gpus on a CPU host)")
    ap.add_argument("--launch-timeout", type=float, default=3600.0,
                    help="seconds before a self-launched multi-rank run is stopped")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    plan, detail = launch_plan(args.gpus, os.environ)
    if plan == "error":
        print(f"bench.py: {detail}", file=sys.stderr, flush=True)
        sys.exit(2)
    if plan == "spawn":
        sys.exit(spawn_ranks(args.gpus, args.launch_timeout))

    world = detail
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, rank, world)
        return

    if args.dry_run:
        run_dry(args, rank, world)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    try:
        line = run_ours(args, rank, world, dev)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


def launch_plan(gpus: int, env) -> tuple:
    """How this process takes part in a run of `gpus` ranks.

    ("run", world) when it is one of the ranks (no WORLD_SIZE: a single rank;
    under torchrun WORLD_SIZE must equal --gpus), ("spawn", None) when --gpus
    asks for more than one rank and no launcher started this process, and
    ("error", why) on a mismatch, which must not silently run fewer ranks.
    """
    if gpus < 1:
        return "error", f"--gpus must be >= 1, got {gpus}"
    ws = env.get("WORLD_SIZE")
    if ws is None:
        return ("spawn", None) if gpus > 1 else ("run", 1)
    if int(ws) != gpus:
        return "error", (f"WORLD_SIZE={ws} (launcher) but --gpus {gpus}: start "
                         f"{gpus} ranks or pass --gpus {ws}")
    return "run", int(ws)


def spawn_ranks(gpus: int, timeout_s: float) -> int:
    """Start `gpus` local ranks of this script through torch.distributed.run
    (rendezvous on 127.0.0.1) and return the launcher's exit code; the whole
    process group is stopped if it runs past `timeout_s`."""
    import signal
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", "--master-port",
           str(port), os.path.abspath(__file__), *sys.argv[1:]]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=timeout_s)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGTERM)
        try:
            proc.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(proc.pid, signal.SIGKILL)
            proc.wait()
        print(f"bench.py: {gpus}-rank run stopped after {timeout_s:.0f} s", file=sys.stderr)
        return 124


def run_dry(args, rank, world):
    """The rank plumbing of a run without GPU work: a gloo process group, the
    barrier around the timed region and the max over ranks of a per-rank
    time; rank 0 prints one JSON line naming the ranks that took part."""
    import datetime
    if world > 1:
        torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        _barrier(world)
        slowest = _max_over_ranks(float(rank + 1), world, cpu)
        ranks = [rank]
        if world > 1:
            got = [None] * world
            torch.distributed.all_gather_object(got, rank)
            ranks = got
        _barrier(world)
        if rank == 0:
            print(json.dumps({"dry_run": True, "n_gpus": world, "ranks": ranks,
                              "max_over_ranks": slowest, "steps": args.steps,
                              "warmup": args.warmup}), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
