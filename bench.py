"""Benchmark of the RRS W4A4 linear layer (prep + GEMM) on B200.

A step is one RRS linear (online rotation/reorder/group max/quantise, then
the group-scaled W4A4 GEMM) on each LLaMA-3-8B projection shape the headline
metric is quoted on: M=2048 tokens, K=4096, N in {4096 (q/o), 1024 (k/v),
14336 (gate/up)}, G=128, Hadamard 4096.  Inputs are synthetic (seeded,
outlier-laden); weights are prepared once, off the timed path, and held as
their INT4 codes one per byte in e4m3 form (the operand of the fp8 tensor-core
GEMM); the same step with the weights packed two codes per byte is reported
beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  With N > 1 it runs one process per GPU (under
torchrun, or relaunching itself under torch.distributed.run): every rank runs
its own replica (independent batches: replicas only); the time is the max over
ranks and the value the operations of all ranks over that time.
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

METRIC = "RRS W4A4 linear TOPS (prep+GEMM) at LLaMA-3-8B shapes; % of INT8 TC peak"
UNIT = "TOPS"
N_XSETS = 4            # distinct activation buffers per layer, rotated between steps
GEMM_SOURCE = os.path.join(ROOT, "activation_smoothing_b200", "csrc", "rrs_gemm_f8.cu")
GEMM_PROFILE = os.path.join(ROOT, "profiles", "gemm_f8_llama3_8b.md")


def gemm_traffic_bytes():
    """DRAM bytes (read + write) per GEMM launch, mean over the step's layers, from the
    ncu capture summarised in the profile file, or None when the GEMM source has changed
    since that capture (the summary records the source's sha256)."""
    import hashlib
    import re
    try:
        src = hashlib.sha256(open(GEMM_SOURCE, "rb").read()).hexdigest()
        txt = open(GEMM_PROFILE).read()
    except OSError:
        return None, "no capture summary"
    m_sha = re.search(r"source sha256: ([0-9a-f]{64})", txt)
    m_b = re.search(r"dram bytes per launch, mean of the step's layers: ([0-9.]+)", txt)
    if not (m_sha and m_b):
        return None, "capture summary lacks the source hash or the traffic figure"
    if m_sha.group(1) != src:
        return None, "GEMM source changed since the capture"
    return float(m_b.group(1)), "ncu dram__bytes_read.sum + dram__bytes_write.sum, mean of the 3 layers' launches"


def peaks():
    """(int8 dense TOPS, HBM GB/s, source).  INT8 = 2 x the measured bf16 figure
    (nominal ratio 4.5 / 2.25 PFLOP/s)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return 2.0 * float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    except Exception:
        return 2.0 * 1590.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def max_over_ranks(x: float, pg, device) -> float:
    """The largest of every rank's x (all ranks get it); x itself with no process group."""
    if pg is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(ops_per_step: int, steps: int, world: int, ms: float) -> float:
    """Operations of all ranks (each runs its own replica) over the slowest rank's time, in TOPS."""
    return ops_per_step * steps * world / (ms * 1e-3) / 1e12


def activation_sample(i: int, rank: int) -> int:
    """Seed offset of the i-th activation set of a rank: replicas never share a batch."""
    return 2 + i + 10 * rank


def bench_config(names, layers, world: int) -> dict:
    """The workload description both arms print."""
    return {"workload": "+".join(names),
            "shapes": [dict(M=L.M, K=L.K, N=L.N, G=L.G, had=L.had_block) for L in layers],
            "parallelism": f"replicas{world}",
            "l2": f"activations rotate over {N_XSETS} sets per layer; per-step footprint exceeds L2"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def relaunch(n: int) -> int:
    """Runs this same command as n processes, one per GPU (torch.distributed.run on
    127.0.0.1, a free port); returns its exit status."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def run_ours(args):
    import datetime

    import activation_smoothing_b200 as rrs
    from activation_smoothing_b200 import workloads as wl

    world, rank, local = dist_setup()
    if world != args.gpus:
        raise SystemExit(f"bench: --gpus {args.gpus} but {world} process(es) are running")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    names = args.workload.split(",") if args.workload else wl.HEADLINE
    layers = [wl.LAYERS[n] for n in names]
    state = []
    for L in layers:
        # calibration draw -> reorder index, on the device (product path)
        Xc = wl.make_activations(L, sample=1, M=min(L.M, 512)).to(dev)
        perm = rrs.calibrate_perm(Xc, L.had_block)
        W = wl.make_weights(L).to(dev)
        qW, sw = rrs.prepare_weights(W, perm, L.had_block)
        qW8 = rrs.expand_weights(qW)          # the codes one per byte (e4m3): the fp8 GEMM's operand
        del W
        xs = [wl.make_activations(L, sample=activation_sample(i, rank)).to(dev) for i in range(N_XSETS)]
        st = dict(L=L, perm=perm, qW=qW, qW8=qW8, sw=sw, xs=xs,
                  qX=torch.empty((L.M, L.K // 2), dtype=torch.uint8, device=dev),
                  s=torch.empty(L.K // L.G, dtype=torch.float32, device=dev),
                  st=torch.empty(L.M, dtype=torch.float32, device=dev),
                  Y=torch.empty((L.M, L.N), dtype=torch.float32, device=dev),
                  ws=rrs.make_workspace(L.M, L.N, L.K, L.G, L.had_block, device=dev))
        state.append(st)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    HEAD = rrs.W_EXPANDED            # headline: fp8 operands (weights expanded offline)

    def step(i, flags, events=None):
        for j, st in enumerate(state):
            L = st["L"]
            X = st["xs"][i % N_XSETS]
            qw = st["qW8"] if flags & rrs.W_EXPANDED else st["qW"]
            if events is not None:
                events[j][0].record(stream)
            rrs.smooth_quant(X, st["perm"], L.G, L.had_block, flags=flags & rrs.W_EXPANDED, qX=st["qX"], s=st["s"],
                             scale_t=st["st"], ws=st["ws"])
            if events is not None:
                events[j][1].record(stream)
            rrs.w4a4_gemm(st["qX"], st["s"], st["st"], qw, st["sw"], L.G, Y=st["Y"], ws=st["ws"],
                          flags=rrs.WS_HOLDS_A8 | flags)
            if events is not None:
                events[j][2].record(stream)

    # Per-kernel CUDA events go on every EV_EVERY-th step of the timed region (an event
    # between two kernels costs ~3 us of GPU time; the other steps run back to back).
    EV_EVERY = 10

    def timed(K, flags, with_events):
        for i in range(args.warmup):
            step(i, flags)
        for st in state:
            rrs.check_workspace(st["ws"])
        torch.cuda.synchronize()
        evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in state]
               if i % EV_EVERY == 0 else None for i in range(K)] if with_events else None
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(K):
            step(i, flags, evs[i] if evs else None)
        t1.record(stream)
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        ms = max_over_ranks(t0.elapsed_time(t1), pg, dev)
        for st in state:
            rrs.check_workspace(st["ws"])
        return ms, evs

    K = args.steps
    with ClockSampler(local) as clk:
        ms, evs = timed(K, HEAD, True)
    sampled = [i for i in range(K) if evs[i] is not None]
    prep_ms = [sum(evs[i][j][0].elapsed_time(evs[i][j][1]) for i in sampled) / len(sampled) for j in range(len(state))]
    gemm_ms = [sum(evs[i][j][1].elapsed_time(evs[i][j][2]) for i in sampled) / len(sampled) for j in range(len(state))]
    ops_step = sum(st["L"].ops for st in state)
    value = whole_job_tops(ops_step, K, world, ms)

    # ---- the same step with the weights packed two codes per byte (INT8 tensor-core
    # kernel that unpacks them on chip); same codes, same results
    Kp = max(3, min(K, 500))
    pms, pevs = timed(Kp, 0, True)
    packed = {"value": round(whole_job_tops(ops_step, Kp, world, pms), 2), "unit": UNIT, "steps": Kp,
              "gemm_ms_per_layer": [round(sum(pevs[i][j][1].elapsed_time(pevs[i][j][2]) for i in range(Kp)
                                              if pevs[i] is not None) / len([e for e in pevs if e is not None]), 5)
                                    for j in range(len(state))],
              "weights": "INT4 codes packed two per byte (N*K/2 bytes); int8 tensor-core GEMM"}

    # ---- the gated MLP block at LLaMA-3-8B sizes on the same path (timed apart from the step)
    mlp = None if args.no_mlp else mlp_block_times(rrs, wl, dev, stream, args.warmup, max(3, min(K, 200)), pg)

    # ---- decode (70B q/o, one token; the single-launch layer) and the INT4 KV cache
    extra = {} if args.no_mlp else extra_rows(rrs, wl, dev, pg)

    # ---- end to end through the C ABI with host buffers (pinned), copies timed.
    e2e = None
    if not args.no_e2e:
        hx = [st["xs"][0].cpu().pin_memory() for st in state]
        hy = [torch.empty((st["L"].M, st["L"].N), dtype=torch.float32).pin_memory() for st in state]
        Ke = max(3, min(K, 50))

        def e2e_step():
            for j, st in enumerate(state):
                L = st["L"]
                rrs.linear_from_host(hx[j], st["xs"][1], st["qW8"], st["sw"], st["perm"], L.G, L.had_block,
                                     st["qX"], st["s"], st["st"], st["Y"], hy[j], st["ws"], flags=HEAD)
        for _ in range(3):
            e2e_step()
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(Ke):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(a.elapsed_time(b), pg, dev)
        e2e = {"value": whole_job_tops(ops_step, Ke, world, ems), "unit": UNIT,
               "h2d_bytes_per_step": sum(st["L"].M * st["L"].K * 2 for st in state),
               "d2h_bytes_per_step": sum(st["L"].M * st["L"].N * 4 for st in state),
               "steps": Ke, "call": "rrs_linear_from_host (RRS_W_EXPANDED)"}

    int8_peak, hbm_peak, src = peaks()
    gemm_tops = ops_step / (sum(gemm_ms) * 1e-3) / 1e12
    prep_bytes = [2 * st["L"].M * st["L"].K + st["L"].M * st["L"].K // 2 + 4 * st["L"].M + 4 * (st["L"].K // st["L"].G)
                  for st in state]
    prep_gbs = sum(prep_bytes) / (sum(prep_ms) * 1e-3) / 1e9
    launches_per_step = 2 * len(state)      # activation kernel + GEMM per layer
    traffic, traffic_note = gemm_traffic_bytes()

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8 (e4m3) MMA on INT4 codes, fp32 accumulate / fp32 prep",
        "data": "synthetic (seeded outlier-laden activations, N(0,0.02) weights); INT4 weight codes held one per "
                "byte (e4m3) for the fp8 GEMM",
        "config": bench_config(names, layers, world),
        "roofline": {"bound": "tensor", "achieved": round(gemm_tops, 1), "peak": round(int8_peak, 1),
                     "unit": "TOPS", "frac": round(gemm_tops / int8_peak, 4), "traffic": traffic,
                     "kernel": "rrs gemm_f8 (tcgen05.mma kind::f8f6f4; CTA-pair 256x256 tiles for q/o and gate/up)",
                     "peak_source": src + " (2 x bf16 burst = the nominal dense fp8/int8 rate)",
                     "traffic_note": traffic_note,
                     "kernel_timing": f"CUDA events around each kernel on every {EV_EVERY}th of the {K} timed steps "
                                      f"({len(sampled)} steps)"},
        "prep": {"ms_per_layer": [round(x, 5) for x in prep_ms], "algorithmic_GBps": round(prep_gbs, 1),
                 "hbm_frac": round(prep_gbs / hbm_peak, 4)},
        "gemm": {"ms_per_layer": [round(x, 5) for x in gemm_ms], "TOPS": round(gemm_tops, 1)},
        "e2e": e2e,
        "packed_weights": packed,
        "mlp_block": mlp,
        **extra,
        "gpu_launches": launches_per_step * K,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(layers, budget_s=args.cpu_budget)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def extra_rows(rrs, wl, dev, pg):
    """Two more rows measured in the same run, apart from the step: the single-launch
    layer for one decode token (70B q/o, weights rotated past L2) and the INT4 KV cache
    of a batch (quantise and dequantise), each against the HBM peak."""
    _, hbm_peak, _ = peaks()
    L = wl.LAYERS["llama3_70b_qo_decode_m1"]
    dec = decode_entry(rrs, wl, dev, L, wl.make_activations(L).to(dev), wl.make_weights(L).to(dev), hbm_peak)
    torch.cuda.empty_cache()
    # KV cache of LLaMA-3-70B (8 KV heads of 128) for 16 sequences of 4096 tokens
    T, H, D = 65536, 8, 128
    g = torch.Generator().manual_seed(404)
    kv = (torch.randn(T, H, D, generator=g) * 2.0)
    kv[:, :, 5] *= 40.0
    kv = kv.to(torch.float16).to(dev)
    q = torch.empty((T, H, D // 2), dtype=torch.uint8, device=dev)
    sc = torch.empty((T, H), dtype=torch.float32, device=dev)
    out = torch.empty_like(kv)
    tq = _time_ms(lambda: rrs.kv_quant(kv, q=q, scale=sc), 10)
    td = _time_ms(lambda: rrs.kv_dequant(q, sc, out=out), 10)
    n = T * H * D
    bq = 2 * n + n // 2 + 4 * T * H
    bd = n // 2 + 4 * T * H + 2 * n
    tq, td = max_over_ranks(tq, pg, dev), max_over_ranks(td, pg, dev)
    kvr = {"T": T, "H": H, "D": D, "quant_us": round(tq * 1e3, 2), "dequant_us": round(td * 1e3, 2),
           "quant_GBps": round(bq / (tq * 1e-3) / 1e9, 1), "dequant_GBps": round(bd / (td * 1e-3) / 1e9, 1),
           "quant_frac_hbm": round(bq / (tq * 1e-3) / 1e9 / hbm_peak, 4),
           "dequant_frac_hbm": round(bd / (td * 1e-3) / 1e9 / hbm_peak, 4),
           "bytes": "quantise: fp16 in, packed codes + fp32 scales out; dequantise: the reverse"}
    del kv, q, sc, out
    torch.cuda.empty_cache()
    return {"decode": dec, "kv_cache": kvr}


def mlp_block_times(rrs, wl, dev, stream, warmup, iters, pg):
    """The gated MLP block of LLaMA-3-8B (M = 2048 tokens, K = 4096, F = 14336, G = 128):
    gate/up RRS linear on the fp8 path with SiLU * up fused into its GEMM epilogue
    (interleaved gate/up weight rows), then the down RRS linear (block-diagonal rotation,
    7 blocks of 2048) on H.  Four launches per block; CUDA events around each."""
    M, K, F, G = 2048, 4096, 14336, 128
    Lgu = wl.Layer("llama3_8b_mlp_gateup", M, K, 2 * F, G, 4096, seed=501)
    Lu = wl.Layer("llama3_8b_mlp_up", M, K, F, G, 4096, seed=503)
    Ld = wl.Layer("llama3_8b_mlp_down", M, F, K, G, 2048, seed=502)
    W = rrs.interleave_gate_up(wl.make_weights(Lgu, N=F), wl.make_weights(Lu)).to(dev)
    perm_gu = rrs.calibrate_perm(wl.make_activations(Lgu, sample=1, M=512).to(dev), Lgu.had_block)
    qW, sw_gu = rrs.prepare_weights(W, perm_gu, Lgu.had_block)
    qW_gu = rrs.expand_weights(qW)
    del W, qW
    xs = [wl.make_activations(Lgu, sample=2 + i).to(dev) for i in range(2)]
    flags = rrs.W_EXPANDED
    qX = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    s = torch.empty(K // G, dtype=torch.float32, device=dev)
    st = torch.empty(M, dtype=torch.float32, device=dev)
    H = torch.empty((M, F), dtype=torch.float16, device=dev)
    ws = rrs.make_workspace(M, 2 * F, K, G, Lgu.had_block, flags, device=dev)
    # calibration of the down projection's reorder on the H of a calibration draw
    rrs.linear(wl.make_activations(Lgu, sample=1).to(dev), qW_gu, sw_gu, perm_gu, G, Lgu.had_block,
               flags=flags | rrs.Y_SILU_MUL, Y=H, qX=qX, s=s, scale_t=st, ws=ws)
    perm_d = rrs.calibrate_perm(H[:512], Ld.had_block)
    Wd = wl.make_weights(Ld).to(dev)
    qWd, sw_d = rrs.prepare_weights(Wd, perm_d, Ld.had_block)
    qW_d = rrs.expand_weights(qWd)
    del Wd, qWd
    qXd = torch.empty((M, F // 2), dtype=torch.uint8, device=dev)
    sd = torch.empty(F // G, dtype=torch.float32, device=dev)
    std = torch.empty(M, dtype=torch.float32, device=dev)
    Yd = torch.empty((M, K), dtype=torch.float32, device=dev)
    wsd = rrs.make_workspace(M, K, F, G, Ld.had_block, flags, device=dev)

    def block(i, ev=None):
        if ev is not None:
            ev[0].record(stream)
        rrs.smooth_quant(xs[i % 2], perm_gu, G, Lgu.had_block, flags=flags, qX=qX, s=s, scale_t=st, ws=ws)
        if ev is not None:
            ev[1].record(stream)
        rrs.w4a4_gemm(qX, s, st, qW_gu, sw_gu, G, Y=H, ws=ws, flags=rrs.WS_HOLDS_A8 | flags | rrs.Y_SILU_MUL)
        if ev is not None:
            ev[2].record(stream)
        rrs.smooth_quant(H, perm_d, G, Ld.had_block, flags=flags, qX=qXd, s=sd, scale_t=std, ws=wsd)
        if ev is not None:
            ev[3].record(stream)
        rrs.w4a4_gemm(qXd, sd, std, qW_d, sw_d, G, Y=Yd, ws=wsd, flags=rrs.WS_HOLDS_A8 | flags)
        if ev is not None:
            ev[4].record(stream)

    for i in range(warmup):
        block(i)
    rrs.check_workspace(ws)
    rrs.check_workspace(wsd)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(iters)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    for i in range(iters):
        block(i, evs[i])
    torch.cuda.synchronize()
    rrs.check_workspace(ws)
    rrs.check_workspace(wsd)
    stages = ["gateup_prep", "gateup_gemm_silu_mul", "down_prep", "down_gemm"]
    us = {nm: sum(e[k].elapsed_time(e[k + 1]) for e in evs) / iters * 1e3 for k, nm in enumerate(stages)}
    total = sum(e[0].elapsed_time(e[4]) for e in evs) / iters * 1e3
    total = max_over_ranks(total, pg, dev)
    ops = 2 * M * (2 * F) * K + 2 * M * K * F
    return {"M": M, "K": K, "F": F, "G": G, "down_hadamard": "7 x 2048", "iters": iters,
            "us": {k: round(v, 2) for k, v in us.items()}, "us_total": round(total, 2),
            "TOPS": round(ops / (total * 1e-6) / 1e12, 1), "launches": 4,
            "path": "fp8 (e4m3) MMA; SiLU * up fused into the gate/up GEMM epilogue (H fp16 written once)"}


def _oracle_sample(layers, rows_per_layer, cols_per_layer=None, seed=0):
    """Times the oracle on a row sample of each layer; returns (ops, seconds)."""
    import numpy as np

    import oracle
    from activation_smoothing_b200 import workloads as wl

    ops, secs = 0, 0.0
    for j, L in enumerate(layers):
        r = rows_per_layer
        ncol = L.N if cols_per_layer is None else min(L.N, cols_per_layer)
        X = wl.make_activations(L, sample=2)[:r].contiguous()
        W = wl.make_weights(L, N=ncol)
        perm = np.arange(L.K, dtype=np.int32)
        _, qW, sw = oracle.prepare_weights(W, L.had_block, perm)     # offline, untimed
        t = time.perf_counter()
        _, qX, s, st = oracle.smooth_quant(X, L.G, L.had_block, perm)
        oracle.linear_rows(qX, s, st, qW, sw, L.G)
        secs += time.perf_counter() - t
        ops += 2 * r * ncol * L.K
    return ops, secs


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_worker(job):
    """One process of the all-cores baseline: the oracle on its own slice of rows."""
    names, rows, offset = job
    import numpy as np

    import oracle
    from activation_smoothing_b200 import workloads as wl

    ops, secs = 0, 0.0
    for name in names:
        L = wl.LAYERS[name]
        X = wl.make_activations(L, sample=2, M=offset + rows)[offset:offset + rows].contiguous()
        W = wl.make_weights(L)
        perm = np.arange(L.K, dtype=np.int32)
        _, qW, sw = oracle.prepare_weights(W, L.had_block, perm)     # offline, untimed
        t = time.perf_counter()
        _, qX, s, st = oracle.smooth_quant(X, L.G, L.had_block, perm)
        oracle.linear_rows(qX, s, st, qW, sw, L.G)
        secs += time.perf_counter() - t
        ops += 2 * rows * L.N * L.K
    return ops, secs


def cpu_baseline(layers, budget_s=20.0):
    """The oracle as it stands (plain single-threaded C), on a bounded row sample: once in
    this process, and once as one process per host core on disjoint rows (wall time)."""
    import multiprocessing as mproc

    ops, secs = _oracle_sample(layers, 1)
    rows = max(1, min(64, int(budget_s / 2 / max(secs, 1e-6))))
    ops, secs = _oracle_sample(layers, rows)
    single = {"value": ops / secs / 1e12, "unit": UNIT, "cores": 1, "seconds": round(secs, 2),
              "sample": f"{rows} token rows of each layer"}
    ncpu = os.cpu_count() or 1
    procs = max(1, min(ncpu, 16))
    per = max(1, rows // 4)
    names = [L.name for L in layers]
    ctx = mproc.get_context("spawn")          # the parent has a CUDA context: never fork
    with ctx.Pool(procs) as pool:
        pool.map(_oracle_worker, [(names[:1], 1, 0)] * procs)        # start-up and imports, untimed
        jobs = [(names, per, i * per) for i in range(procs)]
        t = time.perf_counter()
        res = pool.map(_oracle_worker, jobs)
        wall = time.perf_counter() - t
    tot_ops = sum(r[0] for r in res)
    # the workers also prepare their weights (untimed inside each worker); charge the
    # wall time only with the timed part: the slowest worker's timed seconds
    busy = max(r[1] for r in res)
    return {"value": tot_ops / busy / 1e12, "unit": UNIT, "cores": procs, "kind": "oracle",
            "sample": f"{per} token rows of each layer per process x {procs} processes (disjoint rows; prep of "
                      f"those rows + their GEMM rows, all N); weights prepared untimed; single-threaded C per process",
            "nproc": ncpu, "cpu_model": _cpu_model(), "wall_seconds": round(wall, 2), "single_thread": single}


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    from activation_smoothing_b200 import workloads as wl

    names = args.workload.split(",") if args.workload else wl.HEADLINE
    layers = [wl.LAYERS[n] for n in names]
    # size each step so the whole run stays within about args.cpu_budget seconds
    per_step = args.cpu_budget / max(1, args.steps + args.warmup)
    ops1, s1 = _oracle_sample(layers, 1, cols_per_layer=256)
    cols = max(16, min(max(L.N for L in layers), int(256 * per_step / max(s1, 1e-6))))
    for _ in range(args.warmup):
        _oracle_sample(layers, 1, cols_per_layer=cols)
    tot_ops, tot_s = 0, 0.0
    for _ in range(args.steps):
        o, s = _oracle_sample(layers, 1, cols_per_layer=cols)
        tot_ops += o
        tot_s += s
    v = tot_ops / tot_s / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_s * 1e3 / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32/int (CPU oracle)",
           "data": "synthetic", "config": bench_config(names, layers, world),
           "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                            "sample": f"per step: 1 token row of each layer, prep + GEMM against {cols} "
                                      f"output columns; weights prepared untimed"},
           "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def _time_ms(fn, iters: int = 20) -> float:
    """Mean device time of fn() in ms.  The calls are captured in a CUDA graph and the
    graph is replayed (CUDA events on the current stream), so that host launch overhead
    does not hide the kernel time of small (decode) calls; eager calls if capture fails."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(iters):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters
    except Exception:
        torch.cuda.synchronize()
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters


def run_report(args):
    """The other configurations: group-size sweep (cost and output error of RRS and of
    plain Runtime Smooth against the unquantised fp32 GEMM), the 8B down projection,
    the 70B layers and the 70B decode token counts.  One JSON line; not the bench line."""
    import activation_smoothing_b200 as rrs
    from activation_smoothing_b200 import workloads as wl

    torch.backends.cuda.matmul.allow_tf32 = False
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    out = {"report": "RRS W4A4 linear: other configurations", "sweep": [], "layers": []}

    def layer_times(L, X, W, n, flags=0, iters=20, fp8=True):
        """(prep ms, GEMM ms, Y) of one layer; fp8: the e4m3 operand path (the headline's),
        else the packed INT4 weights on the int8 kernel."""
        perm = rrs.calibrate_perm(wl.make_activations(L, sample=1, M=min(L.M, 512)).to(dev), n)
        qW, sw = rrs.prepare_weights(W, perm, n, flags)
        fx = rrs.W_EXPANDED if fp8 else 0
        if fp8:
            qW = rrs.expand_weights(qW)
        qX = torch.empty((L.M, L.K // 2), dtype=torch.uint8, device=dev)
        s = torch.empty(L.K // L.G, dtype=torch.float32, device=dev)
        st = torch.empty(L.M, dtype=torch.float32, device=dev)
        Y = torch.empty((L.M, L.N), dtype=torch.float32, device=dev)
        ws = rrs.make_workspace(L.M, L.N, L.K, L.G, n, flags | fx, device=dev)
        prep = _time_ms(lambda: rrs.smooth_quant(X, perm, L.G, n, flags | fx, qX=qX, s=s, scale_t=st, ws=ws), iters)
        gemm = _time_ms(lambda: rrs.w4a4_gemm(qX, s, st, qW, sw, L.G, Y=Y, ws=ws, flags=rrs.WS_HOLDS_A8 | fx), iters)
        rrs.smooth_quant(X, perm, L.G, n, flags | fx, qX=qX, s=s, scale_t=st, ws=ws)
        rrs.w4a4_gemm(qX, s, st, qW, sw, L.G, Y=Y, ws=ws, flags=rrs.WS_HOLDS_A8 | fx)
        rrs.check_workspace(ws)
        return prep, gemm, Y

    only = args.workload.split(",") if args.workload else None
    if only is None:
        run_report_sweep_and_mlp(rrs, wl, dev, out, layer_times)
    names = ["llama3_8b_down", "llama3_70b_qo", "llama3_70b_gateup", "llama3_70b_down",
             "llama3_70b_qo_decode_m1", "llama3_70b_qo_decode_m8", "llama3_70b_qo_decode_m16",
             "llama3_70b_gateup_decode_m1", "llama3_70b_gateup_decode_m16",
             "llama3_70b_down_decode_m1", "llama3_70b_down_decode_m16"]
    for nm in only or names:
        if nm not in wl.LAYERS:
            continue
        L = wl.LAYERS[nm]
        X = wl.make_activations(L).to(dev)
        W = wl.make_weights(L).to(dev)
        int8_peak, hbm_peak, _ = peaks()
        if L.M <= 16:
            entry = decode_entry(rrs, wl, dev, L, X, W, hbm_peak)
        else:
            prep, gemm, _ = layer_times(L, X, W, L.had_block)
            entry = {"layer": nm, "M": L.M, "K": L.K, "N": L.N, "G": L.G, "n": L.had_block,
                     "prep_us": round(prep * 1e3, 2), "gemm_us": round(gemm * 1e3, 2),
                     "TOPS": round(L.ops / ((prep + gemm) * 1e-3) / 1e12, 2),
                     "gemm_frac_peak": round(L.ops / (gemm * 1e-3) / 1e12 / int8_peak, 4),
                     "path": "fp8 (e4m3) operands, CTA-pair tiles"}
        out["layers"].append(entry)
        del X, W
        torch.cuda.empty_cache()
    print(json.dumps(out), flush=True)


def decode_entry(rrs, wl, dev, L, X, W, hbm_peak, iters=24):
    """A decode layer (M <= 16): rrs_linear as it chooses, its single launch forced
    (RRS_ONE_LAUNCH), and the two launches (activation kernel, then the GEMM).  Each timed call reads its own copy of the
    packed weights, enough copies that they exceed L2, so the weight stream comes
    from HBM as it would in a model's layer sequence."""
    n = L.had_block
    perm = wl.random_perm(L.K, 1).to(dev)
    qW, sw = rrs.prepare_weights(W, perm, n)
    wbytes = L.N * L.K // 2
    copies = max(2, min(12, -(-320_000_000 // wbytes)))
    qWs = [qW] + [qW.clone() for _ in range(copies - 1)]
    qX = torch.empty((L.M, L.K // 2), dtype=torch.uint8, device=dev)
    s = torch.empty(L.K // L.G, dtype=torch.float32, device=dev)
    st = torch.empty(L.M, dtype=torch.float32, device=dev)
    Y = torch.empty((L.M, L.N), dtype=torch.float32, device=dev)
    ws = rrs.make_workspace(L.M, L.N, L.K, L.G, n, device=dev)
    k = [0]

    def nxt():
        k[0] = (k[0] + 1) % copies
        return qWs[k[0]]

    one = _time_ms(lambda: rrs.linear(X, nxt(), sw, perm, L.G, n, flags=rrs.ONE_LAUNCH, Y=Y, qX=qX, s=s,
                                      scale_t=st, ws=ws), iters)
    dflt = _time_ms(lambda: rrs.linear(X, nxt(), sw, perm, L.G, n, Y=Y, qX=qX, s=s, scale_t=st, ws=ws), iters)
    rrs.check_workspace(ws)

    def two_launches():
        rrs.smooth_quant(X, perm, L.G, n, qX=qX, s=s, scale_t=st, ws=ws)
        rrs.w4a4_gemm(qX, s, st, nxt(), sw, L.G, Y=Y, ws=ws, flags=rrs.WS_HOLDS_A8)

    two = _time_ms(two_launches, iters)
    prep = _time_ms(lambda: rrs.smooth_quant(X, perm, L.G, n, qX=qX, s=s, scale_t=st, ws=ws), iters)
    rrs.check_workspace(ws)
    gbps = wbytes / (one * 1e-3) / 1e9
    return {"layer": L.name, "M": L.M, "K": L.K, "N": L.N, "G": L.G, "n": n,
            "rrs_linear_us": round(dflt * 1e3, 2),
            "single_launch_us": round(one * 1e3, 2), "two_launches_us": round(two * 1e3, 2),
            "prep_us": round(prep * 1e3, 2), "weight_copies_rotated": copies,
            "single_launch_weight_GBps": round(gbps, 1),
            "single_launch_frac_hbm": round(gbps / hbm_peak, 4),
            "TOPS": round(L.ops / (one * 1e-3) / 1e12, 3)}


def run_report_sweep_and_mlp(rrs, wl, dev, out, layer_times):
    # group-size sweep on the K=4096, N=14336, M=2048 layer
    base = wl.Layer("sweep", 2048, 4096, 14336, 128, 4096, seed=4242)
    X = wl.make_activations(base).to(dev)
    W = wl.make_weights(base).to(dev)
    Yref = X.float() @ W.float().t()
    nref = torch.linalg.vector_norm(Yref).item()
    for G in (128, 256, 512, 4096):
        for name, n in (("RRS", 4096), ("RS", 1)):
            L = wl.Layer("sweep", 2048, 4096, 14336, G, n, seed=4242)
            prep, gemm, Y = layer_times(L, X, W, n)
            err = torch.linalg.vector_norm(Y - Yref).item() / nref
            out["sweep"].append({"G": G, "method": name, "prep_us": round(prep * 1e3, 2), "gemm_us": round(gemm * 1e3, 2),
                                 "TOPS": round(L.ops / ((prep + gemm) * 1e-3) / 1e12, 1),
                                 "rel_frobenius_error_vs_fp32_gemm": float(f"{err:.5g}")})
    del X, W, Yref
    torch.cuda.empty_cache()

    # gated MLP block at LLaMA-3-8B sizes: gate/up linear (N = 2 x 14336), SiLU * up, down linear
    Lgu = wl.Layer("llama3_8b_mlp_gateup", 2048, 4096, 2 * 14336, 128, 4096, seed=501)
    Ld = wl.Layer("llama3_8b_mlp_down", 2048, 14336, 4096, 128, 2048, seed=502)
    Xgu = wl.make_activations(Lgu).to(dev)
    prep_gu, gemm_gu, GU = layer_times(Lgu, Xgu, wl.make_weights(Lgu).to(dev), Lgu.had_block, fp8=False)
    H = torch.empty((2048, 14336), dtype=torch.float16, device=dev)
    silu = _time_ms(lambda: rrs.silu_mul(GU, H=H))
    rrs.silu_mul(GU, H=H)
    permd = rrs.calibrate_perm(H[:512], Ld.had_block)
    qWd, swd = rrs.prepare_weights(wl.make_weights(Ld).to(dev), permd, Ld.had_block)
    qXd = torch.empty((Ld.M, Ld.K // 2), dtype=torch.uint8, device=dev)
    sd = torch.empty(Ld.K // Ld.G, dtype=torch.float32, device=dev)
    std = torch.empty(Ld.M, dtype=torch.float32, device=dev)
    Yd = torch.empty((Ld.M, Ld.N), dtype=torch.float32, device=dev)
    wsd = rrs.make_workspace(Ld.M, Ld.N, Ld.K, Ld.G, Ld.had_block, device=dev)
    prep_d = _time_ms(lambda: rrs.smooth_quant(H, permd, Ld.G, Ld.had_block, qX=qXd, s=sd, scale_t=std, ws=wsd))
    gemm_d = _time_ms(lambda: rrs.w4a4_gemm(qXd, sd, std, qWd, swd, Ld.G, Y=Yd, ws=wsd, flags=rrs.WS_HOLDS_A8))
    rrs.check_workspace(wsd)
    total = prep_gu + gemm_gu + silu + prep_d + gemm_d
    out["mlp_block_unfused_packed"] = {"M": 2048, "K": 4096, "F": 14336, "G": 128,
                        "path": "packed INT4 weights (int8 GEMM), rrs_silu_mul as its own pass; the fused fp8 "
                                "block is the bench line's mlp_block",
                        "us": {"gateup_prep": round(prep_gu * 1e3, 2), "gateup_gemm": round(gemm_gu * 1e3, 2),
                               "silu_mul": round(silu * 1e3, 2), "down_prep": round(prep_d * 1e3, 2),
                               "down_gemm": round(gemm_d * 1e3, 2), "total": round(total * 1e3, 2)},
                        "silu_mul_GBps": round(2048 * 14336 * 10 / (silu * 1e-3) / 1e9, 1),
                        "TOPS": round((Lgu.ops + Ld.ops) / (total * 1e-3) / 1e12, 1)}
    del Xgu, GU, H
    torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="", help="comma-separated layer names (default: headline shapes)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mlp", action="store_true", help="skip the MLP-block, decode and KV-cache rows")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--report", action="store_true",
                    help="print the other configurations (group sweep, 8B down, 70B, decode) instead")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit(relaunch(args.gpus))
    if args.report:
        run_report(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
