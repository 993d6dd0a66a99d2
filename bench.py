"""Benchmark: ternary MoE FFN decode, batch 1, through a 24-layer stack on B200.

Workload: 24 residual MoE FFN layers (d=2048, 256 SwiGLU experts of 512x2048 / 2048x512,
ternary weights packed 2 bits per code, per-row fp32 scales, bf16 router, top-8), about
4.93 GB resident in HBM; each step decodes ONE token through all 24 layers with
x <- x + FFN(RMSNorm(x)) in bf16.  Synthetic seeded data (no trained weights exist here).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--act bf16|int8] [--impl reference]

Timing: W warm-up steps, then K timed steps.  The L2 cache (126 MB) is flushed before every
timed step by writing a 256 MB buffer; each step is bracketed by CUDA events on the stream
the library launches on, and the device time of a step excludes the flush.  `value` is
tokens/s over all ranks (one independent replica per GPU, no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# side files (clock samples, per-phase traces) go here
OUT_DIR = os.environ.get("TERNMOE_BENCH_OUT", os.path.join(ROOT, "bench_out"))

METRIC = "ternary MoE FFN decode tokens/s @batch1; achieved HBM GB/s vs B200 peak"
UNIT = "tokens/s"
N_LAYERS = 24
WID = 5
BYTES_PER_LAYER_TOKEN = 8 * (786432 + 12288) + 1048576   # experts' packed codes + scales, router
BYTES_PER_TOKEN = N_LAYERS * BYTES_PER_LAYER_TOKEN       # 178,520,064 B
WORKLOAD = ("24-layer ternary MoE FFN stack, batch-1 decode: d=2048, E=256 SwiGLU experts "
            "512x2048/2048x512, top-8, 2-bit packed ternary weights, bf16 router")


def _config(act_name, world, l2):
    return {"workload": WORKLOAD, "layers": N_LAYERS, "batch": 1, "d": 2048, "f": 512, "experts": 256,
            "top_k": 8, "activations": act_name, "resident_bytes": 4932501504,
            "weight_bytes_per_token": BYTES_PER_TOKEN, "parallelism": f"replicas{world}", "l2": l2}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ rank plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def aggregate(values, op, world, backend_device=None):
    """max/sum of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return float(values)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(values)], dtype=torch.float64, device=backend_device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(OUT_DIR, f"clocks_rank{gpu_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ model

def device_layer(layer, shape, dev):
    """One synthetic layer generated on the device and packed by the library's packer."""
    import torch

    import synth
    import ternary_weight_moe_b200 as tm

    E, d, f = shape.E, shape.d, shape.f
    gc, uc, dc = synth.layer_codes_torch(WID, layer, shape, dev)
    gate = tm.tern_pack(gc.view(E * f, d)).view(E, f, d // 4)
    up = tm.tern_pack(uc.view(E * f, d)).view(E, f, d // 4)
    down = tm.tern_pack(dc.view(E * d, f)).view(E, d, f // 4)
    del gc, uc, dc
    sg, su, sd = synth.layer_scales(WID, layer, shape)
    router = synth.layer_router(WID, layer, shape)
    return tm.MoELayer(gate, up, down, torch.from_numpy(sg).to(dev), torch.from_numpy(su).to(dev),
                       torch.from_numpy(sd).to(dev), torch.from_numpy(router.view(np.int16)).to(dev), k=shape.k)


def build_stack(dev):
    import synth
    import ternary_weight_moe_b200 as tm

    shape = synth.MoEShape()
    layers = [device_layer(l, shape, dev) for l in range(N_LAYERS)]
    return shape, layers, tm.Stack(layers)


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores():
    return len(os.sched_getaffinity(0))


def _oracle_tokens(act_oracle, omp, n_tokens, seed0, hosts=None):
    """Decode n_tokens whole tokens through the 24-layer stack with the CPU oracle; returns
    (seconds inside the oracle, tokens).  Experts are regenerated on the host (from the same
    seeds as the device stack) outside the timed region."""
    import oracle
    import synth
    from tests.gpu_cases import HostLayer

    shape = synth.MoEShape()
    hosts = hosts if hosts is not None else [HostLayer(WID, l, shape) for l in range(N_LAYERS)]
    spent = 0.0
    for t in range(n_tokens):
        x = synth.tokens_bf16(WID, seed0 + t, 1, shape.d)
        for l in range(N_LAYERS):
            n, _ = oracle.rmsnorm(x, 1e-6)
            _, idx, _, _ = hosts[l].route(n)
            hosts[l].fill(idx)
            L = hosts[l].oracle_layer()
            t0 = time.perf_counter()
            x = oracle.stack_layer(L, x, eps=1e-6, act=act_oracle, omp=omp)["x_out"]
            spent += time.perf_counter() - t0
    return spent, n_tokens


def cpu_baseline(act_oracle, n_tokens=4):
    """The oracle (C, fp64/exact) decoding whole tokens through the same 24-layer stack, on
    all host cores (the OpenMP build: rows split across threads, identical results) and on
    one core (the single-threaded build)."""
    import oracle

    oracle.build(omp=True)
    spent_all, tok = _oracle_tokens(act_oracle, True, n_tokens, 50000)
    spent_one, tok1 = _oracle_tokens(act_oracle, False, n_tokens, 50000)
    cores = host_cores()
    return {"value": tok / spent_all, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "single_thread": {"value": tok1 / spent_one, "unit": UNIT, "cores": 1},
            "sample": f"{tok} whole tokens x {N_LAYERS} layers through the CPU oracle (C, fp64/exact): the OpenMP "
                      f"build on all {cores} cores (value) and the single-threaded build (single_thread); host "
                      "expert regeneration excluded"}


PHASES = [("x_wait", 0, 1), ("norm_router", 1, 2), ("limbs_predict", 2, 3), ("logits_wait", 3, 4),
          ("topk_issue", 4, 5), ("gate_up_rows_wait", 5, 6), ("gate_up_dots", 6, 7), ("swiglu", 7, 8),
          ("h_wait", 8, 9), ("h_limbs", 9, 10), ("down_rows_wait", 10, 11), ("down_dots", 11, 12),
          ("y_wait", 12, 13), ("combine", 13, 14)]


INNER_PHASES = [("r", 1, 15), ("n", 15, 16), ("router_rows", 16, 17), ("router_publish", 17, 2),
                ("topk", 4, 18), ("copy_issue", 18, 5)]


def phase_summary(tr, clk=None, mhz=1965.0, k=8):
    """Median over CTAs and layers of each phase (us; from SM clock stamps when given, else
    from %globaltimer), the exchange latencies, and the layer time.  CTA p is part p % G of
    slot group p // G (G = P / k)."""
    if clk is not None:
        d = lambda a, b: np.median((clk[:, :, b] - clk[:, :, a]).astype(np.float64)) / mhz
    else:
        d = lambda a, b: np.median((tr[:, :, b] - tr[:, :, a]).astype(np.float64)) / 1e3
    out = {name: round(float(d(a, b)), 3) for name, a, b in PHASES}
    # inside phases (CTA thread 0): r known (15), n known (16), own router partials (17), top-k
    # known (18)
    out["inner"] = {name: round(float(d(a, b)), 3) for name, a, b in INNER_PHASES}
    L, P, _ = tr.shape
    G = P // k
    by_slot = tr.reshape(L, k, G, -1)            # [layer, slot group, part, stamp]
    by_part = by_slot.transpose(0, 2, 1, 3)      # [layer, part, slot, stamp]
    # exchange latency: last producer's publish -> first consumer's receipt, within the group
    # that exchanges (all CTAs for the logits, a slot group for h and x, a part for y)
    e_log = np.median(tr[:, :, 4].min(1) - tr[:, :, 2].max(1)) / 1e3
    e_h = np.median(by_slot[:, :, :, 9].min(2) - by_slot[:, :, :, 8].max(2)) / 1e3
    e_y = np.median(by_part[:, :, :, 13].min(2) - by_part[:, :, :, 12].max(2)) / 1e3
    e_x = np.median(by_slot[1:, :, :, 1].min(2) - by_slot[:-1, :, :, 14].max(2)) / 1e3
    out["exchange_latency"] = {"logits": round(float(e_log), 3), "h": round(float(e_h), 3),
                               "y": round(float(e_y), 3), "x": round(float(e_x), 3)}
    out["layer_total"] = round(float(np.median(np.diff(tr[:, :, 0].min(1)))) / 1e3, 3)
    return out


def kernel_source_hash():
    import hashlib

    parts = ["stack.cu", "tern_common.cuh", "tma.cuh", "kernels.h", "decode.cuh", "cluster.cuh"]
    src = "".join(open(os.path.join(ROOT, "ternary_weight_moe_b200", "csrc", p)).read() for p in parts)
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def kernel_traffic(act):
    """DRAM bytes per launch from the committed ncu record, or None if the kernel changed since."""
    try:
        tj = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
        rec = tj.get(f"stack_kernel_{act}")
        if rec and rec.get("valid") and rec.get("source_hash") == kernel_source_hash():
            return rec["bytes_per_launch"]
    except (OSError, ValueError):
        pass
    return None


def run_reference(args):
    """--impl reference: the CPU oracle as the reference arm (rank 0 only).  One step = one
    whole token through the 24 layers, on all host cores (the oracle's OpenMP build)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    import synth
    from tests.gpu_cases import HostLayer

    act = oracle.ACT_INT8 if args.act == "int8" else oracle.ACT_BF16
    oracle.build(omp=True)
    shape = synth.MoEShape()
    hosts = [HostLayer(WID, l, shape) for l in range(N_LAYERS)]
    # tokens cycle over a small set so the host copies of the experts stay bounded
    ntok = 4
    for i in range(args.warmup):
        _oracle_tokens(act, True, 1, 60000 + i % ntok, hosts)
    spent = sum(_oracle_tokens(act, True, 1, 60000 + (args.warmup + i) % ntok, hosts)[0] for i in range(args.steps))
    value = args.steps / spent
    cores = host_cores()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": spent / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(args.act, world, "n/a (CPU)"), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": f"{args.steps} whole tokens (24 layers each) through the CPU oracle "
                                       f"(C, fp64/exact, OpenMP build on all {cores} cores)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_latency_probe(args):
    """--latency-probe: compile and run ternary_weight_moe_b200/probes/latency_probe.cu (dependent
    operation chains, barriers, two top-k formulations, bulk-copy issue; cycles) and print its
    JSON line."""
    here = os.path.join(ROOT, "ternary_weight_moe_b200")
    src = os.path.join(here, "probes", "latency_probe.cu")
    exe = os.path.join(here, "_build", "latency_probe")
    os.makedirs(os.path.dirname(exe), exist_ok=True)
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-fmad=false", "--expt-relaxed-constexpr", "-o", exe, src])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    print(out.stdout.strip(), flush=True)
    return out.returncode


def run_gemv_sweep(args):
    """Extra output: device time of one tern_gemv launch (four codes per byte) and one
    tern5_gemv launch (five weights per byte, base 3) per shape of the GEMV sweep (T = 1, bf16
    and int8 activations), L2 flushed before every launch; one JSON line per case.  The last
    shape (128 MB of packed codes) is a bandwidth check, not one of the sweep's."""
    import torch

    import synth
    import ternary_weight_moe_b200 as tm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    shapes = list(synth.GEMV_SWEEP) + [(32768, 16384)]
    if args.shape:
        shapes = [tuple(int(v) for v in args.shape.split("x"))]
    for (M, K) in shapes:
        base = synth.derive(synth.BASE_SEED + 2, M, K)
        w = synth.ternary_codes_torch(synth.derive(base, synth.KIND_W), 0, M * K, synth.P0_SPARSE, dev).view(M, K)
        Wp = tm.tern_pack(w)
        W5 = tm.tern5_pack(w)  # five weights per byte, for the base-3 lines
        del w
        rs = torch.from_numpy(synth.uniform_f32(synth.derive(base, synth.KIND_S), 0, M, 0.01, 0.05)).to(dev)
        xb = torch.from_numpy(synth.normal_bf16(synth.derive(base, synth.KIND_X), 0, K, 1.0).view(np.int16)).to(dev)
        xi = torch.from_numpy(synth.int8_uniform(synth.derive(base, synth.KIND_XQ), 0, K)).to(dev)
        y = torch.empty((1, M), dtype=torch.float32, device=dev)
        cases = [("2bit", act_name, act, x) for act_name, act, x in
                 (("bf16", tm.TERN_ACT_BF16, xb), ("int8", tm.TERN_ACT_INT8, xi))]
        cases += [("base3", c[1], c[2], c[3]) for c in cases]
        for fmt, act_name, act, x in cases:
            if args.act_only and act_name != args.act:
                continue
            if fmt == "2bit":
                call = lambda: tm.tern_gemv(Wp, rs, x, act=act, y=y)  # noqa: E731
                wbytes = M * K // 4
            else:
                call = lambda: tm.tern5_gemv(W5, rs, x, K, act=act, y=y)  # noqa: E731
                wbytes = M * tm.tern5_row_bytes(K)
            for _ in range(max(args.warmup, 3)):
                call()
            # no host wait inside the loop: the flush keeps the device busy while the host
            # enqueues the next launch, so the events see device time only
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            torch.cuda.synchronize(dev)
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                evs[i][0].record(stream)
                call()
                evs[i][1].record(stream)
            torch.cuda.synchronize(dev)
            ms = [a.elapsed_time(b) for a, b in evs]
            if tm.tern_stream_status() != 0:
                raise RuntimeError("device status set during the sweep")
            med = statistics.median(ms)
            nbytes = wbytes + 4 * M + (2 if act_name == "bf16" else 1) * K + 4 * M
            gbs = nbytes / (med * 1e-3) / 1e9
            print(json.dumps({"gemv": f"{M}x{K}", "format": fmt, "act": act_name, "us_median": med * 1e3,
                              "us_p10": float(np.percentile(ms, 10)) * 1e3, "bytes": nbytes, "GB/s": gbs,
                              "frac": gbs / peak, "peak": peak, "peak_kind": peak_kind, "launches": args.steps}),
                  flush=True)
        del Wp, W5
    return 0


def run_batch_sweep(args):
    """Extra output: one MoE FFN layer (d=2048, 256 experts, top-8) through moe_ffn_decode at
    T = 1, 4, 16, 64 tokens per step (the kernel-per-stage path), L2 flushed before every step;
    one JSON line per (T, activations).  Algorithmic bytes per step = U * 798,720 (packed rows
    and scales of the U distinct experts the step routes to) + 1,048,576 (router)."""
    import torch

    import synth
    import ternary_weight_moe_b200 as tm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = peaks()
    shape = synth.MoEShape()
    layer = device_layer(0, shape, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for T in ([int(v) for v in args.batch_T.split(",")] if args.batch_T else (1, 4, 16, 64)):
        xs_host = synth.tokens_bf16(WID, 90000 + 1000 * T, args.steps + 3, T * shape.d).reshape(-1, T, shape.d)
        xs = torch.from_numpy(xs_host.view(np.int16)).to(dev)
        for act_name, act in (("bf16", tm.TERN_ACT_BF16), ("int8", tm.TERN_ACT_INT8)):
            if args.act_only and act_name != args.act:
                continue
            ws = tm.workspace(tm.moe_ffn_workspace_bytes(layer, T, act), dev)
            lay = tm.moe_ffn_workspace_layout(layer, T, act)
            y = torch.empty((T, shape.d), dtype=torch.bfloat16, device=dev)
            for i in range(3):
                tm.moe_ffn_decode(layer, xs[i], act=act, ws=ws, y=y)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            uniq = []
            torch.cuda.synchronize(dev)
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                evs[i][0].record(stream)
                tm.moe_ffn_decode(layer, xs[3 + i], act=act, ws=ws, y=y)
                evs[i][1].record(stream)
                if i < 8:  # distinct experts of a few steps (copied after the step's end event)
                    idx = ws[lay["idx"]:lay["idx"] + 4 * T * shape.k].view(torch.int32).cpu().numpy()
                    uniq.append(len(np.unique(idx)))
            torch.cuda.synchronize(dev)
            if tm.tern_stream_status() != 0:
                raise RuntimeError("device status set during the batch sweep")
            ms = [a.elapsed_time(b) for a, b in evs]
            med = statistics.median(ms)
            U = float(np.mean(uniq))
            nbytes = U * 798720 + 1048576
            gbs = nbytes / (med * 1e-3) / 1e9
            print(json.dumps({"moe_ffn_decode": f"T={T}", "act": act_name, "us_median": med * 1e3,
                              "us_p10": float(np.percentile(ms, 10)) * 1e3, "tokens_per_s": T / (med * 1e-3),
                              "unique_experts": U, "bytes": nbytes, "GB/s": gbs, "frac": gbs / peak,
                              "peak": peak, "peak_kind": peak_kind, "steps": args.steps}), flush=True)
    return 0


def run_stack_batch(args):
    """Extra output: the 24-layer stack through moe_stack_decode with T = 1, 2, 4, 8, 16 tokens
    per call (T = 1: the batch-1 kernel; 2 <= T <= 16: the one-launch small-batch kernel), L2
    flushed before every call; one JSON line per (T, activations).  Algorithmic bytes per call
    = sum over layers of (U_l * 798,720 + 1,048,576), U_l = the distinct experts of layer l
    (from the call's per-layer record)."""
    import torch

    import synth
    import ternary_weight_moe_b200 as tm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = peaks()
    shape, layers, st = build_stack(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for T in ([int(v) for v in args.batch_T.split(",")] if args.batch_T else (1, 2, 4, 8, 16)):
        xs_host = synth.tokens_bf16(WID, 95000 + 1000 * T, args.steps + 3, T * shape.d).reshape(-1, T, shape.d)
        xs = torch.from_numpy(xs_host.view(np.int16)).to(dev)
        for act_name, act in (("bf16", tm.TERN_ACT_BF16), ("int8", tm.TERN_ACT_INT8)):
            if args.act_only and act_name != args.act:
                continue
            ws = tm.workspace(tm.moe_stack_workspace_bytes(layers[0], T, act), dev)
            lay = tm.moe_stack_workspace_layout(layers[0], T, act)
            launches = tm.moe_stack_kernel_launches(layers[0], N_LAYERS, T, act)
            buf = xs[0].clone()
            for i in range(3):
                buf.copy_(xs[i])
                tm.moe_stack_decode(st, buf, act=act, ws=ws)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            uniq = []
            torch.cuda.synchronize(dev)
            for i in range(args.steps):
                buf.copy_(xs[3 + i])
                flush.fill_(i & 0xFF)
                evs[i][0].record(stream)
                tm.moe_stack_decode(st, buf, act=act, ws=ws)
                evs[i][1].record(stream)
                if i < 4 and launches == 1:
                    idx = ws[lay["idx"]:lay["idx"] + 4 * N_LAYERS * T * shape.k].view(torch.int32)
                    idx = idx.view(N_LAYERS, T * shape.k).cpu().numpy()
                    uniq.append([len(np.unique(r)) for r in idx])
            torch.cuda.synchronize(dev)
            if tm.tern_stream_status() != 0:
                raise RuntimeError("device status set during the stack batch sweep")
            ms = [a.elapsed_time(b) for a, b in evs]
            med = statistics.median(ms)
            phases = None
            if launches == 1 and T >= 2:
                # one extra traced call (not timed): clock64 stamps per layer and CTA
                os.environ["TERNMOE_TRACE"] = "1"
                buf.copy_(xs[3])
                tm.moe_stack_decode(st, buf, act=act, ws=ws)
                torch.cuda.synchronize(dev)
                os.environ["TERNMOE_TRACE"] = "0"
                P = torch.cuda.get_device_properties(dev).multi_processor_count
                tr = ws[lay["trace"]:lay["trace"] + 8 * N_LAYERS * P * 16].view(torch.int64)
                tr = tr.view(N_LAYERS, P, 16).cpu().numpy().astype(np.float64) / 1965.0
                phases = batch_phase_summary(tr)
            U = float(np.mean(uniq)) if uniq else float("nan")
            nbytes = N_LAYERS * (U * 798720 + 1048576)
            gbs = nbytes / (med * 1e-3) / 1e9
            print(json.dumps({"moe_stack_decode": f"T={T}", "act": act_name, "layers": N_LAYERS, "launches": launches,
                              "us_per_call": med * 1e3, "us_per_layer": med * 1e3 / N_LAYERS,
                              "us_p10": float(np.percentile(ms, 10)) * 1e3, "tokens_per_s": T / (med * 1e-3),
                              "unique_experts_per_layer": U, "bytes": nbytes, "GB/s": gbs, "frac": gbs / peak,
                              "peak": peak, "peak_kind": peak_kind, "steps": args.steps,
                              "layer_phase_us_traced_call": phases}), flush=True)
    return 0


BATCH_PHASES = [("A_sum_sq", 0, 8), ("A_fold", 8, 9), ("A_limbs_router", 9, 10), ("A_publish", 10, 1),
                ("barrier1_load_logits", 1, 11), ("B_topk_gates", 11, 12), ("B_group", 12, 2), ("C_gate_up", 2, 3),
                ("barrier2", 3, 4), ("D_down", 4, 5), ("barrier3", 5, 6), ("E_combine", 6, 7)]


def batch_phase_summary(tr):
    """Small-batch kernel trace [layers][P][16] (us from SM clock stamps): median over CTAs and
    layers of each phase, the slowest CTA's C and D, and the layer time (start to start)."""
    out = {name: round(float(np.median(tr[:, :, b] - tr[:, :, a])), 3) for name, a, b in BATCH_PHASES}
    out["C_copy_wait"] = round(float(np.median(tr[:, :, 13])), 3)  # stored as durations
    out["D_copy_wait"] = round(float(np.median(tr[:, :, 14])), 3)
    out["C_gate_up_max"] = round(float(np.median((tr[:, :, 3] - tr[:, :, 2]).max(1))), 3)
    out["D_down_max"] = round(float(np.median((tr[:, :, 5] - tr[:, :, 4]).max(1))), 3)
    out["layer_total"] = round(float(np.median(np.diff(tr[:, :, 0].min(1)))), 3)
    return out


def run_head(args):
    """Extra output: the approximate output head (151,936 tokens in 4,748 clusters of 32,
    d = 2048, top 512 clusters) against the full head (every cluster kept), one token per
    call, L2 flushed before every call; one JSON line each."""
    import torch

    import synth
    import ternary_weight_moe_b200 as tm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = peaks()
    hs = synth.head_shape()
    V, d, nc, cs = hs["V"], hs["d"], hs["n_clusters"], hs["cluster_size"]
    W = synth.normal_bf16_torch(synth.derive(synth.BASE_SEED + 6, 1), 0, V * d, 0.02, dev).view(V, d)
    C4, sc = tm.flash_head_centroids(W, cs)
    xs = torch.from_numpy(synth.normal_bf16(synth.derive(synth.BASE_SEED + 6, 3), 0, (args.steps + 3) * d, 1.0)
                          .view(np.int16)).to(dev).view(-1, d)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for name, top_c in (("flash_head top-512", hs["top_c"]), ("full head", nc)):
        out = tm.flash_head(C4, sc, W, xs[0], cs, top_c)
        for i in range(3):
            tm.flash_head(C4, sc, W, xs[i], cs, top_c, out=out)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            evs[i][0].record(stream)
            tm.flash_head(C4, sc, W, xs[3 + i], cs, top_c, out=out)
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        ms = [a.elapsed_time(b) for a, b in evs]
        med = statistics.median(ms)
        nbytes = nc * (d // 2 + 8) + top_c * cs * (2 * d + 12) + 2 * d + 8 * nc
        gbs = nbytes / (med * 1e-3) / 1e9
        print(json.dumps({"head": name, "top_clusters": top_c, "us_median": med * 1e3,
                          "us_p10": float(np.percentile(ms, 10)) * 1e3, "tokens_per_s": 1.0 / (med * 1e-3),
                          "bytes": nbytes, "GB/s": gbs, "frac": gbs / peak, "peak": peak, "peak_kind": peak_kind,
                          "vocab": V, "d": d, "steps": args.steps}), flush=True)
    return 0


def main():
    global N_LAYERS, BYTES_PER_TOKEN
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--act", choices=["bf16", "int8"], default="bf16")
    ap.add_argument("--impl", default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=N_LAYERS,
                    help="profiling only: a shorter stack (the benchmark line is the 24-layer stack)")
    ap.add_argument("--sweep", action="store_true",
                    help="extra output: time tern_gemv over the GEMV shape sweep instead of the stack")
    ap.add_argument("--shape", default=None, help="with --sweep: one shape MxK only")
    ap.add_argument("--act-only", action="store_true", help="with --sweep/--batch-sweep: only the --act activations")
    ap.add_argument("--batch-sweep", action="store_true",
                    help="extra output: time one MoE FFN layer at T = 1, 4, 16, 64 tokens per step")
    ap.add_argument("--batch-T", default=None, help="with --batch-sweep: comma-separated T values only")
    ap.add_argument("--stack-batch", action="store_true",
                    help="time the 24-layer stack at T = 1, 2, 4, 8, 16 tokens per call (one launch each)")
    ap.add_argument("--latency-probe", action="store_true",
                    help="compile and run the on-chip latency probe (probes/latency_probe.cu) and print its JSON")
    ap.add_argument("--head", action="store_true",
                    help="extra output: time the approximate output head against the full head")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.latency_probe:
        return run_latency_probe(args)
    if args.sweep:
        return run_gemv_sweep(args)
    if args.batch_sweep:
        return run_batch_sweep(args)
    if args.stack_batch:
        return run_stack_batch(args)
    if args.head:
        return run_head(args)

    import torch

    import ternary_weight_moe_b200 as tm
    import synth

    def dev_u16(a, device):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device)

    world, rank, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    act = tm.TERN_ACT_INT8 if args.act == "int8" else tm.TERN_ACT_BF16

    if args.layers != N_LAYERS:
        N_LAYERS = args.layers
        BYTES_PER_TOKEN = N_LAYERS * BYTES_PER_LAYER_TOKEN
    shape, layers, stack = build_stack(dev)
    ws = tm.workspace(tm.moe_stack_workspace_bytes(layers[0], 1, act), dev)
    lay = tm.moe_stack_workspace_layout(layers[0], 1, act)
    launches = tm.moe_stack_kernel_launches(layers[0], N_LAYERS, 1, act)
    K, W = args.steps, args.warmup
    xs_host = synth.tokens_bf16(WID, 70000 + 100000 * rank, K + W, shape.d)
    xs = dev_u16(xs_host, dev)                       # inputs resident in HBM before timing
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    for i in range(W):
        tm.moe_stack_decode(stack, xs[i:i + 1], act=act, ws=ws)
    torch.cuda.synchronize(dev)
    if tm.tern_stream_status() != 0:
        raise RuntimeError("device status set during warm-up")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    trace_t = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_wall0 = time.perf_counter()
        torch.cuda.nvtx.range_push("timed")
        for i in range(K):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            tm.moe_stack_decode(stack, xs[W + i:W + i + 1], act=act, ws=ws)
            ev[i][1].record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(dev)
        t_wall = time.perf_counter() - t_wall0
    if tm.tern_stream_status() != 0:
        raise RuntimeError("device status set during the timed region")
    step_ms = [a.elapsed_time(b) for a, b in ev]
    dev_ms = sum(step_ms)
    # one extra, traced step (outside the timed region): every CTA stamps every phase
    P = max(tm.moe_stack_persistent_ctas(layers[0], N_LAYERS, act), 1)
    os.environ["TERNMOE_TRACE"] = "1"
    flush.fill_(1)
    tm.moe_stack_decode(stack, xs[W:W + 1].clone(), act=act, ws=ws)
    torch.cuda.synchronize(dev)
    os.environ["TERNMOE_TRACE"] = "0"
    tr2 = ws[lay["trace"]:lay["trace"] + 2 * N_LAYERS * P * 24 * 8].view(torch.int64).view(2, N_LAYERS, P, 24).cpu().numpy()
    tr = tr2[0]
    phases = phase_summary(tr, tr2[1]) if launches == 1 else None
    try:
        os.makedirs(OUT_DIR, exist_ok=True)
        np.save(os.path.join(OUT_DIR, f"trace_{args.act}_rank{rank}.npy"), tr2)
    except OSError:
        pass

    # back-to-back throughput without flushes (context)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        tm.moe_stack_decode(stack, xs[W + i:W + i + 1], act=act, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    b2b_ms = e0.elapsed_time(e1)

    # end to end through the public call with host buffers: pinned H2D of the token, the
    # stack, D2H of the result, and a host wait per token (the next token needs it)
    hx = torch.from_numpy(xs_host.view(np.int16)).pin_memory()
    hy = torch.empty_like(hx).pin_memory()
    xd = torch.empty((1, shape.d), dtype=torch.int16, device=dev)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e2.record(stream)
    for i in range(K):
        xd.copy_(hx[W + i:W + i + 1], non_blocking=True)
        tm.moe_stack_decode(stack, xd, act=act, ws=ws)
        hy[W + i:W + i + 1].copy_(xd, non_blocking=True)
        stream.synchronize()
    e3.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e2.elapsed_time(e3)

    dev_ms_max = aggregate(dev_ms, "max", world, dev)
    e2e_ms_max = aggregate(e2e_ms, "max", world, dev)
    b2b_ms_max = aggregate(b2b_ms, "max", world, dev)
    tokens_all = K * world
    value = tokens_all / (dev_ms_max / 1e3)
    peak, peak_kind = peaks()
    avg_launch_ms = dev_ms / K / max(launches, 1)
    achieved = BYTES_PER_TOKEN / launches / (avg_launch_ms * 1e-3) / 1e9
    traffic = kernel_traffic(args.act) if N_LAYERS == 24 else None
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": dev_ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8" if args.act == "int8" else "bf16-in/int-limbs/f64-epilogue", "data": "synthetic",
        "config": dict(_config(args.act, world, "flushed before every timed step (256 MB write, not timed)"),
                       layers=N_LAYERS),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "kernel": f"stack_kernel<{1 if args.act == 'int8' else 3}, 0>",
                     "bytes_per_launch": BYTES_PER_TOKEN // launches, "peak_kind": peak_kind},
        "e2e": {"value": tokens_all / (e2e_ms_max / 1e3), "unit": UNIT, "h2d_bytes_per_step": 2 * shape.d,
                "d2h_bytes_per_step": 2 * shape.d},
        "gpu_launches": int(launches * K),
        "clocks": clk.summary(),
        "back_to_back_tokens_per_s": tokens_all / (b2b_ms_max / 1e3),
        "step_ms_p10_p50_p90": [float(np.percentile(step_ms, q)) for q in (10, 50, 90)],
        "layer_phase_us_traced_step": phases,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and not args.no_cpu_baseline:
        from oracle import ACT_BF16, ACT_INT8

        result["cpu_baseline"] = cpu_baseline(ACT_INT8 if args.act == "int8" else ACT_BF16)
    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
