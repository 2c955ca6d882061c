"""Benchmark of the E8-codebook decode GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (the small-batch decode configuration): one Llama-style linear layer,
W 4096 x 4096 ~ N(0, 0.02^2) (seed 2) quantised at 4 bits per weight (16-bit
index + 16-bit residual index per 8 weights, one global scale), activations
X 16 x 4096 bf16 ~ N(0, 1) (seed 3).  One step is one call of the hot path:
the activation-side Hadamard transform plus the fused decode + tcgen05 GEMM
(E8_GEMM_AUTO picks it for 16 tokens).  The compressed weights were produced
by the GPU encoder beforehand and stay resident; the step rotates over 32
copies of them (32 x 8.4 MB > 126 MB L2) so every step reads its codes from HBM.

Printed (rank 0, one JSON line): whole-job TFLOP/s (2 M N K per step), decoded
weights/s, the roofline of the dominant kernel (HBM bound), an end-to-end
number through the public API with host buffers, the other hot-path rows
(encode, decode to bf16, 1 and 4 tokens) and the CPU oracle timed on this
host as a baseline.  Multi-GPU (torchrun): every rank runs its own layer
(independent weight matrices, no collective on the data path), weak scaling.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "llama_4096_b4"
M_HEAD = 16
ROTATE = 32
GRAPH_STEPS = 1000
METRIC = "fused E8-decode GEMM TFLOP/s & decoded weights/s, as % of HBM/tensor roofline"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ clocks --
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi while running."""

    def __init__(self, index: int, period_ms: int = 100):
        self.index, self.period = index, period_ms
        self.samples = []
        self.proc = None
        self.marks = []

    def start(self):
        cmd = ["nvidia-smi", "-i", str(self.index),
               "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", str(self.period)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 3:
                continue
            try:
                self.samples.append((time.time(), float(parts[0]), float(parts[1]),
                                     int(parts[2], 16)))
            except ValueError:
                pass

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1, fallback_t0=None):
        sel = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if len(sel) < 3 and fallback_t0 is not None:
            sel = [s for s in self.samples if fallback_t0 <= s[0] <= t1]
            window = "timed region and the load phase just before it (same workload)"
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "window": window}
        mask = 0
        for s in sel:
            mask |= s[3]
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": max(s[2] for s in sel),
                "reasons": sorted(v for k, v in _REASONS.items() if mask & k and k != 0x1),
                "samples": len(sel), "window": window}


# ------------------------------------------------------------- distributed --
def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _max_over_ranks(x: float, ws: int, device):
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _rank_layer_seeds(lay, rank: int):
    """(weight seed, RHT seed) of the layer rank `rank` quantises and multiplies:
    rank 0 takes the workload's own seeds, every other rank a distinct layer of
    the same shape (weak scaling: no data-path collective)."""
    return (lay.w_seed if rank == 0 else (lay.w_seed, rank)), lay.rht_seed + 7919 * rank


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# -------------------------------------------------------------- our arm ----
def _graph_of(fn, n, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fn(i)
    return g


def _time_graphs(fn, steps, warmup, stream):
    """Captures fn(i) for i in [0, G) into graphs covering exactly `steps` calls,
    returns elapsed ms of their timed replay.

    Warm-up replays the very graphs that are timed (at least `warmup` calls and
    at least one replay of each graph), so the first launch of a graph, which
    also uploads it to the device, is never inside the timed region."""
    import torch
    G = min(GRAPH_STEPS, max(1, steps))
    full, rem = divmod(steps, G)
    g_full = _graph_of(fn, G, stream)
    g_rem = _graph_of(fn, rem, stream) if rem else None
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-max(1, warmup) // G))):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def run_ours(args):
    import torch
    import decode_gemm_e8_b200 as e8
    from decode_gemm_e8_b200 import build, synth

    ws, rank, local = _dist()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.profile == "decode":
        _profile_decode(e8, dev)
        return
    if args.profile in ("dense_up", "dense_out", "encode", "gemm_mlp", "ep_decode", "grouped"):
        _profile_other(e8, synth, dev, args.profile)
        return
    peaks = _peaks()
    lay = synth.workloads()[WORKLOAD].layers[0]
    N, K, bpw = lay.N, lay.K, lay.bpw
    M = args.M
    cb = e8.Codebook(local)
    # every rank quantises its own layer (weak scaling); rank 0 is the seeded workload
    w_seed, rs = _rank_layer_seeds(lay, rank)
    W = synth.gaussian_weights(N, K, lay.std, w_seed)
    s = synth.suggest_scale(W, bpw)
    Wd = torch.from_numpy(W).to(dev)
    i1, i2 = e8.e8_encode(cb, Wd, bpw, rs, s)
    torch.cuda.synchronize()
    codes = [(i1, i2)] + [(i1.clone(), i2.clone()) for _ in range(ROTATE - 1)]
    Xh = synth.activations_bf16(M, K, synth.workloads()[WORKLOAD].x_seed)
    X = torch.from_numpy(Xh.view(np.int16)).to(dev).view(torch.bfloat16)
    Y = torch.empty((M, N), dtype=torch.float32, device=dev)
    mode = e8.e8_gemm_auto_mode(M, N, K, bpw)
    wsb = torch.empty(max(16, e8.e8_workspace_bytes(mode, M, N, K, bpw)), dtype=torch.uint8,
                      device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i, M=M, X=X, Y=Y, wsb=wsb, mode=mode):
        c1, c2 = codes[i % ROTATE]
        e8.e8_gemm(cb, X, c1, c2, N, K, bpw, rs, s, mode=mode, Y=Y, workspace=wsb, stream=stream)

    if args.profile:
        # a few eager steps of the headline kernel pair, for ncu captures
        for i in range(8):
            step(i)
        torch.cuda.synchronize()
        print("profile steps done", flush=True)
        cb.free()
        return
    sampler = ClockSampler(local)
    if rank == 0:
        sampler.start()
    # load phase right before the timed region, for the clock record only
    t_load = time.time()
    if not args.no_load:
        _time_graphs(step, 20 * GRAPH_STEPS, 0, stream)
    _barrier(ws)
    torch.cuda.synchronize()
    t0 = time.time()
    ms = _time_graphs(step, args.steps, args.warmup, stream)
    t1 = time.time()
    torch.cuda.synchronize()
    _barrier(ws)
    ms = _max_over_ranks(ms, ws, dev)
    clocks = sampler.summary(t0, t1, fallback_t0=t_load) if rank == 0 else None

    flop_step = 2.0 * M * N * K
    sec = ms / 1e3
    value = flop_step * args.steps * ws / sec / 1e12
    step_us = ms * 1e3 / args.steps
    code_bytes = N * K * bpw // 8
    alg_bytes = code_bytes + M * K * 2 + M * N * 4

    # dominant kernel alone: fused decode-GEMM on pre-transformed activations
    xq = e8.e8_act_rht_q8(X, rs)

    def gemm_only(i, M=M, xq=xq, Y=Y):
        c1, c2 = codes[i % ROTATE]
        e8.e8_gemm_xt(cb, xq, M, c1, c2, N, K, bpw, s, Y=Y, stream=stream)

    kern_steps = min(args.steps, 20 * GRAPH_STEPS)
    k_ms = _time_graphs(gemm_only, kern_steps, args.warmup, stream)
    k_us = k_ms * 1e3 / kern_steps
    achieved = alg_bytes / (k_us * 1e-6) / 1e9

    def rht_only(i, X=X, xq=xq):
        e8.e8_act_rht_q8(X, rs, out=xq, stream=stream)

    r_ms = _time_graphs(rht_only, kern_steps, args.warmup, stream)
    rht_us = r_ms * 1e3 / kern_steps

    # end to end through the public API with host buffers: every step copies its
    # input in from pinned host memory and its result out to pinned host memory;
    # two buffer slots on two streams let one step's copies overlap the other's
    # kernels, as a serving loop would
    streams = [stream, torch.cuda.Stream(device=dev)]
    Xpin = [torch.from_numpy(Xh.view(np.int16)).view(torch.bfloat16).pin_memory() for _ in range(2)]
    Ypin = [torch.empty((M, N), dtype=torch.float32).pin_memory() for _ in range(2)]
    wse = [torch.empty(e8.e8_gemm_host_workspace_bytes(mode, M, N, K, bpw), dtype=torch.uint8,
                       device=dev) for _ in range(2)]

    def e2e_step(i):
        # one library call: X copied in from pinned host memory, the product,
        # Y copied back to pinned host memory
        k = i & 1
        c1, c2 = codes[i % ROTATE]
        e8.e8_gemm_host(cb, Xpin[k], c1, c2, N, K, bpw, rs, s, Y_host=Ypin[k], mode=mode,
                        workspace=wse[k], stream=streams[k])

    e2e_steps = min(args.steps, 2000)
    for i in range(max(4, min(args.warmup, 50))):
        e2e_step(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(streams[0])
    streams[1].wait_event(a)
    for i in range(e2e_steps):
        e2e_step(i)
    done1 = torch.cuda.Event()
    done1.record(streams[1])
    streams[0].wait_event(done1)
    b.record(streams[0])
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(a.elapsed_time(b), ws, dev)
    e2e_val = flop_step * e2e_steps * ws / (e2e_ms / 1e3) / 1e12

    rows_out = {}
    if rank == 0 and not args.quick:
        rows_out = _other_rows(e8, synth, cb, Wd, W, codes, X, N, K, bpw, rs, s, dev, stream, args,
                               peaks)
    if rank == 0:
        launches = 2 * args.steps
        traffic = _traffic_from_profile()
        out = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": "TFLOP/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": step_us / 1e3,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "i8",
            "dtype_detail": "tcgen05 kind::i8: activations as two int8 pieces per element on a "
                            "per-token step (xt = s (q0 + q1/128), error <= s/256), weights as the "
                            "exact integers z + 128 (unsigned bytes), int32 accumulation, fp32 "
                            "epilogue and output",
            "data": "synthetic",
            "config": {
                "workload": "%s: W %dx%d N(0,%.2f^2) seed %d, %d bpw, X %dx%d bf16 N(0,1) seed %d"
                            % (WORKLOAD, N, K, lay.std, lay.w_seed, bpw, M, K,
                               synth.workloads()[WORKLOAD].x_seed),
                "M": M, "N": N, "K": K, "bpw": bpw,
                "gemm_mode": "act_rht: int8 activation pieces, codes decoded into tensor memory, "
                             "tcgen05 kind::i8",
                "l2": "inputs larger than L2: %d rotating code sets, %.0f MB" %
                      (ROTATE, ROTATE * code_bytes / 1e6),
                "launch": "CUDA graphs of %d steps" % GRAPH_STEPS,
                "parallelism": "independent layer per GPU" if ws > 1 else "single GPU",
            },
            "decoded_weights_per_s": N * K * args.steps * ws / sec,
            "roofline": {
                "bound": "hbm",
                "kernel": "k_gemm_q8 (fused decode + tcgen05 GEMM, stream-K over all SMs)",
                "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"],
                "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic,
                "algorithmic_bytes": alg_bytes,
                "kernel_us": round(k_us, 3),
                "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)",
                "step_frac": round(alg_bytes / (step_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                "act_rht_us": round(rht_us, 3),
            },
            "e2e": {"value": round(e2e_val, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 4,
                    "steps": e2e_steps,
                    "path": "e8_gemm_host: pinned host X -> device -> product -> pinned host Y "
                            "in one library call per step, two buffer slots on two streams"},
            "gpu_launches": launches,
            "clocks": clocks,
            "rows": rows_out,
        }
        if not args.no_cpu:
            out["cpu_baseline"] = _cpu_baseline(M)
        sampler.stop()
        print(json.dumps(out), flush=True)
    cb.free()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _traffic_from_profile():
    """DRAM bytes per launch of k_gemm_q8 from the committed ncu summary, or None
    when the kernel source changed since the counters were taken."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", "k_gemm_q8_llama4096_m16.md")
    src = os.path.join(ROOT, "decode_gemm_e8_b200", "csrc", "e8_gemm_q8.cu")
    if not os.path.exists(prof):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    text = open(prof).read()
    import re
    m_h = re.search(r"source sha256\[:16\]: ([0-9a-f]{16})", text)
    m_t = re.search(r"dram bytes per launch: ([0-9]+)", text)
    if not m_h or not m_t or m_h.group(1) != h:
        return None
    return int(m_t.group(1))


def _profile_decode(e8, dev):
    """Three bf16 decodes of a 14336 x 4096 matrix at 4 bpw (about 150 MB on the
    device, more than L2), for ncu captures of the tensor-core decoder."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    N, K, bpw = 14336, 4096, 4
    c1, c2 = _random_codes(torch, dev, N, K, bpw, gen)
    cb = e8.Codebook(dev.index)
    out = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        e8.e8_decode_to_bf16(cb, c1, c2, N, K, bpw, 7, 0.02, out=out)
    torch.cuda.synchronize()
    if e8.e8_sync_status(cb) != 0:
        raise RuntimeError("decoder reported a device error")
    print("profile decodes done", flush=True)
    cb.free()


def _profile_other(e8, synth, dev, mode):
    """Small workloads for ncu captures of one kernel each (a few hundred MB on
    the device at most):
      dense_up   prefill GEMM of the MLP up-projection (14336 x 4096, 3 bpw,
                 4096 tokens): decode to bf16, then k_dense_gemm, twice
      dense_out  the same for the DiT out projection (3072 x 3072, 4 bpw)
      encode     two encodes of the 4096 x 4096 Llama layer at 4 bpw
      gemm_mlp   three small-batch products (16 tokens) of a 14336 x 4096
                 matrix at 4 bpw on pre-transformed activations (k_gemm_q8)
      ep_decode  the entropy-coded variant: three decodes of a 14336 x 4096
                 Gaussian matrix at delta 0.075 (about 4 bpp)
      grouped    three grouped small-batch calls (e8_gemm_grouped) of the q, k,
                 v projections of a Llama-3-8B layer (4096, 1024, 1024 rows x
                 4096, 4 bpw, 16 tokens): one transform and one GEMM launch each"""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)
    cb = e8.Codebook(dev.index)
    if mode.startswith("dense"):
        M, N, K, bpw = (4096, 14336, 4096, 3) if mode == "dense_up" else (4096, 3072, 3072, 4)
        c1, c2 = _random_codes(torch, dev, N, K, bpw, gen)
        X = torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16)
        ws = torch.empty(e8.e8_workspace_bytes(e8.E8_GEMM_DECODED_W, M, N, K, bpw),
                         dtype=torch.uint8, device=dev)
        for _ in range(2):
            e8.e8_gemm(cb, X, c1, c2, N, K, bpw, 1, 0.02, mode=e8.E8_GEMM_DECODED_W, workspace=ws)
    elif mode == "grouped":
        K, bpw, M = 4096, 4, 16
        items = []
        for j, N in enumerate((4096, 1024, 1024)):
            c1, c2 = _random_codes(torch, dev, N, K, bpw, gen)
            items.append((c1, c2, N, 100 + j, 0.02))
        X = torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16)
        ws = torch.empty(e8.e8_gemm_grouped_workspace_bytes(M, K, bpw, len(items)),
                         dtype=torch.uint8, device=dev)
        for _ in range(3):
            e8.e8_gemm_grouped(cb, X, items, K, bpw, workspace=ws)
    elif mode == "ep_decode":
        W = torch.from_numpy(synth.gaussian_weights(14336, 4096, 0.02, 4)).to(dev)
        m = e8.e8_ep_encode(cb, W, 0.075)
        out = torch.empty((14336, 4096), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            e8.e8_ep_decode_to_bf16(cb, m, out=out)
    elif mode == "encode":
        lay = synth.workloads()[WORKLOAD].layers[0]
        W = synth.gaussian_weights(lay.N, lay.K, lay.std, lay.w_seed)
        s = synth.suggest_scale(W, lay.bpw)
        Wd = torch.from_numpy(W).to(dev)
        ws = torch.empty(e8.e8_workspace_bytes(e8.E8_OP_ENCODE, 0, lay.N, lay.K, lay.bpw),
                         dtype=torch.uint8, device=dev)
        for _ in range(2):
            e8.e8_encode(cb, Wd, lay.bpw, lay.rht_seed, s, workspace=ws)
            cnt = ws[:16].view(torch.int32).cpu().tolist()
            print("encode %dx%d at %d bpw: %d groups; fast path left %d open, brute force "
                  "took %d, second round %d / %d" % (lay.N, lay.K, lay.bpw, lay.N * lay.K // 8,
                                                     cnt[0], cnt[1], cnt[2], cnt[3]))
    else:
        M, N, K, bpw = 16, 14336, 4096, 4
        codes = [_random_codes(torch, dev, N, K, bpw, gen) for _ in range(3)]
        X = torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16)
        xq = e8.e8_act_rht_q8(X, 2)
        Y = torch.zeros((M, N), device=dev)
        for c1, c2 in codes:
            e8.e8_gemm_xt(cb, xq, M, c1, c2, N, K, bpw, 0.02, Y=Y)
    torch.cuda.synchronize()
    if e8.e8_sync_status(cb) != 0:
        raise RuntimeError("a kernel reported a device error")
    print("profile %s done" % mode, flush=True)
    cb.free()


def _random_codes(torch, dev, N, K, bpw, gen):
    """Uniform random indices of the given rate (decode cost does not depend on
    which entries are chosen beyond shared-memory bank spread)."""
    c1 = torch.randint(0, 65536, (N, K // 8), dtype=torch.int32, device=dev,
                       generator=gen).to(torch.uint16)
    c2 = None
    if bpw == 4:
        c2 = torch.randint(0, 65536, (N, K // 8), dtype=torch.int32, device=dev,
                           generator=gen).to(torch.uint16)
    elif bpw == 3:
        c2 = torch.randint(0, 256, (N, K // 8), dtype=torch.int32, device=dev,
                           generator=gen).to(torch.uint8)
    return c1, c2


def _prefill_rows(e8, synth, cb, dev, stream, peaks):
    """Prefill-sized fused decode GEMM (decode to a bf16 workspace + tcgen05 GEMM)
    on the MLP up-projection and the four DiT block linears, 4096 tokens."""
    import torch
    rows = {}
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    cases = [("mlp_up_14336_b3", synth.workloads()["mlp_up_14336_b3"].layers[0], 4096, 5)]
    for lay in synth.workloads()["dit_3072_b4"].layers:
        cases.append(("dit_3072_b4." + lay.name, lay, 4096, 10))
    for name, lay, M, xseed in cases:
        N, K, bpw = lay.N, lay.K, lay.bpw
        codes = [_random_codes(torch, dev, N, K, bpw, gen) for _ in range(2)]
        Xh = synth.activations_bf16(M, K, xseed)
        X = torch.from_numpy(Xh.view(np.int16)).to(dev).view(torch.bfloat16)
        Y = torch.empty((M, N), dtype=torch.float32, device=dev)
        ws = torch.empty(e8.e8_workspace_bytes(e8.E8_GEMM_DECODED_W, M, N, K, bpw),
                         dtype=torch.uint8, device=dev)

        def g(i, X=X, Y=Y, ws=ws, codes=codes, N=N, K=K, bpw=bpw):
            c1, c2 = codes[i % 2]
            e8.e8_gemm(cb, X, c1, c2, N, K, bpw, 1, 0.02, mode=e8.E8_GEMM_DECODED_W, Y=Y,
                       workspace=ws, stream=stream)

        n = 20
        t = _time_graphs(g, n, 4, stream) / 1e3 / n
        flop = 2.0 * M * N * K
        byt = N * K * bpw / 8 + M * K * 2 + M * N * 4
        roof = max(flop / (peaks["bf16_tflops"] * 1e12), byt / (peaks["hbm_gbs"] * 1e9))
        rows["prefill_" + name] = {"TFLOP_s": round(flop / t / 1e12, 1), "us": round(t * 1e6, 1),
                                   "M": M, "N": N, "K": K, "bpw": bpw,
                                   "roofline_frac": round(roof / t, 4),
                                   "bound": "tensor" if flop / (peaks["bf16_tflops"] * 1e12) >=
                                   byt / (peaks["hbm_gbs"] * 1e9) else "hbm"}
        del codes, X, Y, ws
    return rows


def _ep_rows(e8, synth, cb, dev, stream, peaks):
    """Entropy-coded variant at a 4 bpp target on the DiT out projection
    (3072 x 3072, Student-t with outlier columns) and the MLP up-projection
    (14336 x 4096, Gaussian): the step the rate search picks, the actual rate
    with metadata, the decode to bf16 (stream read + 2 bytes written per
    weight) and the prefill GEMM on 4096 tokens (decode included)."""
    import torch
    rows = {}
    for name, N, K, W in (("dit_3072_out", 3072, 3072, synth.student_t_outlier_weights(3072, 3072, 7)),
                          ("mlp_up_14336", 14336, 4096,
                           synth.gaussian_weights(14336, 4096, 0.015, 4))):
        Wd = torch.from_numpy(W).to(dev)
        d = e8.e8_ep_choose_delta(cb, Wd, 4.0)
        m = e8.e8_ep_encode(cb, Wd, d)
        outs = [torch.empty((N, K), dtype=torch.bfloat16, device=dev) for _ in range(4)]

        def dec(i, m=m, outs=outs):
            e8.e8_ep_decode_to_bf16(cb, m, out=outs[i % 4], stream=stream)

        n = 20
        t = _time_graphs(dec, n, 4, stream) / 1e3 / n
        byt = m.total_words * 2 + N * K * 2
        M = 4096
        X = torch.from_numpy(synth.activations_bf16(M, K, 11).view(np.int16)).to(dev).view(
            torch.bfloat16)
        Y = torch.empty((M, N), dtype=torch.float32, device=dev)
        ws = torch.empty(e8.load_library().e8_ep_gemm_workspace_bytes(M, N, K), dtype=torch.uint8,
                         device=dev)

        def gem(i, m=m, X=X, Y=Y, ws=ws):
            e8.e8_ep_gemm(cb, X, m, Y=Y, workspace=ws, stream=stream)

        tg = _time_graphs(gem, 10, 3, stream) / 1e3 / 10
        flop = 2.0 * M * N * K
        rows["ep_" + name + "_4bpp"] = {
            "delta": d, "actual_bpp": round(m.actual_bpp(), 4),
            "decode_us": round(t * 1e6, 1), "decode_GB_s": round(byt / t / 1e9, 1),
            "decode_hbm_frac": round(byt / t / 1e9 / peaks["hbm_gbs"], 4),
            "prefill_TFLOP_s": round(flop / tg / 1e12, 1), "prefill_us": round(tg * 1e6, 1),
            "prefill_frac": round(flop / tg / 1e12 / peaks["bf16_tflops"], 4)}
        del Wd, m, outs, X, Y, ws
    return rows


def _decode_sweep_rows(e8, synth, cb, dev, stream, peaks):
    """Decode to bf16 of one Llama-3-8B-shaped decoder layer (7 matrices) per rate;
    the 32-layer figure is 32 times the layer."""
    import torch
    rows = {}
    gen = torch.Generator(device=dev)
    gen.manual_seed(100)
    for bpw in (2, 3, 4):
        mats = synth.workloads()["llama3_8b_x32_b%d" % bpw].layers[:7]
        data = []
        for lay in mats:
            codes = [_random_codes(torch, dev, lay.N, lay.K, bpw, gen) for _ in range(2)]
            outs = [torch.empty((lay.N, lay.K), dtype=torch.bfloat16, device=dev)
                    for _ in range(2)]
            data.append((lay, codes, outs))

        def d(i, data=data, bpw=bpw):
            for lay, codes, outs in data:
                c1, c2 = codes[i % 2]
                e8.e8_decode_to_bf16(cb, c1, c2, lay.N, lay.K, bpw, lay.rht_seed, 0.02,
                                     out=outs[i % 2], stream=stream)

        n = 10
        t = _time_graphs(d, n, 2, stream) / 1e3 / n
        nw = sum(lay.N * lay.K for lay in mats)
        byt = nw * (2 + bpw / 8)
        rows["decode_llama3_8b_layer_b%d" % bpw] = {
            "weights_per_s": nw / t, "us_per_layer": round(t * 1e6, 1),
            "ms_32_layers": round(32 * t * 1e3, 3), "GB_s": round(byt / t / 1e9, 1),
            "hbm_frac": round(byt / t / 1e9 / peaks["hbm_gbs"], 4)}
        del data
        rows["encode_llama3_8b_layer_b%d" % bpw] = _encode_layer_row(e8, synth, cb, dev, stream,
                                                                      mats, bpw)
    return rows


def _encode_layer_row(e8, synth, cb, dev, stream, mats, bpw):
    """Batched RHT + exact nearest-point encode of the 7 matrices of one
    Llama-3-8B-shaped layer (weights N(0, 0.02^2) drawn on the device, one scale
    per matrix from its rms); the 32-layer figure is 32 times the layer."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(200 + bpw)
    total_s = 0.0
    nw = 0
    for lay in mats:
        W = torch.randn((lay.N, lay.K), generator=gen, device=dev, dtype=torch.float32) * lay.std
        rms = float(torch.sqrt(torch.mean(W.double() ** 2)))
        s = float(np.float32(rms / synth.SIGMA_T[bpw]))
        i1 = torch.empty((lay.N, lay.K // 8), dtype=torch.uint16, device=dev)
        i2 = (torch.empty((lay.N, lay.K // 8), dtype=torch.uint8 if bpw == 3 else torch.uint16,
                          device=dev) if bpw > 2 else None)
        wsz = e8.e8_workspace_bytes(e8.E8_OP_ENCODE, 0, lay.N, lay.K, bpw)
        ws = torch.empty(max(16, wsz), dtype=torch.uint8, device=dev)
        e8.e8_encode(cb, W, bpw, lay.rht_seed, s, idx1=i1, idx2=i2, workspace=ws, stream=stream)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e8.e8_encode(cb, W, bpw, lay.rht_seed, s, idx1=i1, idx2=i2, workspace=ws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        total_s += a.elapsed_time(b) / 1e3
        nw += lay.N * lay.K
        del W, i1, i2, ws
    byt = nw * (4 + bpw / 8)
    return {"weights_per_s": nw / total_s, "ms_per_layer": round(total_s * 1e3, 2),
            "s_32_layers": round(32 * total_s, 2), "GB_s": round(byt / total_s / 1e9, 2),
            "hbm_frac": round(byt / total_s / 1e9 / _peaks()["hbm_gbs"], 5)}


def _layer_chain_rows(e8, synth, cb, dev, stream, peaks, M=16):
    """The seven projections of one Llama-3-8B-shaped decoder layer (q, k, v, o,
    gate, up, down) through the fused small-batch decode GEMM, back to back in one
    stream (programmatic dependent launch between the calls), M tokens, per rate;
    two code sets alternate so more than L2 streams from HBM.  Timed twice: seven
    single-matrix calls, and four calls with q, k, v and gate, up grouped
    (e8_gemm_grouped: the matrices of a group read the same tokens)."""
    import torch
    rows = {}
    gen = torch.Generator(device=dev)
    gen.manual_seed(300)
    for bpw in (2, 3, 4):
        mats = synth.workloads()["llama3_8b_x32_b%d" % bpw].layers[:7]
        data = []
        for lay in mats:
            codes = [_random_codes(torch, dev, lay.N, lay.K, bpw, gen) for _ in range(2)]
            X = (torch.randn((M, lay.K), generator=gen, device=dev)).to(torch.bfloat16)
            Y = torch.empty((M, lay.N), dtype=torch.float32, device=dev)
            wsz = e8.e8_workspace_bytes(e8.E8_GEMM_ACT_RHT, M, lay.N, lay.K, bpw)
            ws = torch.empty(max(16, wsz), dtype=torch.uint8, device=dev)
            data.append((lay, codes, X, Y, ws))

        def chain(i, data=data, bpw=bpw):
            for lay, codes, X, Y, ws in data:
                c1, c2 = codes[i % 2]
                e8.e8_gemm(cb, X, c1, c2, lay.N, lay.K, bpw, lay.rht_seed, 0.02,
                           mode=e8.E8_GEMM_ACT_RHT, Y=Y, workspace=ws, stream=stream)

        # the same layer with the matrices that read the same tokens grouped:
        # (q, k, v), o, (gate, up), down -- four calls instead of seven
        groups = [[0, 1, 2], [3], [4, 5], [6]]
        gws = [torch.empty(max(16, e8.e8_gemm_grouped_workspace_bytes(M, mats[g[0]].K, bpw,
                                                                      len(g))),
                           dtype=torch.uint8, device=dev) for g in groups]

        def chain_grouped(i, data=data, bpw=bpw, groups=groups, gws=gws):
            for g, ws in zip(groups, gws):
                X = data[g[0]][2]
                items = []
                for j in g:
                    lay, codes, _, Y, _ = data[j]
                    c1, c2 = codes[i % 2]
                    items.append((c1, c2, lay.N, lay.rht_seed, 0.02, Y))
                e8.e8_gemm_grouped(cb, X, items, mats[g[0]].K, bpw, workspace=ws, stream=stream)

        n = 200
        nw = sum(lay.N * lay.K for lay in mats)
        flop = sum(2.0 * M * lay.N * lay.K for lay in mats)
        byt = sum(lay.N * lay.K * bpw / 8 + M * lay.K * 2 + M * lay.N * 4 for lay in mats)
        for name, fn in (("gemm_llama3_8b_layer_m%d_b%d" % (M, bpw), chain),
                         ("gemm_llama3_8b_layer_m%d_b%d_grouped" % (M, bpw), chain_grouped)):
            t = _time_graphs(fn, n, 4, stream) / 1e3 / n
            rows[name] = {
                "us_per_layer": round(t * 1e6, 1), "TFLOP_s": round(flop / t / 1e12, 2),
                "decoded_weights_per_s": nw / t, "GB_s": round(byt / t / 1e9, 1),
                "hbm_frac": round(byt / t / 1e9 / peaks["hbm_gbs"], 4)}
        del data, gws
    return rows


def _other_rows(e8, synth, cb, Wd, W, codes, X, N, K, bpw, rs, s, dev, stream, args, peaks):
    """Encode, decode-to-bf16 and the 1- and 4-token GEMM on the same layer."""
    import torch
    rows = {}
    reps = 4
    # encode: rotate over copies of W so the 64 MB matrix is read from HBM
    Ws = [Wd] + [Wd.clone() for _ in range(reps - 1)]
    wsb = torch.empty(e8.e8_workspace_bytes(e8.E8_OP_ENCODE, 0, N, K, bpw), dtype=torch.uint8,
                      device=dev)
    i1 = torch.empty((N, K // 8), dtype=torch.uint16, device=dev)
    i2 = torch.empty((N, K // 8), dtype=torch.uint16, device=dev)
    n_enc = 8

    def enc(i):
        e8.e8_encode(cb, Ws[i % reps], bpw, rs, s, idx1=i1, idx2=i2, workspace=wsb, stream=stream)

    ms = _time_graphs(enc, n_enc, 2, stream)
    t = ms / 1e3 / n_enc
    byt = N * K * (4 + bpw / 8)
    cnt = wsb[:16].view(torch.int32).cpu().tolist()   # documented counters of e8_encode
    rows["encode"] = {"weights_per_s": N * K / t, "ms": t * 1e3, "GB_s": byt / t / 1e9,
                      "hbm_frac": round(byt / t / 1e9 / peaks["hbm_gbs"], 4),
                      "bytes_per_weight": 4 + bpw / 8, "groups": N * K // 8,
                      "groups_class_search": cnt[0], "groups_brute_force": cnt[1],
                      "groups_second_round": [cnt[2], cnt[3]]}
    # four outputs (134 MB) so that the written weights leave the L2 cache
    outs = [torch.empty((N, K), dtype=torch.bfloat16, device=dev) for _ in range(4)]

    def dec(i):
        c1, c2 = codes[i % len(codes)]
        e8.e8_decode_to_bf16(cb, c1, c2, N, K, bpw, rs, s, out=outs[i % 4], stream=stream)

    ms = _time_graphs(dec, 200, 10, stream)
    t = ms / 1e3 / 200
    byt = N * K * (2 + bpw / 8)
    rows["decode_to_bf16"] = {"weights_per_s": N * K / t, "us": t * 1e6, "GB_s": byt / t / 1e9,
                              "hbm_frac": round(byt / t / 1e9 / peaks["hbm_gbs"], 4),
                              "bytes_per_weight": 2 + bpw / 8}
    rows.update(_prefill_rows(e8, synth, cb, dev, stream, peaks))
    rows.update(_ep_rows(e8, synth, cb, dev, stream, peaks))
    rows.update(_decode_sweep_rows(e8, synth, cb, dev, stream, peaks))
    rows.update(_layer_chain_rows(e8, synth, cb, dev, stream, peaks))
    for Mx in (1, 4):
        Xm = X[:Mx].contiguous()
        Ym = torch.empty((Mx, N), dtype=torch.float32, device=dev)
        mode = e8.e8_gemm_auto_mode(Mx, N, K, bpw)
        wsm = torch.empty(max(16, e8.e8_workspace_bytes(mode, Mx, N, K, bpw)), dtype=torch.uint8,
                          device=dev)

        def g(i, Xm=Xm, Ym=Ym, wsm=wsm, mode=mode):
            c1, c2 = codes[i % len(codes)]
            e8.e8_gemm(cb, Xm, c1, c2, N, K, bpw, rs, s, mode=mode, Y=Ym, workspace=wsm,
                       stream=stream)

        ms = _time_graphs(g, 2000, 100, stream)
        t = ms / 1e3 / 2000
        byt = N * K * bpw // 8 + Mx * K * 2 + Mx * N * 4
        rows["gemm_m%d" % Mx] = {"TFLOP_s": 2.0 * Mx * N * K / t / 1e12, "us": t * 1e6,
                                 "hbm_frac": round(byt / t / 1e9 / peaks["hbm_gbs"], 4)}
    return rows


def _cpu_baseline(M):
    """The CPU oracle (decode + binary64 GEMM) on the same workload, this host's cores."""
    from decode_gemm_e8_b200 import synth
    from oracle import oracle as orc
    lay = synth.workloads()[WORKLOAD].layers[0]
    N, K, bpw = lay.N, lay.K, lay.bpw
    rng = np.random.default_rng(0)
    i1 = rng.integers(0, 65536, (N, K // 8)).astype(np.uint16)
    i2 = rng.integers(0, 65536, (N, K // 8)).astype(np.uint16)
    X = synth.activations_bf16(M, K, synth.workloads()[WORKLOAD].x_seed)
    threads = orc.threads()
    t0 = time.perf_counter()
    n = 0
    while True:
        wd = orc.decode(i1, i2, N, K, bpw, lay.rht_seed, 0.02)
        orc.gemm(X, wd)
        n += 1
        if time.perf_counter() - t0 > 10.0:
            break
    dt = (time.perf_counter() - t0) / n
    return {"value": 2.0 * M * N * K / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": "whole step of the workload (decode 4096x4096 at 4 bpw + binary64 GEMM with "
                      "%d rows), repeated %d times over %.1f s; codes random" % (M, n, dt * n)}


# -------------------------------------------------------- reference arm ----
def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    from decode_gemm_e8_b200 import synth
    from oracle import oracle as orc
    lay = synth.workloads()[WORKLOAD].layers[0]
    N, K, bpw, M = lay.N, lay.K, lay.bpw, args.M
    rng = np.random.default_rng(0)
    i1 = rng.integers(0, 65536, (N, K // 8)).astype(np.uint16)
    i2 = rng.integers(0, 65536, (N, K // 8)).astype(np.uint16)
    X = synth.activations_bf16(M, K, synth.workloads()[WORKLOAD].x_seed)
    # bounded sample: each step decodes and multiplies a slice of the rows
    rows = max(64, min(N, 4096))
    steps, warm = min(args.steps, 20), min(args.warmup, 3)

    def one():
        wd = orc.decode(i1[:rows], i2[:rows], rows, K, bpw, lay.rht_seed, 0.02)
        orc.gemm(X, wd)

    for _ in range(warm):
        one()
    t0 = time.perf_counter()
    for _ in range(steps):
        one()
    dt = (time.perf_counter() - t0) / steps
    v = 2.0 * M * rows * K / dt / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": ws,
           "steps": steps, "warmup": warm, "ms_per_step": dt * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "%s: decode %dx%d at %d bpw + GEMM with %d tokens" %
                                  (WORKLOAD, rows, K, bpw, M), "M": M, "N": rows, "K": K},
           "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": orc.threads(),
                            "kind": "oracle", "sample": "%d weight rows per step" % rows},
           "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--M", type=int, default=M_HEAD)
    ap.add_argument("--quick", action="store_true", help="skip the extra rows")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-load", action="store_true",
                    help="skip the load phase that precedes the timed region (clock record)")
    ap.add_argument("--profile", nargs="?", const="gemm",
                    choices=["gemm", "decode", "dense_up", "dense_out", "encode", "gemm_mlp",
                             "ep_decode", "grouped"],
                    help="small runs for ncu captures, then exit: 8 eager steps of the "
                         "headline call (gemm), 3 bf16 decodes of a 14336 x 4096 matrix "
                         "(decode), prefill GEMMs (dense_up, dense_out), two encodes "
                         "(encode), small-batch products of a 14336 x 4096 matrix (gemm_mlp)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
