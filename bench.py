"""Benchmark: single-token MoE layer decode on B200 through the C-ABI engine.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fmoe|reference] [--config full4|full2|tiny|stacked|batch16|deltanet]

One step = one token decoded through one full MoE layer (router GEMV over 512
experts, softmax/top-4/renormalise, 4 routed + 1 shared 4-bit experts, fused
combine) with the weights resident in HBM.  The default workload is the
full-size 4-bit layer: hidden 4096, expert intermediate 1024, 512 experts,
group 64 (3.6 GB of experts per layer, 39.6 MB read per decode).

Timing: W untimed warm-up steps; then K steps timed with CUDA events on the
launching stream, bracketed by a barrier and a device synchronise.  Step j
decodes token j mod 64 of a pre-drawn pool through layer instance j mod L
(L = 16 distinct full-size layers, 58 GB of experts): the weights a step reads
are never L2-resident (inputs larger than L2, no flush between steps).  The
steps are the library's decode call captured in CUDA graphs of 64 steps, so
the timed region is device time plus the gaps between back-to-back kernels,
not Python launch latency (the end-to-end figure keeps that).  The value is
the total over all ranks divided by the slowest rank's time.  With --gpus
N > 1 (torchrun) every rank decodes its own replicas: the path has no
data-path exchange.

`--config deltanet` times the other decode step instead: one token through
one 64-head x 128x128 gated delta-rule state (45 states in rotation, 180 MiB),
with the same timing rules and JSON keys.

The JSON line also carries: the latency of one isolated step after a 256 MiB
L2 flush; the roofline of the layer kernel (algorithmic bytes per launch /
measured time per launch vs the measured HBM copy bandwidth); an
end-to-end figure through the same C-ABI call with host buffers (pinned host
-> device copy of x and residual, decode, device -> host copy of out inside
the event pair), the SM clocks sampled during the timed region, and the CPU
oracle timed on a bounded sample as a baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth as S  # noqa: E402

CONFIGS = {
    "full4": dict(workload="full_h4096_i1024_e512_k4_shared_4bit", hidden=4096, inter=1024, experts=512,
                  top_k=4, bits=4, shared_bits=4),
    "full2": dict(workload="full_h4096_i1024_e512_k4_routed2bit_shared4bit", hidden=4096, inter=1024,
                  experts=512, top_k=4, bits=2, shared_bits=4),
    "tiny": dict(workload="tiny_h512_i128_e16_k4_shared_4bit", hidden=512, inter=128, experts=16, top_k=4,
                 bits=4, shared_bits=4),
    # 40 independent full-size 4-bit layers (145.6 GB of experts); a step is one
    # token decoded through all 40 layers, each normalising its input.
    "stacked": dict(workload="stacked_40x_full_h4096_i1024_e512_k4_shared_4bit", hidden=4096, inter=1024,
                    experts=512, top_k=4, bits=4, shared_bits=4, layers_per_step=40),
    # The linear-attention state update: one token through one layer's
    # 64-head x 128x128 gated delta-rule state (45 such layers in rotation).
    "deltanet": dict(workload="gated_delta_h64_dk128_dv128", kind="deltanet", heads=64, dk=128, dv=128,
                     layers=45),
    # Routed experts streamed from pinned host memory (the pages' SSD expert
    # streaming): 2 full-size 4-bit layers whose 1024 routed experts (7.25 GB)
    # stay on the host, device slot caches of several sizes, one token of an
    # autoregressive stream (rho 0.9) decoded through both layers per step.
    "stream": dict(workload="stream_2x_full_h4096_i1024_e512_k4_shared_4bit_host_experts", kind="stream",
                   hidden=4096, inter=1024, experts=512, top_k=4, bits=4, shared_bits=4, stream_layers=2,
                   slot_counts=[128, 512, 1024], default_slots=512, rho=0.9),
    # 16 tokens per step through the full-size 4-bit layer, grouped by expert.
    "batch16": dict(workload="batch16_full_h4096_i1024_e512_k4_shared_4bit", hidden=4096, inter=1024,
                    experts=512, top_k=4, bits=4, shared_bits=4, tokens=16),
}
METRIC = "MoE layer decodes/s (batch 1)"
DELTA_METRIC = "GatedDeltaNet state updates/s (64 heads x 128x128, one token, batch 1)"
UNIT = "decodes/s"
SEED = 2026
POOL = 64
FLUSH_BYTES = 256 << 20


def expert_bytes(h, i, b):
    return 3 * h * i * b // 8 + 3 * h * i // 64 * 4


def algorithmic_bytes(cfg, distinct_routed: float | None = None) -> dict:
    """Bytes one decode step must read or write at least (each weight once).

    With several tokens per step, the routed experts are counted once per
    distinct expert the step selects (`distinct_routed`, measured).
    """
    h, i, e, k = cfg["hidden"], cfg["inter"], cfg["experts"], cfg["top_k"]
    tt = cfg.get("tokens", 1)
    n_routed = k if distinct_routed is None else distinct_routed
    experts = n_routed * expert_bytes(h, i, cfg["bits"]) + expert_bytes(h, i, cfg["shared_bits"])
    router = e * h * 2 + h * 2
    vectors = 3 * tt * h * 4  # x, residual in; out
    return dict(experts=experts, router=router, vectors=vectors, total=experts + router + vectors)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# Device sources the single-token layer kernel is compiled from (its DRAM
# traffic depends on nothing else).
LAYER_KERNEL_SOURCES = ("common.cuh", "dequant.cuh", "layer_kernel.cuh")


def source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_expert_router_b200", "csrc")
    for f in LAYER_KERNEL_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(cfg_name: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernel source."""
    p = os.path.join(ROOT, "profiles", f"layer_kernel_{cfg_name}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != source_hash():
        return None
    return d.get("dram_bytes_per_launch")


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise maximum of per-rank values; every rank gets the result."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units all ranks processed divided by the slowest rank's time (per second)."""
    return world * units_per_rank / (max_ms / 1000.0)


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
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smmax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smmax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smmax) if smmax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CPU oracle leg (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------

REF_WARMUP_S = 30.0   # the reference arm's warm-up stops after this much host time
REF_BUDGET_S = 120.0  # and its timed steps after this much


def host_cpu_model() -> str:
    """The host CPU's model name (first processor in /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        return 1


def oracle_prepare(cfg):
    """Draw the oracle's inputs for the layer workload once (untimed input
    preparation) and return decode(t): one single-token decode of pool token t."""
    import oracle as O
    h, i, e, k = cfg["hidden"], cfg["inter"], cfg["experts"], cfg["top_k"]
    w_router = S.router_bf16(SEED, 0, e, h)
    w_sg = S.sgate_bf16(SEED, 0, h)

    def blob(ex, bits):
        return O.assemble_blob(S.expert_parts(SEED, 0, ex, h, i, bits), h, i, bits)

    shared = blob(S.SHARED_EXPERT_ID, cfg["shared_bits"])
    n_tok = min(POOL, 8)
    xs = S.token_x(SEED, 0, 0, n_tok, h)
    res = S.token_residual(SEED, 0, 0, n_tok, h)
    pre = {}
    for t in range(n_tok):
        for ex in O.route(w_router, w_sg, xs[t], k)["idx"]:
            if int(ex) not in pre:
                pre[int(ex)] = blob(int(ex), cfg["bits"])

    def decode(t):
        t %= n_tok
        O.layer_decode(w_router, w_sg, lambda ex: pre[ex], shared, xs[t], res[t], k, h, i, cfg["bits"],
                       cfg["shared_bits"])
    return decode


def delta_oracle_prepare(cfg):
    """The same for the delta-rule workload: decode(t) is one token's update."""
    import oracle as O
    H, dk, dv = cfg["heads"], cfg["dk"], cfg["dv"]
    cur = {"state": S.delta_state(SEED, 0, H, dv, dk)}
    toks = [S.delta_tokens(SEED, 0, j, 1, H, dk, dv) for j in range(8)]

    def decode(t):
        tk = toks[t % len(toks)]
        cur["state"], _ = O.delta_update(cur["state"], tk["q"], tk["k"], tk["v"], tk["alpha"], tk["beta"])
    return decode


def time_oracle(decode, max_steps: int, budget_s: float):
    """Run decode(0), decode(1), ... until max_steps or budget_s; (steps, seconds)."""
    n = 0
    t0 = time.perf_counter()
    while n < max_steps:
        decode(n)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return n, time.perf_counter() - t0


def oracle_sample(cfg, budget_s: float) -> dict:
    """Time the oracle (as it stands) on a bounded sample of the same workload."""
    delta = cfg.get("kind") == "deltanet"
    decode = (delta_oracle_prepare if delta else oracle_prepare)(cfg)
    n, el = time_oracle(decode, 1 << 30, budget_s)
    what = (f"one-token updates of the {cfg['workload']} state" if delta else
            f"single-token decodes of the {cfg['workload']} layer (fp64 numpy oracle, expert blobs pre-drawn)")
    return dict(value=n / el, unit="updates/s" if delta else UNIT, cores=host_cores(), cpu_model=host_cpu_model(),
                kind="oracle", seconds=el, tokens=n, sample=f"{n} {what}, {el:.1f} s")


def run_reference(args, cfg, rank, world):
    """The reference arm: the CPU oracle as it stands, on rank 0 only.  Its
    inputs are drawn once; W warm-up steps (at most REF_WARMUP_S of host time)
    and then up to K timed steps, stopping after REF_BUDGET_S so that the run
    ends within a few minutes whatever K is; the rate is taken over the steps
    that ran, and the line says how many."""
    if rank != 0:
        return
    delta = cfg.get("kind") == "deltanet"
    decode = (delta_oracle_prepare if delta else oracle_prepare)(cfg)
    time_oracle(decode, args.warmup, REF_WARMUP_S)
    n, el = time_oracle(decode, args.steps, REF_BUDGET_S)
    lps = cfg.get("layers_per_step", cfg.get("stream_layers", 1))
    tt = cfg.get("tokens", 1)
    metric, unit = METRIC, UNIT
    if cfg.get("kind") == "stream":
        metric, unit = (f"tokens/s through {lps} MoE layers with routed experts streamed from host memory "
                        "(batch 1)"), "tokens/s"
    elif delta:
        metric, unit = DELTA_METRIC, "updates/s"
    elif lps > 1:
        metric, unit = f"decode steps/s through {lps} MoE layers (batch 1)", "steps/s"
    elif tt > 1:
        metric, unit = f"token decodes/s through one MoE layer ({tt}-token batches)", "tokens/s"
    value = n / el / lps  # one oracle step is one token through one layer (or one state update)
    what = "one-token state updates" if delta else "single-token single-layer decodes"
    sample = (f"{n} {what} timed of the {args.steps} steps asked (at most {REF_BUDGET_S:.0f} s of host time), "
              f"{el:.1f} s" + (f"; steps/s = decodes/s / {lps}" if lps > 1 else ""))
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**cfg, "batch": 1, "parallelism": "host cores"},
        "steps_timed": n,
        "cpu_baseline": {"value": value, "unit": unit, "cores": host_cores(), "cpu_model": host_cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------

def run_fmoe(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_quantized_expert_router_b200 as F
    import synth.gpu as SG
    from bit_quantized_expert_router_b200 import build as B

    if rank == 0 or not os.path.exists(F.LIB_PATH):
        B.build_engine()
        SG.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    F.set_dependent_launch(args.launch == "dependent")
    h, i, e, k = cfg["hidden"], cfg["inter"], cfg["experts"], cfg["top_k"]
    LPS = cfg.get("layers_per_step", 1)  # layer decodes per timed step
    NL = LPS if LPS > 1 else args.layers
    # NL distinct layer instances of the workload, decoded in turn: the weights
    # a step reads were last touched NL - 1 steps earlier, so they come from
    # HBM (NL * 40 MB >> 126 MB of L2) without any flush between steps.
    layers = []
    for l in range(NL):
        t = SG.make_layer(SEED + 1000 * rank, l, h, i, e, cfg["bits"], cfg["shared_bits"], F.blob_offsets,
                          F.expert_bytes, dev)
        # stacked layers normalise their input (the decoder stack's RMS norm)
        nw = SG.bf16_tensor(S.norm_bf16(SEED + 1000 * rank, l, h), dev) if LPS > 1 else None
        layers.append(F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], h, i, k, cfg["bits"],
                              cfg["shared_bits"], norm_weight=nw))
    TT = cfg.get("tokens", 1)  # tokens per decode call
    shape = (POOL, h) if TT == 1 else (POOL, TT, h)
    xs = torch.from_numpy(S.token_x(SEED + rank, 0, 0, POOL * TT, h).reshape(shape)).to(dev)
    rs = torch.from_numpy(S.token_residual(SEED + rank, 0, 0, POOL * TT, h).reshape(shape)).to(dev)
    out = torch.empty(shape, dtype=torch.float32, device=dev)
    ws = [L.workspace(TT) for L in layers]
    stream = torch.cuda.current_stream()

    hbuf = torch.empty(2, h, dtype=torch.float32, device=dev)

    def decode(j):
        l = j % NL
        if LPS == 1:
            layers[l].decode(xs[j % POOL], rs[j % POOL], out=out[j % POOL], ws=ws[l])
        else:
            # Stacked layers: layer l reads the hidden state layer l - 1 wrote,
            # as its input (normalised inside) and its residual; layer 0 starts
            # from a pool token.
            src = xs[(j // NL) % POOL] if l == 0 else hbuf[(l - 1) % 2]
            layers[l].decode(src, src, out=hbuf[l % 2], ws=ws[l])

    for j in range(args.warmup):
        decode(j)
    torch.cuda.synchronize()
    if F.get_status():
        raise RuntimeError("device status word set during warm-up")
    distinct = None
    if TT > 1:
        # distinct routed experts per step, over one period of the rotation
        idx = torch.empty(TT, k, dtype=torch.int32, device=dev)
        counts = []
        for j in range(64):
            layers[j % NL].decode(xs[j % POOL], rs[j % POOL], out=out[j % POOL], idx_out=idx, ws=ws[j % NL])
            counts.append(len(set(idx.flatten().tolist())))
        distinct = float(np.mean(counts))

    # Each captured step is the library's decode call; a graph holds GSTEPS
    # consecutive steps so that the timed region is device time, without the
    # Python/ctypes launch latency (the end-to-end figure below keeps that).
    GSTEPS = 64 if LPS == 1 else LPS
    K = args.steps * LPS  # layer decodes in the timed region

    def capture(first, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for j in range(first, first + n):
                decode(j)
        return g

    g_full = capture(0, GSTEPS)
    rem = K % GSTEPS
    g_rem = capture(0, rem) if rem else None
    # replay every graph the timed region uses once first, so that no first
    # replay (graph upload, first launch) falls inside it
    g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local_rank)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.1)
    ev0.record(stream)
    for _ in range(K // GSTEPS):
        g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = ev0.elapsed_time(ev1)
    status = F.get_status()

    # Latency of one isolated step with L2 flushed before it (single launch,
    # so it also carries the launch and event overheads of a lone kernel).
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    g_one = [capture(j, 1) for j in range(min(NL, 8))]
    lat = []
    for j in range(min(K, 400)):
        flush.fill_(j & 0xFF)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        g_one[j % len(g_one)].replay()
        a1.record(stream)
        lat.append((a0, a1))
    torch.cuda.synchronize()
    lat_us = [1000.0 * a.elapsed_time(b) for a, b in lat]
    del flush

    # The expert path alone: the same decodes with the routing given (the
    # selected experts' blobs, weights and gate passed in; no router rows, no
    # top-K), through fmoe_experts_decode, from graphs of GSTEPS calls.
    expert_path = None
    if LPS == 1 and TT == 1:
        routes = []
        idx = torch.empty(1, k, dtype=torch.int32, device=dev)
        wk = torch.empty(1, k, dtype=torch.float32, device=dev)
        for j in range(NL * 4):
            layers[j % NL].decode(xs[j % POOL], rs[j % POOL], out=out[j % POOL], idx_out=idx, w_out=wk,
                                  ws=ws[j % NL])
            routes.append((idx.cpu().numpy()[0].tolist(), wk.cpu().numpy()[0].tolist()))
        stride = layers[0].experts.stride(0)

        def expert_step(j):
            l = j % NL
            ix, wv = routes[j % len(routes)]
            base = layers[l].experts.data_ptr()
            F.experts_decode(layers[l], [base + e * stride for e in ix], wv, 0.5, xs[j % POOL], rs[j % POOL],
                             out=out[j % POOL], ws=ws[l])

        def capture_e(first, n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for j in range(first, first + n):
                    expert_step(j)
            return g

        for j in range(3):
            expert_step(j)
        ge = capture_e(0, GSTEPS)
        ge.replay()
        torch.cuda.synchronize()
        reps = max(1, K // GSTEPS)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(reps):
            ge.replay()
        c1.record(stream)
        torch.cuda.synchronize()
        ep_us = 1000.0 * c0.elapsed_time(c1) / (reps * GSTEPS)
        ab_e = algorithmic_bytes(cfg)
        ep_bytes = ab_e["experts"] + ab_e["vectors"]
        pk, _ = peaks()
        expert_path = {"us_per_decode": ep_us, "decodes_per_s": 1e6 / ep_us,
                       "bytes_per_decode": ep_bytes, "gbs": ep_bytes / (ep_us * 1e-6) / 1e9,
                       "frac_of_hbm": ep_bytes / (ep_us * 1e-6) / 1e9 / pk,
                       "note": "fmoe_experts_decode: the routed and shared experts' gate/up, SwiGLU, down and "
                               "the combine with the routing given (no router GEMV or top-K), same rotation"}
        del ge

    # End to end through the same call with host buffers: pinned host -> device
    # copy of x and residual, decode, device -> host copy of out, every step.
    xh = torch.from_numpy(S.token_x(SEED + rank, 0, 1, POOL * TT, h).reshape(shape)).pin_memory()
    rh = torch.from_numpy(S.token_residual(SEED + rank, 0, 1, POOL * TT, h).reshape(shape)).pin_memory()
    oh = torch.empty(shape, dtype=torch.float32).pin_memory()
    xd = torch.empty(shape[1:], dtype=torch.float32, device=dev)
    rd = torch.empty(shape[1:], dtype=torch.float32, device=dev)
    od = torch.empty(shape[1:], dtype=torch.float32, device=dev)
    K2 = min(K, 2000)

    def e2e_step(j):
        if LPS == 1:
            l = j % NL
            xd.copy_(xh[j % POOL], non_blocking=True)
            rd.copy_(rh[j % POOL], non_blocking=True)
            layers[l].decode(xd, rd, out=od, ws=ws[l])
            oh[j % POOL].copy_(od, non_blocking=True)
        else:
            # One token through every layer: its input goes up once and the last
            # layer's output comes back once.
            xd.copy_(xh[j % POOL], non_blocking=True)
            src = xd
            for l in range(NL):
                dst = hbuf[l % 2] if l + 1 < NL else od
                layers[l].decode(src, src, out=dst, ws=ws[l])
                src = dst
            oh[j % POOL].copy_(od, non_blocking=True)

    n_e2e = K2 if LPS == 1 else max(1, K2 // LPS)  # e2e steps
    for j in range(3):
        e2e_step(j)
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for j in range(n_e2e):
        e2e_step(j)
    b1.record(stream)
    torch.cuda.synchronize()
    e2e_ms_per_decode = b0.elapsed_time(b1) / (n_e2e * LPS)

    # max over ranks
    total_ms_max, e2e_ms_max = max_over_ranks([total_ms, e2e_ms_per_decode * K], world, dev)

    if rank == 0:
        ab = algorithmic_bytes(cfg, distinct)
        peak, peak_kind = peaks()
        avg_launch_s = total_ms / 1000.0 / K
        achieved = ab["total"] / avg_launch_s / 1e9
        steps = K // LPS
        value = whole_job_rate(steps * TT, world, total_ms_max)
        metric, unit = METRIC, UNIT
        if LPS > 1:
            metric, unit = f"decode steps/s through {LPS} MoE layers (batch 1)", "steps/s"
        elif TT > 1:
            metric, unit = f"token decodes/s through one MoE layer ({TT}-token batches)", "tokens/s"
        line = {
            "impl": "fmoe", "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": total_ms_max / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {**cfg, "batch": TT, "group": 64,
                       "weights": f"{cfg['bits']}-bit routed / {cfg['shared_bits']}-bit shared codes, bf16 scale+bias "
                                  "per group of 64, bf16 router",
                       "l2": f"inputs larger than L2: {NL} distinct layer instances decoded in turn "
                             f"({NL * e * expert_bytes(h, i, cfg['bits']) / 1e9:.0f} GB of experts), no flush",
                       "layers_in_rotation": NL, "input_pool": POOL, "parallelism": f"replicas x{world}",
                       **({"launch": args.launch} if TT == 1 else {})},
            "us_per_decode": 1000.0 * total_ms_max / K,
            "latency_us_l2_flushed": {"p50": statistics.median(lat_us), "p99": float(np.percentile(lat_us, 99)),
                                      "steps": len(lat_us),
                                      "note": "one isolated graph launch after a 256 MiB L2 flush"},
            "expert_gbs": ab["experts"] / avg_launch_s / 1e9,
            "expert_frac_of_hbm": ab["experts"] / avg_launch_s / 1e9 / peak,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(args.config),
                         "kernel": (f"layer_kernel<{cfg['bits']},{cfg['shared_bits']}>" if TT == 1 else
                                    "grouped decode step (router + shared gate/up, prep + shared down, routed "
                                    "gate/up, activation staging, routed down, combine launches)"),
                         "algorithmic_bytes_per_launch": ab["total"]},
            "layer_decodes_per_s": whole_job_rate(K, world, total_ms_max),
            "sustained_gbs": world * K * ab["total"] / (total_ms_max / 1000.0) / 1e9,
            "e2e": {"value": whole_job_rate(K * TT / LPS, world, e2e_ms_max), "unit": unit,
                    "h2d_bytes_per_step": (2 if LPS == 1 else 1) * TT * h * 4, "d2h_bytes_per_step": TT * h * 4},
            # a grouped step is six launches (see the kernel entry above)
            "gpu_launches": K * (1 if TT == 1 else 6),
            **({"distinct_routed_experts_per_step": distinct} if distinct is not None else {}),
            **({"expert_path": expert_path} if expert_path is not None else {}),
            "clocks": clk,
            "device_status": status,
        }
        if not args.no_cpu_baseline:
            cb = oracle_sample(cfg, args.cpu_seconds)
            cb.pop("seconds", None)
            cb.pop("tokens", None)
            if LPS > 1:  # a step is LPS layer decodes
                cb["value"] /= LPS
                cb["sample"] += f"; steps/s = decodes/s / {LPS}"
            cb["unit"] = unit  # one oracle decode is one token through one layer
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# The linear-attention state update (config "deltanet")
# ---------------------------------------------------------------------------

DELTA_KERNEL_SOURCES = ("common.cuh", "deltanet.cuh")


def delta_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_expert_router_b200", "csrc")
    for f in DELTA_KERNEL_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def delta_bytes(cfg) -> int:
    """Algorithmic bytes of one token's update: the state read and written,
    q and k read, v read and o written, the two gates read (all fp32)."""
    H, dk, dv = cfg["heads"], cfg["dk"], cfg["dv"]
    return 4 * (2 * H * dv * dk + 2 * H * dk + 2 * H * dv + 2 * H)


def run_delta(args, cfg, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_quantized_expert_router_b200 as F
    from bit_quantized_expert_router_b200 import build as B

    if rank == 0 or not os.path.exists(F.LIB_PATH):
        B.build_engine()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    H, dk, dv, NL = cfg["heads"], cfg["dk"], cfg["dv"], cfg["layers"]
    # NL layer states updated in turn: 45 x 4 MiB = 180 MiB, larger than L2,
    # so a step's state comes from HBM without any flush between steps.
    states = torch.stack([torch.from_numpy(S.delta_state(SEED + 1000 * rank, l, H, dv, dk)) for l in range(NL)]).to(dev)
    pool = [S.delta_tokens(SEED + rank, 0, j, 1, H, dk, dv) for j in range(POOL)]
    tok = {n: torch.from_numpy(np.stack([p[n] for p in pool])).to(dev) for n in pool[0]}
    o = torch.empty(POOL, 1, H, dv, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(j):
        t = j % POOL
        F.delta_update(states[j % NL], tok["q"][t], tok["k"][t], tok["v"][t], tok["alpha"][t], tok["beta"][t],
                       o=o[t])

    for j in range(args.warmup):
        step(j)
    torch.cuda.synchronize()
    GSTEPS = 64
    K = args.steps

    def capture(first, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for j in range(first, first + n):
                step(j)
        return g

    g_full = capture(0, GSTEPS)
    rem = K % GSTEPS
    g_rem = capture(0, rem) if rem else None
    # every graph the timed region uses is replayed once first (no first replay timed)
    g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.1)
    ev0.record(stream)
    for _ in range(K // GSTEPS):
        g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    total_ms = ev0.elapsed_time(ev1)

    # one isolated update after a 256 MiB L2 flush
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    g_one = capture(0, 1)
    lat = []
    for j in range(min(K, 400)):
        flush.fill_(j & 0xFF)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        g_one.replay()
        a1.record(stream)
        lat.append((a0, a1))
    torch.cuda.synchronize()
    lat_us = [1000.0 * a.elapsed_time(b) for a, b in lat]
    del flush

    # End to end through the same call with host buffers: the token's q, k, v
    # and gates go up from pinned memory and its readout comes back, every step.
    host = {n: torch.from_numpy(np.stack([p[n] for p in pool])).pin_memory() for n in pool[0]}
    dbuf = {n: torch.empty_like(tok[n][0]) for n in tok}
    oh = torch.empty(POOL, 1, H, dv, dtype=torch.float32).pin_memory()
    od = torch.empty(1, H, dv, dtype=torch.float32, device=dev)
    K2 = min(K, 2000)

    def e2e_step(j):
        t = j % POOL
        for n in dbuf:
            dbuf[n].copy_(host[n][t], non_blocking=True)
        F.delta_update(states[j % NL], dbuf["q"], dbuf["k"], dbuf["v"], dbuf["alpha"], dbuf["beta"], o=od)
        oh[t].copy_(od, non_blocking=True)

    for j in range(3):
        e2e_step(j)
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for j in range(K2):
        e2e_step(j)
    b1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = b0.elapsed_time(b1) / K2
    total_ms_max, e2e_ms_max = max_over_ranks([total_ms, e2e_ms * K], world, dev)
    status = F.get_status()

    if rank == 0:
        ab = delta_bytes(cfg)
        peak, peak_kind = peaks()
        achieved = ab / (total_ms / 1000.0 / K) / 1e9
        traffic = None
        pj = os.path.join(ROOT, "profiles", "delta_update_deltanet.json")
        if os.path.exists(pj):
            d = json.load(open(pj))
            if d.get("source_hash") == delta_source_hash():
                traffic = d.get("dram_bytes_per_launch")
        h2d = sum(int(dbuf[n].numel()) * 4 for n in dbuf)
        line = {
            "impl": "fmoe", "metric": DELTA_METRIC, "value": whole_job_rate(K, world, total_ms_max),
            "unit": "updates/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": total_ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {**cfg, "batch": 1,
                       "l2": f"inputs larger than L2: {NL} layer states of {H * dv * dk * 4 / 2**20:.0f} MiB "
                             f"updated in turn, no flush",
                       "input_pool": POOL, "parallelism": f"replicas x{world}"},
            "us_per_update": 1000.0 * total_ms_max / K,
            "latency_us_l2_flushed": {"p50": statistics.median(lat_us), "p99": float(np.percentile(lat_us, 99)),
                                      "steps": len(lat_us),
                                      "note": "one isolated graph launch after a 256 MiB L2 flush"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "kernel": f"delta_update_kernel<{dk // 128}>",
                         "algorithmic_bytes_per_launch": ab},
            "e2e": {"value": whole_job_rate(K, world, e2e_ms_max), "unit": "updates/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": int(od.numel()) * 4},
            "gpu_launches": K,
            "clocks": clk,
            "device_status": status,
        }
        if not args.no_cpu_baseline:
            cb = oracle_sample(cfg, args.cpu_seconds)
            cb.pop("seconds", None)
            cb.pop("tokens", None)
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Routed experts streamed from host memory (config "stream")
# ---------------------------------------------------------------------------

STREAM_MAX_STEPS = 2000


def run_stream(args, cfg, rank, world, local_rank):
    """Tokens/s through a stack of layers whose routed experts live in pinned
    host memory, per device slot count: each step copies the token in from
    pinned host memory, decodes it through every layer with the streamer
    (routing on the GPU, the decision to the host, one copy per missed expert
    on a copy stream, the shared expert and the hits decoded meanwhile) and
    reads the result back.  The hit rate and the host-to-device GB/s are those
    of the timed steps (the warm-up steps fill the slots)."""
    import torch

    import bit_quantized_expert_router_b200 as F
    import synth.gpu as SG
    from bit_quantized_expert_router_b200 import build as B

    if rank == 0 or not os.path.exists(F.LIB_PATH):
        B.build_engine()
        SG.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    h, i, e, k = cfg["hidden"], cfg["inter"], cfg["experts"], cfg["top_k"]
    NLS = cfg["stream_layers"]
    layers, hosts = [], []
    for l in range(NLS):
        t = SG.make_layer(SEED + 1000 * rank, l, h, i, e, cfg["bits"], cfg["shared_bits"], F.blob_offsets,
                          F.expert_bytes, dev)
        stride = t["experts"].stride(0)
        host = torch.empty(e, stride, dtype=torch.uint8, pin_memory=True)
        host.copy_(t["experts"])
        stub = torch.zeros(1, stride, dtype=torch.uint8, device=dev)
        layers.append(F.Layer(t["w_router"], t["w_sgate"], stub, t["shared"], h, i, k, cfg["bits"],
                              cfg["shared_bits"]))
        hosts.append(host)
        del t
        torch.cuda.empty_cache()
    steps = min(args.steps, STREAM_MAX_STEPS)
    n_tok = args.warmup + steps
    xs_host = torch.from_numpy(S.token_stream(SEED + rank, n_tok, h, cfg["rho"])).pin_memory()
    out_host = torch.empty(h, dtype=torch.float32).pin_memory()
    ws = layers[0].workspace(1)
    stream = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream()
    xbuf = torch.empty(h, dtype=torch.float32, device=dev)
    hbuf = [torch.empty(h, dtype=torch.float32, device=dev) for _ in range(2)]
    blob = F.expert_bytes(h, i, cfg["bits"])
    results = []
    for n_slots in cfg["slot_counts"]:
        slots = torch.empty(n_slots, hosts[0].shape[1], dtype=torch.uint8, device=dev)
        st = F.Streamer(layers, hosts, slots)
        launches = [0]

        def step(j, count=False):
            xbuf.copy_(xs_host[j], non_blocking=True)
            src = xbuf
            for l in range(NLS):
                before = st.stats()["misses"] if count else 0
                st.decode(l, src, src, out=hbuf[l % 2], ws=ws, copy_stream=copy_stream)
                if count:
                    # router + top-K, the hits/shared launch, and one more if anything was missed
                    launches[0] += 3 + (st.stats()["misses"] > before)
                src = hbuf[l % 2]
            out_host.copy_(src, non_blocking=True)
            stream.synchronize()

        for j in range(args.warmup):
            step(j)
        s0 = st.stats()
        torch.cuda.synchronize()
        clocks = ClockSampler(local_rank)
        clocks.start()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        for j in range(args.warmup, n_tok):
            step(j, count=True)
        ev1.record()
        torch.cuda.synchronize()
        clk = clocks.stop()
        ms = ev0.elapsed_time(ev1)
        s1 = st.stats()
        hits, misses = s1["hits"] - s0["hits"], s1["misses"] - s0["misses"]
        h2d = s1["h2d_bytes"] - s0["h2d_bytes"]
        status = F.get_status()
        (ms_max,) = max_over_ranks([ms], world, dev)
        results.append({"slots": n_slots, "slot_gb": n_slots * hosts[0].shape[1] / 1e9,
                        "hit_rate": hits / max(1, hits + misses), "misses_per_layer_decode": misses / (steps * NLS),
                        "h2d_gbs": h2d / (ms / 1000.0) / 1e9, "tokens_per_s": whole_job_rate(steps, world, ms_max),
                        "ms_per_token": ms_max / steps, "gpu_launches": launches[0], "clocks": clk,
                        "h2d_bytes_per_step": h * 4 + h2d / steps,
                        "device_status": status})
        if n_slots == cfg["default_slots"]:
            # Independent layer inputs (each layer its own token stream): each
            # step decoded layer after layer, and with every layer prepared
            # while the previous one decodes (its misses copied meanwhile).
            xs_ind = [torch.from_numpy(S.token_stream(SEED + 17 * (l + 1) + rank, n_tok, h, cfg["rho"])).pin_memory()
                      for l in range(NLS)]
            xin = [torch.empty(h, dtype=torch.float32, device=dev) for _ in range(NLS)]
            route_stream = torch.cuda.Stream()
            indep = {}
            for mode in ("one_step", "prepared_ahead"):
                def istep(j):
                    for l in range(NLS):
                        xin[l].copy_(xs_ind[l][j], non_blocking=True)
                    stream.synchronize()
                    if mode == "one_step":
                        for l in range(NLS):
                            st.decode(l, xin[l], xin[l], out=hbuf[l % 2], ws=ws, copy_stream=copy_stream)
                    else:
                        # layer l + 1 is routed and its misses copied while layer l decodes
                        st.prepare(0, xin[0], route_stream=route_stream, copy_stream=copy_stream)
                        for l in range(NLS):
                            st.finish(l, xin[l], xin[l], out=hbuf[l % 2], ws=ws)
                            if l + 1 < NLS:
                                st.prepare(l + 1, xin[l + 1], route_stream=route_stream, copy_stream=copy_stream)
                    out_host.copy_(hbuf[(NLS - 1) % 2], non_blocking=True)
                    stream.synchronize()
                for j in range(args.warmup):
                    istep(j)
                q0 = st.stats()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for j in range(args.warmup, n_tok):
                    istep(j)
                e1.record()
                torch.cuda.synchronize()
                q1 = st.stats()
                ims = e0.elapsed_time(e1)
                hh, mm = q1["hits"] - q0["hits"], q1["misses"] - q0["misses"]
                (ims_max,) = max_over_ranks([ims], world, dev)
                indep[mode] = {"tokens_per_s": whole_job_rate(steps, world, ims_max), "ms_per_token": ims_max / steps,
                               "hit_rate": hh / max(1, hh + mm),
                               "h2d_gbs": (q1["h2d_bytes"] - q0["h2d_bytes"]) / (ims / 1000.0) / 1e9}
            results[-1]["independent_layer_inputs"] = indep
        del st, slots
        torch.cuda.empty_cache()
    if rank == 0:
        main_r = next(r for r in results if r["slots"] == cfg["default_slots"])
        line = {
            "impl": "fmoe", "metric": f"tokens/s through {NLS} MoE layers with routed experts streamed from host "
                                      "memory (batch 1)",
            "value": main_r["tokens_per_s"], "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": main_r["ms_per_token"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {**cfg, "batch": 1, "group": 64, "slots": cfg["default_slots"],
                       "expert_bytes": blob, "host_expert_gb": NLS * e * hosts[0].shape[1] / 1e9,
                       "tokens": f"autoregressive stream, rho {cfg['rho']}, N(0,1) per element",
                       "l2": "experts stream from host memory; the device slots and the layers' router and shared "
                             "weights total far less than L2 per token only when they hit",
                       "parallelism": f"replicas x{world}"},
            "caches": results,
            "e2e": {"value": main_r["tokens_per_s"], "unit": "tokens/s",
                    "h2d_bytes_per_step": main_r["h2d_bytes_per_step"], "d2h_bytes_per_step": h * 4,
                    "note": "the timed steps copy each token in from pinned host memory and its result back, "
                            "and copy every missed expert from host memory: the value is end to end; "
                            f"per step the input is {h * 4} B plus misses x {blob} B of experts"},
            "gpu_launches": main_r["gpu_launches"],
            "clocks": main_r["clocks"],
            "device_status": max(r["device_status"] for r in results),
        }
        if not args.no_cpu_baseline:
            cb = oracle_sample(cfg, args.cpu_seconds)
            cb.pop("seconds", None)
            cb.pop("tokens", None)
            cb["value"] /= NLS
            cb["unit"] = "tokens/s"
            cb["sample"] += f"; tokens/s = decodes/s / {NLS} (experts resident in host memory, as here)"
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--layers", type=int, default=16, help="distinct layer instances decoded in turn")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["fmoe", "reference"], default="fmoe")
    ap.add_argument("--config", choices=sorted(CONFIGS), default="full4")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--launch", choices=["dependent", "cooperative"], default="dependent",
                    help="single-token layer kernel: programmatic dependent launch (overlaps the previous "
                         "decode's end) or cooperative launch")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = CONFIGS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    delta = cfg.get("kind") == "deltanet"
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, cfg, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if cfg.get("kind") == "stream":
            run_stream(args, cfg, rank, world, local_rank)
        else:
            (run_delta if delta else run_fmoe)(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
