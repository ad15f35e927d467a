"""Benchmark of the routed-expert MoE layer on B200.

Default workload: the GLM-scale decode layer (hidden 6144, expert intermediate
2048, 256 routed + 1 shared int4 experts resident in HBM, top-8 of 8 groups /
4 kept, routed_scaling_factor 2.5), one token per step with a fresh seed.  A
step is one moe_layer_forward call: router logits + top-k, bucketing, expert
gate/up + SwiGLU, down projection, combine.  Weight quantisation is load time
and is reported separately.

Timing: W warm-up steps, then K timed steps; L2 (126 MB) is flushed before each
step by writing a 256 MB buffer and reading it back (so the lines the step
evicts are clean) outside the timed events; each step is timed
with CUDA events on the launching stream; the job time is the max over ranks.
With --gpus N > 1 every rank runs its own replica (the layer does not shard:
no collective on the data path), so scaling is weak.

--impl reference times the CPU oracle (test infrastructure) on the same
workload, one token per step.
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

import int4_routed_expert_route_b200 as lib  # noqa: E402
from int4_routed_expert_route_b200 import synthetic as syn  # noqa: E402

METRIC = "MoE-layer tokens/s and int4 expert-weight HBM GB/s (fraction of roofline) on 1 B200"


def _code_only(text):
    """Source text without comments, whitespace collapsed: what the compiler sees."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def source_sha256(files):
    """sha256 over the code (comments and layout ignored) of the named library
    sources (csrc/), in the order given."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "int4_routed_expert_route_b200", "csrc", f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()


def measured_traffic(kernel, path=None):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    capture (profiles/roofline_traffic.txt), or None when the kernel's sources
    changed after that capture (their sha256 no longer matches)."""
    path = path or os.path.join(ROOT, "profiles", "roofline_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        for line in fh:
            f = line.split()
            if not f or f[0].startswith("#") or f[0] != kernel:
                continue
            try:
                return float(f[3]) if source_sha256(f[1].split(",")) == f[2] else None
            except OSError:
                return None
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
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
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [c.strip() for c in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(backend="nccl"):
    """One process per GPU (torchrun env vars); the layer is replicated, so the
    only collectives are the timing barrier and the max over ranks."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local if world > 1 else 0)
    if world > 1:
        import datetime
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def ranks_max(x, world, device):
    """Max over ranks of one float (an all-reduce on the device; identity for
    a single rank): every multi-rank time is the slowest rank's."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_step, steps, world, max_ms):
    """Whole-job throughput: the tokens all ranks processed over the slowest
    rank's time."""
    return tokens_per_step * steps * world / (max_ms * 1e-3)


# Profiling captures only (--alias-experts N): quantise N experts and let the
# router's E slots alias them, for a small device footprint under ncu.  The
# kernels stream the same bytes per step (8 routed experts hit 8 slots; two slots
# aliasing one expert are still read twice), but timed numbers are not taken so.
ALIAS_EXPERTS = 0


def build_layer(cfg, layer=0, dev="cuda"):
    experts = []
    t0 = time.perf_counter()
    qbytes = 0
    n_real = cfg.E if not ALIAS_EXPERTS else min(ALIAS_EXPERTS, cfg.E)
    for e in list(range(n_real)) + [cfg.E]:
        w = [syn.expert_weight(cfg, layer, e, m, dev) for m in ("gate", "up", "down")]
        ex = lib.QuantExpert.from_fp32(*w, bits=cfg.bits)
        qbytes += sum(x.numel() * 4 for x in w)
        experts.append(ex)
        del w
    torch.cuda.synchronize()
    load_s = time.perf_counter() - t0
    table = lib.ExpertTable([experts[e % n_real] for e in range(cfg.E)], dev)
    shared = lib.SharedExpert(experts[n_real], dev)
    gate = syn.router_gate(cfg, layer, dev)
    bias = syn.router_bias(cfg, layer, dev)
    rc = lib.router_cfg(cfg.E, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf, cfg.topp)
    return dict(experts=experts, table=table, shared=shared, gate=gate, bias=bias, rc=rc,
                load_s=load_s, fp32_bytes=qbytes,
                expert_bytes=experts[0].nbytes())


WORKLOADS = {
    "decode": syn.DECODE,
    "prefill": syn.PREFILL,
    "small_batch": syn.SMALL_BATCH.with_(T=32),
    # adaptive expert top-p 0.7: slots beyond the cumulative weight are dropped
    "decode_topp": syn.DECODE.with_(name="glm-scale decode, expert top-p 0.7", topp=0.7),
    # MTP verify: 4 drafts from one position, x_t = x_0 + 0.05 n_t, Zipf router
    "mtp_verify": syn.SMALL_BATCH.with_(name="glm-scale MTP verify, 4 correlated drafts, zipf bias", T=4),
}
# stacks of decode layers (RMSNorm + residual between layers), T = 1
STACKS = {
    "stack": syn.STACK,
    "stack_int8": syn.STACK_INT8,
    "stack_int2": syn.STACK_INT2,
}


def step_inputs(cfg, workload, n, rank, dev):
    """Per-step activations [n, T, H] bf16 (drafts share x_0 for mtp_verify)."""
    T = cfg.T
    if workload == "mtp_verify":
        x0 = syn.normal((n, 1, cfg.H), 1.0, syn.seed_of("mtp-x0", rank, n), dev)
        noise = syn.normal((n, T, cfg.H), 0.05, syn.seed_of("mtp-noise", rank, n), dev)
        return (x0 + noise).to(torch.bfloat16)
    return syn.activations(n * T, cfg.H, 1 + 1000003 * rank, dev).view(n, T, cfg.H)


DTYPE_DETAIL = {
    1: "int4 codes decoded to f32, f32 FMA (CUDA cores); bf16 activations",
    2: ("int4 codes against activations in 23-bit fixed point split into byte limbs (dp4a, "
        "s32 accumulation, exact), limb sums combined in f64 and rounded once to f32"),
    3: ("int4 codes converted to bf16 (gate/up) / f16 (down), tcgen05 MMA with f32 accumulation; "
        "bf16 activations"),
}


def workload_name(cfg):
    return (f"{cfg.name}: T={cfg.T} per step, H={cfg.H} I={cfg.I} E={cfg.E}+1 shared "
            f"top-{cfg.k} n_group={cfg.n_group} topk_group={cfg.topk_group} rsf={cfg.rsf} "
            f"int{cfg.bits}, router bias {cfg.bias_kind}")



def flush_l2(buf, i):
    """Evict L2 before a step: write the 256 MB buffer (twice L2), then read it
    back, so that the lines the step evicts are clean (a decode loop evicts the
    previous layer's weights, which are clean too) and no write-back of the
    flush itself lands inside the timed step."""
    buf.fill_(i & 0xff)
    buf.view(torch.int64).sum()


def _staged_steps(L, bias, xs, cfg, T, flush, dev):
    """Per-step device times of moe_layer_forward over the steps in xs [n, T, H]
    (L2 flushed before each step, outside the events), replayed from one
    captured graph; returns (step_ms [n], stage_ms [n, 5], idx [n, T, k])."""
    stream = torch.cuda.current_stream()
    n = xs.shape[0]
    rc = L["rc"]
    y = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    idx = torch.empty((n, T, cfg.k), dtype=torch.int32, device=dev)
    ws = lib.Workspace(lib.moe_layer_workspace_bytes(T, cfg.H, cfg.I, rc), dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(lib.LAYER_EVENTS)] for _ in range(n)]
    for e in (x for row in ev for x in row):
        e.record(stream)

    def step(i):
        flush_l2(flush, i)
        lib.moe_layer_forward(xs[i], L["gate"], bias, rc, L["table"], L["shared"], cfg.bits, y=y,
                              ws=ws, events=ev[i], idx_out=idx[i])

    for i in range(min(n, 2)):  # warm-up outside the graph
        step(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            step(i)
    g.replay()
    torch.cuda.synchronize()
    assert ws.flags() == 0
    step_ms = np.array([ev[i][0].elapsed_time(ev[i][-1]) for i in range(n)])
    stage_ms = np.array([[ev[i][s].elapsed_time(ev[i][s + 1]) for s in range(lib.LAYER_EVENTS - 1)]
                         for i in range(n)])
    del g
    return step_ms, stage_ms, idx.cpu().numpy()


def secondary_numbers(L, cfg, flush, dev, peaks, peak_kind, steps=8):
    """Small batches with the Zipf-skewed router (T = 2, 4, 8, 32) and the
    4096-token prefill, on the same resident experts as the headline."""
    H, I = cfg.H, cfg.I
    ex_bytes = 2 * (I * H // 2 + I * 4) + (H * I // 2 + H * 4)
    out = {"note": "same resident int4 experts as the headline; L2 flushed before every step; "
                   "per-step CUDA events, medians over the steps"}
    zipf = syn.router_bias(syn.SMALL_BATCH, 0, dev)
    small = {}
    for T in (2, 4, 8, 32):
        xs = syn.activations(steps * T, H, 7001 + T, dev).view(steps, T, H)
        step_ms, _, idx = _staged_steps(L, zipf, xs, cfg, T, flush, dev)
        uniq = np.array([len(np.unique(r[r >= 0])) for r in idx])
        byts = (uniq + 1) * ex_bytes + cfg.E * H * 4
        ms = float(np.median(step_ms))
        gbs = float(np.median(byts / (step_ms * 1e-3))) / 1e9
        small[f"T{T}"] = {"tokens_per_s": round(T / (ms * 1e-3), 1), "ms_per_step": round(ms, 5),
                          "unique_experts": float(np.mean(uniq)),
                          "expert_gbs": round(gbs, 1),
                          "hbm_frac": round(gbs / peaks["hbm_gbs"], 4)}
    out["small_batch_zipf"] = small
    T = 4096
    xs = syn.activations(3 * T, H, 7777, dev).view(3, T, H)
    step_ms, stage_ms, idx = _staged_steps(L, L["bias"], xs, cfg, T, flush, dev)
    pairs = np.array([int((r >= 0).sum()) for r in idx])
    f1 = (pairs + T) * 2.0 * (2 * I) * H
    f2 = (pairs + T) * 2.0 * I * H
    t1 = float(np.median(f1 / (stage_ms[:, 2] * 1e-3))) / 1e12
    t2 = float(np.median(f2 / (stage_ms[:, 3] * 1e-3))) / 1e12
    ms = float(np.median(step_ms))
    pk = peaks["bf16_tflops"]
    out["prefill_T4096"] = {
        "tokens_per_s": round(T / (ms * 1e-3), 1), "ms_per_step": round(ms, 4),
        "layer_tflops": round(float(np.median((f1 + f2) / (step_ms * 1e-3))) / 1e12, 1),
        "tc_ffn1_tflops": round(t1, 1), "tc_ffn1_frac": round(t1 / pk, 4),
        "tc_ffn2_tflops": round(t2, 1), "tc_ffn2_frac": round(t2 / pk, 4),
        "peak": pk, "peak_source": peak_kind + " (bf16 burst)",
        "stage_ms_median": {n: round(float(np.median(stage_ms[:, s])), 4) for s, n in
                            enumerate(["router", "bucket", "gate_up", "down", "combine"])}}
    return out


def run_ours(args, world, rank):
    cfg = WORKLOADS[args.workload]
    T = cfg.T
    dev = torch.device("cuda")
    L = build_layer(cfg)
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup
    xs = step_inputs(cfg, args.workload, K + W, rank, dev)
    idx_buf = torch.empty((K + W, T, cfg.k), dtype=torch.int32, device=dev)
    y = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    ws = lib.Workspace(lib.moe_layer_workspace_bytes(T, cfg.H, cfg.I, L["rc"]), dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    nsteps = K + W
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(lib.LAYER_EVENTS)]
          for _ in range(nsteps)]
    for e in (x for row in ev for x in row):
        e.record(stream)
    torch.cuda.synchronize()

    def step(i, events=None):
        lib.moe_layer_forward(xs[i], L["gate"], L["bias"], L["rc"], L["table"], L["shared"],
                              cfg.bits, y=y, ws=ws, events=events, idx_out=idx_buf[i])

    # The timed loop runs as one CUDA graph (flush + layer per step), so
    # host-side launch overhead does not leak into device time.  It records
    # only each step's start and end: an event between two of the layer's
    # kernels would cut their programmatic-launch overlap.  A second graph of
    # the same steps with every stage event gives the stage breakdown and the
    # dominant kernel's duration.
    for i in range(W):
        flush_l2(flush, i)
        step(i, ev[i])
    torch.cuda.synchronize()
    ends = [[ev[i][0]] + [None] * (lib.LAYER_EVENTS - 2) + [ev[i][-1]] for i in range(nsteps)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(W, nsteps):
            flush_l2(flush, i)
            step(i, ends[i])
    staged = torch.cuda.CUDAGraph()
    with torch.cuda.graph(staged):
        for i in range(W, nsteps):
            flush_l2(flush, i)
            step(i, ev[i])
    torch.cuda.synchronize()
    staged.replay()
    torch.cuda.synchronize()
    stage_ms = np.array([[ev[i][s].elapsed_time(ev[i][s + 1]) for s in range(lib.LAYER_EVENTS - 1)]
                         for i in range(W, nsteps)])
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    for _rep in range(args.repeat):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = np.array([ev[i][0].elapsed_time(ev[i][-1]) for i in range(W, nsteps)])
    total_ms = ranks_max(float(step_ms.sum()), world, dev)
    clk = clocks.stop()

    # end to end through the C ABI with host buffers: pinned x in, y out, per step
    hx = xs.cpu().pin_memory()
    hy = torch.empty((T, cfg.H), dtype=torch.float32).pin_memory()
    dx = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(nsteps)]
    for i in range(nsteps):
        flush_l2(flush, i)
        e2e_ev[i][0].record(stream)
        dx.copy_(hx[i], non_blocking=True)
        lib.moe_layer_forward(dx, L["gate"], L["bias"], L["rc"], L["table"], L["shared"],
                              cfg.bits, y=y, ws=ws)
        hy.copy_(y, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks_max(sum(a.elapsed_time(b) for a, b in e2e_ev[W:]), world, dev)
    assert ws.flags() == 0

    peaks, peak_kind = measured_peaks()
    H, I = cfg.H, cfg.I
    idx_np = idx_buf[W:].cpu().numpy()
    uniq = np.array([len(np.unique(r[r >= 0])) for r in idx_np])  # unique routed experts per step
    pairs = np.array([int((r >= 0).sum()) for r in idx_np])        # routed (token, slot) pairs
    ex_bytes = 2 * (I * H // 2 + I * 4) + (H * I // 2 + H * 4)    # one int4 expert
    gu_bytes = (uniq + 1) * 2 * (I * H // 2 + I * 4)               # + shared expert
    expert_bytes_step = (uniq + 1) * ex_bytes
    gu_ms = stage_ms[:, 2]
    tokens = K * T * world
    value = job_tokens_per_s(T, K, world, total_ms)
    if T <= 2:
        kern = "gateup_decode (int4 gate+up GEMV + SwiGLU, CUDA cores)"
        achieved = float(np.mean(gu_bytes / (gu_ms * 1e-3))) / 1e9
        roof = {"kernel": kern, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "peak_source": peak_kind, "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": measured_traffic("gateup_decode"),
                "algorithmic_bytes_per_launch": int(np.mean(gu_bytes))}
        launches = 3
    elif T <= 8:  # 3..8 tokens
        # one persistent kernel per layer call: router, selection, experts, combine
        kern = "decode_layer (router, int4 gate/up + SwiGLU, down + combine; CUDA cores, dp4a)"
        layer_bytes = expert_bytes_step + cfg.E * H * 4
        k_ms = stage_ms[:, 0]
        achieved = float(np.mean(layer_bytes / (k_ms * 1e-3))) / 1e9
        roof = {"kernel": kern, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "peak_source": peak_kind, "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": measured_traffic("decode_layer"),
                "algorithmic_bytes_per_launch": int(np.mean(layer_bytes))}
        launches = 1
    else:
        kern = "tc_ffn<1> (tcgen05 int4->bf16 grouped GEMM, gate+up + SwiGLU)"
        gu_flops = (pairs + T) * 2.0 * (2 * I) * H                  # 2 * M * N * K, gate and up
        achieved = float(np.mean(gu_flops / (gu_ms * 1e-3))) / 1e12
        roof = {"kernel": kern, "bound": "tensor", "achieved": round(achieved, 1),
                "peak": peaks["bf16_tflops"], "peak_source": peak_kind + " (bf16 burst)",
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": measured_traffic("tc_ffn<1>"),
                "algorithmic_flops_per_launch": float(np.mean(gu_flops))}
        launches = 7  # router logits, select, bucket, gather, two tc_ffn passes, combine
    total_flops_step = (pairs + T) * 2.0 * 3 * I * H
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32" if T <= 2 else ("s32" if T <= 8 else "bf16"),
        "dtype_detail": DTYPE_DETAIL[1 if T <= 2 else (2 if T <= 8 else 3)],
        "data": "synthetic (seeded N(0,0.02) weights quantised on device; x ~ N(0,1) bf16)",
        "config": {"workload": workload_name(cfg), "tokens_per_step": T,
                   "l2": "flushed before every step (256 MB write, then read back so the evicted lines are clean; outside the timed events)",
                   "parallelism": f"replicas x{world}"},
        "expert_gbs": round(float(np.mean(expert_bytes_step)) / (total_ms / K * 1e-3) / 1e9, 1),
        "expert_bytes_per_step": int(np.mean(expert_bytes_step)),
        "unique_experts_per_step": float(np.mean(uniq)),
        "layer_tflops": round(float(np.mean(total_flops_step)) / (total_ms / K * 1e-3) / 1e12, 2),
        "stage_ms_median": {n: round(float(np.median(stage_ms[:, s])), 5) for s, n in
                            enumerate(["router", "bucket", "gate_up", "down", "combine"])},
        "roofline": roof,
        "e2e": {"value": round(job_tokens_per_s(T, K, world, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 4},
        "gpu_launches": launches * K,
        "clocks": clk,
        "load": {"quantize_s": round(L["load_s"], 3), "fp32_bytes": L["fp32_bytes"],
                 "int4_expert_bytes": L["expert_bytes"]},
    }
    if args.workload == "decode" and not args.no_secondary and world == 1:
        res["secondary"] = secondary_numbers(L, cfg, flush, dev, peaks, peak_kind)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, L, xs[W:W + 4], samples=4)
    return res


def run_stack(args, world, rank):
    """A stack of decode layers (moe_stack_forward: per layer RMSNorm -> router
    -> gate/up -> down, residual add in fp32), T = 1 token per step; every step
    streams every layer's selected experts, far more than L2 holds."""
    cfg = STACKS[args.workload]
    T, H, I, nl = cfg.T, cfg.H, cfg.I, cfg.layers
    dev = torch.device("cuda")
    layers = [build_layer(cfg, layer=l) for l in range(nl)]
    rc = layers[0]["rc"]
    params = [(L["gate"], L["bias"], L["table"], L["shared"], cfg.bits) for L in layers]
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup
    nsteps = K + W
    resid = syn.normal((nsteps, T, H), 1.0, syn.seed_of("stack-resid", rank, nsteps), dev)
    idx = torch.empty((nsteps, nl, T, cfg.k), dtype=torch.int32, device=dev)
    ws = lib.Workspace(lib.moe_stack_workspace_bytes(T, H, I, rc), dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # recorded inside the graph capture: external event nodes, or they time nothing
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(nsteps)]
    for a, b in ev:  # create them outside the capture
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()

    def step(i):
        lib.moe_stack_forward(resid[i], params, rc, I, eps=1e-6, idx_out=idx[i], ws=ws)

    for i in range(W):
        flush_l2(flush, i)
        step(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(W, nsteps):
            flush_l2(flush, i)
            ev[i][0].record()  # the capturing stream
            step(i)
            ev[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    graph.replay()  # the stacks are one replay: each step already streams tens of GB
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = np.array([ev[i][0].elapsed_time(ev[i][1]) for i in range(W, nsteps)])
    total_ms = ranks_max(float(step_ms.sum()), world, dev)
    clk = clocks.stop()

    # end to end through the C ABI: the residual comes from and goes back to pinned host memory
    hr = resid[:nsteps].cpu().pin_memory()
    dr = torch.empty((T, H), dtype=torch.float32, device=dev)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nsteps)]
    for i in range(nsteps):
        flush_l2(flush, i)
        e2e_ev[i][0].record(stream)
        dr.copy_(hr[i], non_blocking=True)
        lib.moe_stack_forward(dr, params, rc, I, eps=1e-6, ws=ws)
        hr[i].copy_(dr, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks_max(sum(a.elapsed_time(b) for a, b in e2e_ev[W:]), world, dev)
    assert ws.flags() == 0

    peaks, peak_kind = measured_peaks()
    ib = layers[0]["expert_bytes"]  # one expert of this width
    idx_np = idx[W:].cpu().numpy()
    uniq = np.array([[len(np.unique(r[l][r[l] >= 0])) for l in range(nl)] for r in idx_np])
    bytes_step = ((uniq + 1) * ib).sum(axis=1)  # + the shared expert of every layer
    achieved = float(np.mean(bytes_step / (step_ms * 1e-3))) / 1e9
    return {
        "metric": METRIC,
        "value": round(job_tokens_per_s(T, K, world, total_ms), 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "dtype_detail": f"int{cfg.bits} codes decoded to f32, f32 FMA; bf16 layer inputs, f32 residual",
        "data": "synthetic (seeded N(0,0.02) weights quantised on device; residual ~ N(0,1) fp32)",
        "config": {"workload": f"{cfg.name}: {nl} layers, T={T} per step, H={H} I={I} E={cfg.E}+1 "
                               f"shared top-{cfg.k}, RMSNorm eps 1e-6 + fp32 residual",
                   "tokens_per_step": T,
                   "l2": "flushed before every step (256 MB write, then read back) and the step streams "
                         f"{float(np.mean(bytes_step)) / 1e9:.1f} GB",
                   "parallelism": f"replicas x{world}"},
        "expert_gbs": round(achieved, 1),
        "expert_bytes_per_step": int(np.mean(bytes_step)),
        "unique_experts_per_layer": float(np.mean(uniq)),
        "roofline": {"kernel": f"whole stack step ({nl} x (RMSNorm, router, gate/up, down))",
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "peak_source": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
                     "algorithmic_bytes_per_launch": int(np.mean(bytes_step))},
        "e2e": {"value": round(job_tokens_per_s(T, K, world, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 4, "d2h_bytes_per_step": T * H * 4},
        "gpu_launches": 4 * nl * K,
        "clocks": clk,
    }


def _oracle_expert(orc, cfg, e, dev="cuda"):
    w = [syn.expert_weight(cfg, 0, e, m, dev).cpu().numpy() for m in ("gate", "up", "down")]
    q = [orc.quantize_rows(wi, cfg.bits) for wi in w]
    return orc.Expert(q[0][0], q[0][1], q[1][0], q[1][1], q[2][0], q[2][1], cfg.bits)


def cpu_baseline(cfg, L, xs, samples=4):
    """The oracle timed on the host cores on `samples` tokens of the workload,
    once on one thread and once on every core (the oracle splits each expert
    FFN's output rows over its threads; the results do not depend on the count)."""
    import oracle as orc
    gate = L["gate"].cpu().numpy()
    bias = L["bias"].cpu().numpy()
    xb = syn.bf16_bits(xs.reshape(-1, cfg.H)[:samples])
    samples = xb.shape[0]
    r = orc.route(xb, gate, bias, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf)
    need = sorted(set(int(e) for e in r["idx"].reshape(-1)))
    experts = [_oracle_expert(orc, cfg, e) if e in need else None for e in range(cfg.E)]
    shared = _oracle_expert(orc, cfg, cfg.E)
    ncores = os.cpu_count() or 1
    out = {}
    for threads in (1, ncores):
        orc.set_num_threads(threads)
        t0 = time.perf_counter()
        orc.layer(xb, gate, bias, experts, shared, cfg.H, cfg.I, cfg.k, cfg.n_group,
                  cfg.topk_group, cfg.rsf)
        out[threads] = samples / (time.perf_counter() - t0)
    orc.set_num_threads(ncores)
    return {"value": round(out[ncores], 4), "unit": "tokens/s", "cores": ncores,
            "value_1_thread": round(out[1], 4), "kind": "oracle",
            "sample": f"{samples} token(s) of the GLM-scale decode layer through the fp64 C "
                      f"oracle (routing + 9 experts per token), on 1 thread and on {ncores}; "
                      f"experts quantised beforehand (untimed)"}


def run_reference(args, world, rank):
    import oracle as orc
    cfg = syn.DECODE
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    gate = syn.router_gate(cfg, 0, dev).cpu().numpy()
    bias = syn.router_bias(cfg, 0, dev).cpu().numpy()
    K, W = args.steps, args.warmup
    xs = syn.bf16_bits(syn.activations(K + W, cfg.H, 1, dev))
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = _oracle_expert(orc, cfg, e, dev)
        return cache[e]

    def step(i):
        r = orc.route(xs[i:i + 1], gate, bias, cfg.k, cfg.n_group, cfg.topk_group, cfg.rsf)
        experts = [None] * cfg.E
        for e in r["idx"].reshape(-1):
            experts[int(e)] = expert(int(e))
        return experts, r

    sh = expert(cfg.E)
    ncores = os.cpu_count() or 1
    orc.set_num_threads(ncores)
    times = []
    for i in range(K + W):
        experts, r = step(i)  # expert preparation (quantisation) is load time, untimed
        t0 = time.perf_counter()
        orc.layer(xs[i:i + 1], gate, bias, experts, sh, cfg.H, cfg.I, cfg.k, cfg.n_group,
                  cfg.topk_group, cfg.rsf)
        dt = time.perf_counter() - t0
        if i >= W:
            times.append(dt)
    total = sum(times)
    value = K / total
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": 1,
        "steps": K, "warmup": W, "ms_per_step": round(total / K * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_name(cfg), "tokens_per_step": 1},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": ncores,
                         "kind": "oracle",
                         "sample": f"one token per step through the fp64 C oracle layer "
                                   f"(routing + 9 experts, each expert's rows split over "
                                   f"{ncores} threads); expert quantisation untimed"},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS) + sorted(STACKS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the small-batch and prefill numbers of the decode workload")
    ap.add_argument("--repeat", type=int, default=10,
                    help="replays of the captured timed loop (the last one is reported)")
    ap.add_argument("--alias-experts", type=int, default=0,
                    help="profiling captures only: quantise this many experts and alias the "
                         "router's slots onto them (small device footprint)")
    args = ap.parse_args()
    global ALIAS_EXPERTS
    ALIAS_EXPERTS = args.alias_experts
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, 1, 0)))
        return
    lib.load()
    world, rank, _ = dist_setup()
    res = run_stack(args, world, rank) if args.workload in STACKS else run_ours(args, world, rank)
    if rank == 0:
        if ALIAS_EXPERTS:
            res["config"]["alias_experts"] = f"{ALIAS_EXPERTS} (profiling capture; not a benchmark number)"
        print(json.dumps(res))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
