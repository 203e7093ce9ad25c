#!/usr/bin/env python
"""Throughput of the DeepSeek-V3-style MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step is one pass of the whole layer (router, dispatch, grouped SwiGLU
experts, combine) over one batch of the workload through the C ABI
(moe_forward), with inputs resident in HBM. The default workload is the
DeepSeek-V3-shape decode batch (T=128, D=7168, 256 experts, top-8, I=2048, one
shared expert, bf16); --config v3_prefill etc. select the other workloads.
Every step streams ~22 GB of expert weights, far more than the 126 MB L2, so
no L2 flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the layer (the layer does not shard: replicas only); value is the
tokens of all ranks over the slowest rank's device time.

Printed (rank 0, one JSON line): tokens/s from CUDA events on the launching
stream; e2e tokens/s through the same C call with x copied in from pinned host
memory and y copied back every step; the roofline of the dominant kernel from
per-kernel CUDA events recorded inside the timed region; the layer roofline;
the CPU oracle's rate on a bounded token sample (N=1 only); SM clocks sampled
during the run.

--impl reference times the CPU oracle (the plain fp64 statement of the layer)
on the host cores, on the same workload, metric and unit.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_42_b200 import inputs  # noqa: E402

METRIC = "MoE-layer tokens/sec on 1 B200 at V3 shape; % of roofline (HBM or tensor)"
UNIT = "tokens/s"
FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)
NOMINAL_PEAKS = dict(hbm_gbs=8000.0, bf16_tflops=2250.0)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="v3_decode", choices=sorted(inputs.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=0,
                    help="tokens in the CPU oracle sample (0: sized to ~15 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T of the workload (smaller cases for profiling)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the number of routed experts (smaller cases for profiling)")
    ap.add_argument("--expert-kernel", default="auto", choices=["auto", "simt", "one_cta", "pair"],
                    help="GEMM kernels of a bf16 layer (moe_select_expert_kernel)")
    return ap.parse_args()


def workload(a):
    cfg = inputs.CONFIGS[a.config]
    if a.tokens:
        cfg = cfg.with_(T=a.tokens, name=f"{cfg.name}[T={a.tokens}]")
    if a.experts:
        cfg = cfg.with_(n_routed=a.experts, name=f"{cfg.name}[E={a.experts}]")
    return cfg


# ---------------------------------------------------------------- distributed

class Dist:
    """One process per GPU (torchrun env). The layer does not shard: ranks run
    independent replicas and only meet for the timing barrier and the max of
    the per-rank device times (NCCL on GPUs, gloo when there are none)."""

    def __init__(self, backend=None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if self.world > 1:
            import torch.distributed as dist
            backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
            self.dev = torch.device("cuda", self.local) if backend == "nccl" else torch.device("cpu")
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = self.dev
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=self.dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ---------------------------------------------------------------- measurements

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class Clocks:
    """nvidia-smi samples of the SM clock and throttle reasons, every 100 ms."""

    Q = ("timestamp,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self, t0, t1, uuid):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = []
        for line in self.f.read().splitlines():
            c = [x.strip() for x in line.split(",")]
            if len(c) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(c[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, c[1].lower(), float(c[2]), float(c[3]), float(c[4]), c[5:]))
            except ValueError:
                continue
        os.unlink(self.f.name)
        mine = [r for r in rows if uuid and uuid.lower() in r[1]] or rows
        inside = [r for r in mine if t0 <= r[0] <= t1]
        window = "timed"
        if len(inside) < 3:
            inside, window = mine, "warmup+timed"
        if not inside:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[5][1:5]) if v.strip() == "Active"})
        return {"sm_mhz": float(np.median([r[2] for r in inside])), "sm_max_mhz": max(r[3] for r in inside),
                "reasons": reasons, "samples": len(inside), "window": window,
                "power_w_max": max(r[4] for r in inside)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


REFERENCE_BUDGET_S = 120.0   # wall time of the reference arm's warm-up and timed steps


def host_bits(t):
    """A tensor's values for the oracle: bf16 as raw uint16 bits, else numpy."""
    t = t.detach().contiguous().cpu()
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()


def oracle_rate(cfg, x_cpu, w_r, bias, w_dev, n_tok, seed=0, reps=1):
    """Tokens/s of the CPU oracle on a seeded sample of n_tok tokens of the
    workload (routing and experts of those tokens; a token's routing and
    output depend only on its own row). Host copies of the weights are made
    outside the timed part."""
    from oracle import moe_oracle as O

    host = host_bits
    rng = np.random.default_rng(seed)
    tok = np.sort(rng.choice(x_cpu.shape[0], size=min(n_tok, x_cpu.shape[0]), replace=False))
    xs, wr = host(x_cpu)[tok], host(w_r)
    b = None if bias is None else bias.numpy().astype(np.float64)
    kw = dict(n_groups=cfg.n_groups, topk_groups=cfg.topk_groups, topk=cfg.topk, score_func=cfg.score,
              route_scale=cfg.route_scale)
    # copy the experts these tokens use to the host first
    r = O.route(O.router_logits(xs, wr), b, **kw)
    used = sorted(set(r["idx"].ravel().tolist()))
    w1, w3, w2, ws1, ws3, ws2 = w_dev
    hw = {e: (host(w1[e]), host(w3[e]), host(w2[e])) for e in used}
    shared = None if ws1 is None else (host(ws1), host(ws3), host(ws2))
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        O.moe_forward(xs, wr, b, lambda e: hw[e], shared, act_dtype=cfg.dtype, **kw)
        times.append(time.perf_counter() - t0)
    return len(tok) / float(np.median(times)), len(tok), len(used), times


def layer_roofline(cfg, n_active, pk):
    """Algorithmic FLOPs and bytes of one layer pass (router, routed and
    shared experts; each active expert's weights, the shared weights, W_r,
    x and y counted once)."""
    T, D, E, k, I, Is = cfg.T, cfg.dim, cfg.n_routed, cfg.topk, cfg.moe_inter, cfg.shared_inter
    ab = 4 if cfg.dtype == "f32" else 2
    flops = 2 * T * D * E + 6 * T * k * D * I + 6 * T * D * Is
    byts = (n_active * 3 * I * D + 3 * Is * D + E * D + 2 * T * D) * ab
    t_f = flops / (pk["bf16_tflops"] * 1e12)
    t_b = byts / (pk["hbm_gbs"] * 1e9)
    return flops, byts, max(t_f, t_b), "tensor" if t_f >= t_b else "hbm"


def l2_note(cfg, n_active):
    """How the timed loop stands to the 126 MB L2: the weights every step
    streams exceed it (no flush needed), or the workload fits (a small,
    launch-bound case)."""
    wbytes = (n_active * 3 * cfg.moe_inter + 3 * cfg.shared_inter) * cfg.dim * (4 if cfg.dtype == "f32" else 2)
    if wbytes > 126e6:
        return f"inputs larger than L2 (every step streams the active experts' weights, {wbytes / 1e9:.1f} GB)"
    return (f"inputs fit in L2 ({wbytes / 1e6:.2f} MB of weights, no flush): a small, launch-bound "
            "workload, not the roofline case")


def up_kernel_work(cfg, n_active):
    """Algorithmic FLOPs and bytes of one launch of the grouped up-projection
    (w1 and w3 of every active expert and of the shared expert, x_perm and x
    read once, h and h_shared written once)."""
    T, D, k, I, Is = cfg.T, cfg.dim, cfg.topk, cfg.moe_inter, cfg.shared_inter
    ab = 4 if cfg.dtype == "f32" else 2
    flops = 4 * T * k * D * I + 4 * T * D * Is
    byts = (n_active * 2 * I * D + 2 * Is * D + T * k * D + T * k * I + T * D + T * Is) * ab
    return flops, byts


def source_digest(path):
    """sha256 (16 hex digits) of a C++/CUDA source with its comments and
    whitespace removed: it changes when the code changes, not the comments."""
    import re
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return hashlib.sha256("".join(src.split()).encode()).hexdigest()[:16]


def traffic_for(kernel, config_name):
    """DRAM bytes per launch of `kernel` on `config_name` from the committed
    ncu summary, if the kernel source is unchanged since it was captured."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}@{config_name}")
    if not ent:
        return None
    src = os.path.join(ROOT, "mixture_experts_layer_42_b200", "csrc", ent["source"])
    if not os.path.exists(src) or source_digest(src) != ent["source_sha256_16"]:
        return None
    return float(ent["dram_bytes_per_launch"])


# ---------------------------------------------------------------- arms

def reference_arm(a, D):
    """The CPU oracle, as it stands, on the host cores (rank 0 only). Every
    step runs it on the same seeded token sample (the experts those tokens
    use are copied to the host once, outside all timing); the sample is sized
    from a one-token probe so that warm-up and timed steps together take
    about REFERENCE_BUDGET_S seconds."""
    if D.rank != 0:
        return
    from oracle import moe_oracle as O
    cfg = workload(a)
    x, w_r, bias = inputs.routing_inputs(cfg)
    w = inputs.expert_weights(cfg, "cuda" if torch.cuda.is_available() else "cpu")
    kw = dict(n_groups=cfg.n_groups, topk_groups=cfg.topk_groups, topk=cfg.topk,
              score_func=cfg.score, route_scale=cfg.route_scale)
    xs_all, wr = host_bits(x), host_bits(w_r)
    b = None if bias is None else bias.numpy().astype(np.float64)
    rng = np.random.default_rng(1000)
    cap = a.cpu_tokens or (8 if cfg.dim >= 4096 else 64)
    tok = np.sort(rng.choice(x.shape[0], size=min(cap, x.shape[0]), replace=False))
    r = O.route(O.router_logits(xs_all[tok], wr), b, **kw)
    w1, w3, w2, ws1, ws3, ws2 = w
    hw = {e: (host_bits(w1[e]), host_bits(w3[e]), host_bits(w2[e]))
          for e in sorted(set(r["idx"].ravel().tolist()))}
    shared = None if ws1 is None else (host_bits(ws1), host_bits(ws3), host_bits(ws2))

    def run(n):
        t0 = time.perf_counter()
        O.moe_forward(xs_all[tok[:n]], wr, b, lambda e: hw[e], shared, act_dtype=cfg.dtype, **kw)
        return time.perf_counter() - t0

    t_one = run(1)
    n_tok = int(max(1, min(len(tok), REFERENCE_BUDGET_S / max(t_one, 1e-6) / (a.warmup + a.steps))))
    rates = []
    for i in range(a.warmup + a.steps):
        dt = run(n_tok)
        if i >= a.warmup:
            rates.append(n_tok / dt)
    v = float(np.median(rates))
    cores = blas_threads()
    sample = (f"the same {n_tok} seeded tokens of the {cfg.name} batch every step (their routing "
              f"and experts, fp64 numpy oracle; sized to a ~{REFERENCE_BUDGET_S:.0f} s run); "
              f"median of {a.steps} steps")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": cfg.T / v * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": cfg.name, "T": cfg.T, "dim": cfg.dim,
                                            "experts": cfg.n_routed, "topk": cfg.topk},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def ours_arm(a, D):
    from mixture_experts_layer_42_b200 import binding as M
    cfg = workload(a)
    dev = torch.device("cuda", torch.cuda.current_device())
    x_cpu, w_r_cpu, bias_cpu = inputs.routing_inputs(cfg)
    x = x_cpu.to(dev)
    w_r = w_r_cpu.to(dev)
    bias = bias_cpu.to(dev) if bias_cpu is not None else None
    w = inputs.expert_weights(cfg, dev)
    T = cfg.T
    y = torch.empty(T, cfg.dim, dtype=cfg.torch_dtype, device=dev)
    idx = torch.empty(T, cfg.topk, dtype=torch.int32, device=dev)
    ws = M.alloc_workspace(cfg, T, dev)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    M.moe_select_expert_kernel({"auto": M.MOE_EXPERT_KERNEL_AUTO, "simt": M.MOE_EXPERT_KERNEL_SIMT,
                                "one_cta": M.MOE_EXPERT_KERNEL_TCGEN05,
                                "pair": M.MOE_EXPERT_KERNEL_TCGEN05_PAIR}[a.expert_kernel])
    launches = M.moe_forward_launch_count(cfg, T)

    def step(xin=x, idx_out=None):
        M.moe_forward(cfg, xin, w_r, bias, *w, y, ws, idx_out=idx_out, stream=stream)

    with torch.cuda.stream(stream):
        step(idx_out=idx)
    torch.cuda.synchronize()
    if M.moe_check_error(ws, stream) != M.MOE_OK:
        raise RuntimeError("device error word set after the first forward")
    counts = torch.bincount(idx.flatten().long(), minlength=cfg.n_routed).cpu()
    n_active = int((counts > 0).sum().item())
    routing = {"active_experts": n_active, "max_count": int(counts.max()), "min_count": int(counts.min()),
               "mean_count": T * cfg.topk / cfg.n_routed,
               "rows_useful_in_128_row_tiles": float(counts.sum() / (128 * ((counts + 127) // 128).sum()))}
    if cfg.name == "v3_zipf":
        routing.update(zipf_s=inputs.ZIPF_S, zipf_beta=inputs.ZIPF_BETA)

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except AttributeError:
        pass
    clocks = Clocks() if D.rank == 0 else None

    # ------------------------------------------------------------ device-timed loop
    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    D.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # per-kernel CUDA events on one step in `every` (about 20 steps), inside
    # the same timed loop: events between every kernel of every step would
    # cost the decode step ~1%
    every = max(1, a.steps // 20)
    M.moe_stage_timing_begin_every((a.steps + every - 1) // every, every)
    wall0 = time.time()
    ev0.record(stream)
    for _ in range(a.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    D.barrier()
    torch.cuda.synchronize()
    n_rec, stage_ms = M.moe_stage_timing_end()
    ms = D.max(ev0.elapsed_time(ev1))
    if M.moe_check_error(ws, stream) != M.MOE_OK:
        raise RuntimeError("device error word set during the timed loop")

    # ------------------------------------------------------------ end to end (host buffers)
    # Each step copies its x in from pinned host memory and its y back out.
    # A serving loop overlaps them: the H2D of step i+1 (copy stream) and the
    # D2H of step i (a second copy stream) run under the compute of the
    # neighbouring steps, with double-buffered device x and y.
    x_h = x_cpu.pin_memory()
    y_h = [torch.empty(T, cfg.dim, dtype=cfg.torch_dtype).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(x) for _ in range(2)]
    y_d = [torch.empty_like(y) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e_run(n):
        ev = lambda: torch.cuda.Event()
        x_ready = [ev(), ev()]
        done = [ev(), ev()]       # compute of the step that used buffer b
        y_out = [ev(), ev()]      # D2H of buffer b finished
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        h2d.wait_event(start)
        with torch.cuda.stream(h2d):
            x_d[0].copy_(x_h, non_blocking=True)
            x_ready[0].record(h2d)
        for i in range(n):
            b = i & 1
            stream.wait_event(x_ready[b])
            if i >= 2:
                stream.wait_event(y_out[b])
            M.moe_forward(cfg, x_d[b], w_r, bias, *w, y_d[b], ws, stream=stream)
            done[b].record(stream)
            if i + 1 < n:
                nb = (i + 1) & 1
                if i >= 1:
                    h2d.wait_event(done[nb])
                with torch.cuda.stream(h2d):
                    x_d[nb].copy_(x_h, non_blocking=True)
                    x_ready[nb].record(h2d)
            d2h.wait_event(done[b])
            with torch.cuda.stream(d2h):
                y_h[b].copy_(y_d[b], non_blocking=True)
                y_out[b].record(d2h)
        stream.wait_event(y_out[(n - 1) & 1])
        if n >= 2:
            stream.wait_event(y_out[n & 1])
        end.record(stream)
        return start, end

    e2e_run(a.warmup)
    torch.cuda.synchronize()
    D.barrier()
    torch.cuda.synchronize()
    e0, e1 = e2e_run(a.steps)
    torch.cuda.synchronize()
    D.barrier()
    torch.cuda.synchronize()
    ms_e2e = D.max(e0.elapsed_time(e1))
    if not torch.equal(y_h[(a.steps - 1) & 1], y.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")
    ck = clocks.stop(wall0, wall1, uuid) if clocks else None

    N = D.world
    value = N * T * a.steps / (ms / 1e3)
    e2e = N * T * a.steps / (ms_e2e / 1e3)

    l2 = l2_note(cfg, n_active)
    pk, pk_kind = peaks()
    flops, byts, t_roof, bound = layer_roofline(cfg, n_active, pk)
    ms_step = ms / a.steps
    per_kernel_ms = {k: v / max(n_rec, 1) for k, v in stage_ms.items()}
    dom = max(per_kernel_ms, key=per_kernel_ms.get)
    up_f, up_b = up_kernel_work(cfg, n_active)
    t_up = per_kernel_ms["experts_up"] / 1e3
    long_run = ms > 1000.0
    tpk = pk.get("bf16_tflops_sustained" if long_run else "bf16_tflops")
    if up_f / (tpk * 1e12) >= up_b / (pk["hbm_gbs"] * 1e9):
        roof = {"bound": "tensor", "achieved": up_f / t_up / 1e12, "peak": tpk, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": up_b / t_up / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    tr = traffic_for("grouped_tc_kernel_up", cfg.name)
    roof.update({"traffic": tr, "kernel": "experts_up (grouped_tc_kernel<UP>)",
                 "algorithmic_flops": up_f, "algorithmic_bytes": up_b,
                 "ms_per_launch": per_kernel_ms["experts_up"],
                 "peak_source": f"{pk_kind} ({'sustained' if long_run and roof['bound'] == 'tensor' else 'burst'})"})

    cpu = None
    if D.rank == 0 and N == 1 and not a.no_cpu_baseline:
        n_tok = a.cpu_tokens or (12 if cfg.dim >= 4096 else 96)
        rate, n, n_used, _ = oracle_rate(cfg, x_cpu, w_r_cpu, bias_cpu, w, n_tok)
        cpu = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n} seeded tokens of the {cfg.name} batch ({n_used} experts): their routing "
                         f"and expert math in the fp64 numpy oracle, one run"}

    if D.rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": N, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "seed": cfg.seed, "T": T, "dim": cfg.dim,
                       "experts": cfg.n_routed,
                       "groups": f"{cfg.n_groups}/{cfg.topk_groups}", "topk": cfg.topk,
                       "moe_inter": cfg.moe_inter, "shared_inter": cfg.shared_inter,
                       "score": cfg.score, "parallelism": f"replicas x{N}",
                       "expert_kernel": a.expert_kernel,
                       "l2": l2},
            "e2e": {"value": e2e, "unit": UNIT, "h2d_bytes_per_step": x.numel() * x.element_size(),
                    "d2h_bytes_per_step": y.numel() * y.element_size()},
            "gpu_launches": launches * a.steps * N,
            "roofline": roof,
            "layer_roofline": {"flops": flops, "bytes": byts, "bound": bound,
                               "t_roofline_ms": t_roof * 1e3, "frac": t_roof * 1e3 / ms_step,
                               "peak_source": f"{pk_kind} (burst)",
                               # the same against the seconds-long (power-capped) GEMM peak
                               "frac_sustained": layer_roofline(
                                   cfg, n_active, dict(pk, bf16_tflops=pk["bf16_tflops_sustained"]))[2]
                               * 1e3 / ms_step,
                               # and against the nominal B200 figures (8 TB/s HBM3e, 2.25
                               # PFLOP/s dense bf16), for context
                               "frac_nominal": layer_roofline(cfg, n_active, NOMINAL_PEAKS)[2]
                               * 1e3 / ms_step},
            "kernels_ms": per_kernel_ms, "kernels_ms_steps": {"recorded": n_rec, "every": every},
            "dominant_kernel": dom, "active_experts": n_active,
            "routing": routing,
            "cpu_baseline": cpu, "clocks": ck,
        }
        print(json.dumps(line), flush=True)


def main():
    a = parse()
    D = Dist()
    if D.world != a.gpus:
        raise SystemExit(f"--gpus {a.gpus} but {D.world} process(es) were launched "
                         "(use torchrun --nproc-per-node N for N > 1)")
    try:
        if a.impl == "reference":
            reference_arm(a, D)
        else:
            ours_arm(a, D)
    finally:
        D.close()


if __name__ == "__main__":
    main()
