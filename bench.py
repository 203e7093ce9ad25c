#!/usr/bin/env python
"""Throughput of the DeepSeek-V3-style MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]
    python bench.py --routing-only [--config NAME] [--iters N]

One step is one pass of the whole layer (router, dispatch, grouped SwiGLU
experts, combine) over one batch of the workload through the C ABI
(moe_forward), with inputs resident in HBM. The default workload is the
DeepSeek-V3-shape decode batch (T=128, D=7168, 256 experts, top-8, I=2048, one
shared expert, bf16); --config v3_prefill etc. select the other workloads.
Every step streams more expert weights than the 126 MB L2 holds (14-22 GB at
the V3 shape), so no L2 flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the layer (the layer does not shard: replicas only); value is the
tokens of all ranks over the slowest rank's device time.

Printed (rank 0, one JSON line): tokens/s from CUDA events on the launching
stream; e2e tokens/s through the same C call with x copied in from pinned host
memory and y copied back every step; the roofline of the dominant kernel from
per-kernel CUDA events recorded in a separate untimed pass after the timed
loop (which records no other event); the layer roofline; the CPU oracle's rate on a bounded token sample (N=1
only); SM clocks sampled during the run. At N=1 the line also carries
`workloads`: the same device-timed measurements for the other workloads (V3
prefill, the Zipf-skewed prefill, the softmax layer, and the V3 decode and
prefill batches with FP8 expert weights), each timed for about a second.

--impl reference times the CPU oracle (the plain fp64 statement of the layer)
on the host cores, on the same workload, metric and unit.

--routing-only runs the layer's non-expert kernels (router, dispatch,
combine) on a workload's shapes without allocating any expert weights, so
that a profiler can capture them with a small device footprint; it prints no
measurement.
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


def parse(argv=None):
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
    ap.add_argument("--fp8-kernel", default="auto", choices=["auto", "tokens_on_n", "tokens_on_m"],
                    help="form of the FP8 expert GEMMs (moe_select_fp8_kernel)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' measurements (N=1 only runs them)")
    ap.add_argument("--routing-only", action="store_true",
                    help="run only the router, dispatch and combine kernels (for profilers)")
    ap.add_argument("--iters", type=int, default=3, help="iterations of --routing-only")
    return ap.parse_args(argv)


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


def weight_bytes(cfg):
    """Bytes per expert weight element: the activation dtype's, or 1 + the
    share of a 4-byte scale per 128 x 128 block for FP8 weights."""
    if cfg.fp8:
        return 1.0 + 4.0 / (128 * 128)
    return 4.0 if cfg.dtype == "f32" else 2.0


def layer_roofline(cfg, n_active, pk):
    """Algorithmic FLOPs and bytes of one layer pass (router, routed and
    shared experts; each active expert's weights, the shared weights, W_r,
    x and y counted once). FP8 expert weights count their e4m3 bytes and
    scales, and their products run at twice the bf16 tensor peak."""
    T, D, E, k, I, Is = cfg.T, cfg.dim, cfg.n_routed, cfg.topk, cfg.moe_inter, cfg.shared_inter
    ab = 4 if cfg.dtype == "f32" else 2
    flops = 2 * T * D * E + 6 * T * k * D * I + 6 * T * D * Is
    byts = (n_active * 3 * I * D + 3 * Is * D) * weight_bytes(cfg) + (E * D + 2 * T * D) * ab
    t_f = (2 * T * D * E + (6 * T * k * D * I + 6 * T * D * Is) / (2 if cfg.fp8 else 1)) / \
        (pk["bf16_tflops"] * 1e12)
    t_b = byts / (pk["hbm_gbs"] * 1e9)
    return flops, byts, max(t_f, t_b), "tensor" if t_f >= t_b else "hbm"


def l2_note(cfg, n_active):
    """How the timed loop stands to the 126 MB L2: the weights every step
    streams exceed it (no flush needed), or the workload fits (a small,
    launch-bound case)."""
    wbytes = (n_active * 3 * cfg.moe_inter + 3 * cfg.shared_inter) * cfg.dim * weight_bytes(cfg)
    if wbytes > 126e6:
        return f"inputs larger than L2 (every step streams the active experts' weights, {wbytes / 1e9:.1f} GB)"
    return (f"inputs fit in L2 ({wbytes / 1e6:.2f} MB of weights, no flush): a small, launch-bound "
            "workload, not the roofline case")


def up_kernel_work(cfg, n_active):
    """Algorithmic FLOPs and bytes of one launch of the grouped up-projection
    (w1 and w3 of every active expert and of the shared expert and x read
    once -- the routed rows are gathered from x --, h and h_shared written
    once)."""
    T, D, k, I, Is = cfg.T, cfg.dim, cfg.topk, cfg.moe_inter, cfg.shared_inter
    ab = 4 if cfg.dtype == "f32" else 2
    flops = 4 * T * k * D * I + 4 * T * D * Is
    if cfg.fp8:   # e4m3 x and h (1 byte each) and the weights' bytes with scales
        byts = (n_active * 2 * I * D + 2 * Is * D) * weight_bytes(cfg) + T * D + T * k * I + T * Is
    else:
        byts = (n_active * 2 * I * D + 2 * Is * D + T * D + T * k * I + T * Is) * ab
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

def config_dict(cfg, N, expert_kernel, l2):
    """The `config` object of both arms' lines: the workload and its shape."""
    return {"workload": cfg.name, "seed": cfg.seed, "T": cfg.T, "dim": cfg.dim,
            "experts": cfg.n_routed, "groups": f"{cfg.n_groups}/{cfg.topk_groups}",
            "topk": cfg.topk, "moe_inter": cfg.moe_inter, "shared_inter": cfg.shared_inter,
            "score": cfg.score, "parallelism": f"replicas x{N}", "expert_kernel": expert_kernel,
            "expert_weights": "fp8 e4m3, 128x128 power-of-two block scales" if cfg.fp8 else cfg.dtype,
            **({"fp8_gemm": "tokens on M" if fp8_tokens_on_m(cfg) else "tokens on N"} if cfg.fp8 else {}),
            "l2": l2}


def reference_arm(a, D):
    """The CPU oracle, as it stands, on the host cores (rank 0 only). Every
    step runs it on the same seeded token sample (the experts those tokens
    use are copied to the host once, outside all timing); the sample is sized
    from a one-token probe so that warm-up and timed steps together take
    about REFERENCE_BUDGET_S seconds. ms_per_step is the measured wall time
    of one step (the sample's tokens), value the sample's tokens per second."""
    if D.rank != 0:
        return
    from oracle import moe_oracle as O
    cfg = workload(a)
    if cfg.fp8:
        raise SystemExit("the reference arm times the oracle's bf16 layer; pick a bf16 workload")
    x, w_r, bias = inputs.routing_inputs(cfg)
    w = inputs.expert_weights(cfg, "cuda" if torch.cuda.is_available() else "cpu")
    kw = dict(n_groups=cfg.n_groups, topk_groups=cfg.topk_groups, topk=cfg.topk,
              score_func=cfg.score, route_scale=cfg.route_scale)
    xs_all, wr = host_bits(x), host_bits(w_r)
    b = None if bias is None else bias.numpy().astype(np.float64)
    # the experts every token of the batch uses (for the config's L2 note)
    n_active = len(set(O.route(O.router_logits(xs_all, wr), b, **kw)["idx"].ravel().tolist()))
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
    dts = []
    for i in range(a.warmup + a.steps):
        dt = run(n_tok)
        if i >= a.warmup:
            dts.append(dt)
    dt_med = float(np.median(dts))
    v = n_tok / dt_med
    cores = blas_threads()
    sample = (f"the same {n_tok} seeded tokens of the {cfg.name} batch every step (their routing "
              f"and experts, fp64 numpy oracle; sized to a ~{REFERENCE_BUDGET_S:.0f} s run); "
              f"median of {a.steps} steps; ms_per_step is the measured time of one such step")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": dt_med * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": config_dict(cfg, a.gpus, a.expert_kernel, l2_note(cfg, n_active)),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class Setup:
    """Device copies of one workload's inputs, its workspace and outputs."""

    def __init__(self, cfg, dev, w=None):
        from mixture_experts_layer_42_b200 import binding as M
        self.M, self.cfg, self.dev = M, cfg, dev
        self.x_cpu, self.w_r_cpu, self.bias_cpu = inputs.routing_inputs(cfg)
        self.x = self.x_cpu.to(dev)
        self.w_r = self.w_r_cpu.to(dev)
        self.bias = self.bias_cpu.to(dev) if self.bias_cpu is not None else None
        self.w = w if w is not None else inputs.expert_weights(cfg, dev)
        self.y = torch.empty(cfg.T, cfg.dim, dtype=cfg.torch_dtype, device=dev)
        self.idx = torch.empty(cfg.T, cfg.topk, dtype=torch.int32, device=dev)
        self.stream = torch.cuda.Stream(device=dev)
        if cfg.fp8:
            # the drawn bf16 weights in the FP8 layout (the library's quantizer)
            self.q = []
            for t in self.w:
                if t is None:
                    self.q += [None, None]
                    continue
                a = t.reshape(-1, t.shape[-1])
                q = torch.empty(a.shape, dtype=torch.uint8, device=dev)
                s = torch.empty(a.shape[0] // 128, a.shape[1] // 128, dtype=torch.float32, device=dev)
                M.moe_quantize_fp8(cfg, a, 128, q, s)
                self.q += [q, s]
            q = self.q
            self.fw = M.fp8_weights(q[0], q[2], q[4], q[1], q[3], q[5], q[6], q[8], q[10], q[7], q[9], q[11])
            self.ws = M.alloc_workspace_fp8(cfg, cfg.T, dev)
        else:
            self.ws = M.alloc_workspace(cfg, cfg.T, dev)
        torch.cuda.synchronize()

    def step(self, xin=None, y=None, idx_out=None):
        if self.cfg.fp8:
            self.M.moe_forward_fp8(self.cfg, self.x if xin is None else xin, self.w_r, self.bias, self.fw,
                                   self.y if y is None else y, self.ws, idx_out=idx_out,
                                   stream=self.stream)
            return
        self.M.moe_forward(self.cfg, self.x if xin is None else xin, self.w_r, self.bias, *self.w,
                           self.y if y is None else y, self.ws, idx_out=idx_out, stream=self.stream)

    def routing(self):
        """Route once, check the error word, summarise the expert counts."""
        cfg, T = self.cfg, self.cfg.T
        with torch.cuda.stream(self.stream):
            self.step(idx_out=self.idx)
        torch.cuda.synchronize()
        if self.M.moe_check_error(self.ws, self.stream) != self.M.MOE_OK:
            raise RuntimeError(f"{cfg.name}: device error word set after the first forward")
        counts = torch.bincount(self.idx.flatten().long(), minlength=cfg.n_routed).cpu()
        n_active = int((counts > 0).sum().item())
        routing = {"active_experts": n_active, "max_count": int(counts.max()),
                   "min_count": int(counts.min()), "mean_count": T * cfg.topk / cfg.n_routed,
                   "rows_useful_in_128_row_tiles":
                       float(counts.sum() / (128 * ((counts + 127) // 128).sum()))}
        if cfg.name == "v3_zipf":
            routing.update(zipf_s=inputs.ZIPF_S, zipf_beta=inputs.ZIPF_BETA)
        return n_active, routing


def device_timed(S, D, steps, warmup, uuid, clocks_on):
    """Time `steps` forwards on the device after `warmup` untimed ones:
    barrier + synchronize on both sides, CUDA events on the launching stream,
    max over ranks; the timed loop records no other event. The per-kernel
    times come from a separate, untimed pass right after it (a tenth of the
    steps, 2 to 20), whose forwards record an event between every two kernels
    (and launch the up-projection as an ordinary launch, so each interval
    holds one kernel). Returns (ms, kernels_ms per launch, kernels_ms_steps,
    clocks)."""
    M = S.M
    clocks = Clocks() if clocks_on else None
    for _ in range(warmup):
        S.step()
    torch.cuda.synchronize()
    D.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.time()
    ev0.record(S.stream)
    for _ in range(steps):
        S.step()
    ev1.record(S.stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    D.barrier()
    torch.cuda.synchronize()
    ms = D.max(ev0.elapsed_time(ev1))
    n_pass = min(20, max(2, steps // 10))
    M.moe_stage_timing_begin(n_pass)
    for _ in range(n_pass):
        S.step()
    torch.cuda.synchronize()
    n_rec, stage_ms = M.moe_stage_timing_end()
    if M.moe_check_error(S.ws, S.stream) != M.MOE_OK:
        raise RuntimeError(f"{S.cfg.name}: device error word set during the timed loop")
    ck = clocks.stop(wall0, wall1, uuid) if clocks else None
    rec = {"recorded": n_rec, "pass": "separate, untimed, after the timed loop; a recorded "
                                      "forward launches each kernel only after the one before"}
    return ms, {k: v / max(n_rec, 1) for k, v in stage_ms.items()}, rec, ck


def fp8_tokens_on_m(cfg):
    """Whether moe_forward_fp8 runs this batch's expert GEMMs with the tokens
    on the MMA's M side, as the library resolves it (its selection, or by the
    average rows per expert)."""
    from mixture_experts_layer_42_b200 import binding as M
    return M.moe_fp8_kernel_for(cfg, cfg.T) == M.MOE_FP8_KERNEL_TOKENS_ON_M


def rooflines(cfg, n_active, ms_step, per_kernel_ms, long_run):
    """The dominant kernel's roofline object and the layer roofline object."""
    pk, pk_kind = peaks()
    flops, byts, t_roof, bound = layer_roofline(cfg, n_active, pk)
    up_f, up_b = up_kernel_work(cfg, n_active)
    t_up = per_kernel_ms["experts_up"] / 1e3
    tpk = pk.get("bf16_tflops_sustained" if long_run else "bf16_tflops")
    if cfg.fp8:   # e4m3 products: the measured bf16 peak times the nominal 4.5 / 2.25 ratio
        tpk = 2.0 * tpk
    if up_f / (tpk * 1e12) >= up_b / (pk["hbm_gbs"] * 1e9):
        roof = {"bound": "tensor", "achieved": up_f / t_up / 1e12, "peak": tpk, "unit": "TFLOP/s"}
        nominal = NOMINAL_PEAKS["bf16_tflops"] * (2 if cfg.fp8 else 1)
    else:
        roof = {"bound": "hbm", "achieved": up_b / t_up / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
        nominal = NOMINAL_PEAKS["hbm_gbs"]
    roof["frac"] = roof["achieved"] / roof["peak"]
    kname = ("grouped_fp8m_kernel_up" if fp8_tokens_on_m(cfg) else "grouped_fp8_kernel_up") if cfg.fp8 \
        else "grouped_tc_kernel_up"
    roof.update({"traffic": traffic_for(kname, cfg.name),
                 "kernel": f"experts_up ({kname.replace('_up', '<UP>')})",
                 "algorithmic_flops": up_f, "algorithmic_bytes": up_b,
                 "ms_per_launch": per_kernel_ms["experts_up"],
                 "peak_source": f"{pk_kind} ({'sustained' if long_run and roof['bound'] == 'tensor' else 'burst'})",
                 # against the nominal B200 figure (8 TB/s HBM3e, 2.25 PFLOP/s dense bf16)
                 "peak_nominal": nominal, "frac_nominal": roof["achieved"] / nominal})
    if roof["frac"] > 1.0:
        roof["note"] = ("above 1: the measured peak is a copy (read + write) bandwidth, and a "
                        "read-mostly weight stream draws a little more from HBM; frac_nominal is "
                        "the fraction of the nominal bandwidth")
    layer = {"flops": flops, "bytes": byts, "bound": bound, "t_roofline_ms": t_roof * 1e3,
             "frac": t_roof * 1e3 / ms_step, "peak_source": f"{pk_kind} (burst)",
             # the same against the seconds-long (power-capped) GEMM peak
             "frac_sustained": layer_roofline(
                 cfg, n_active, dict(pk, bf16_tflops=pk["bf16_tflops_sustained"]))[2] * 1e3 / ms_step,
             # and against the nominal B200 figures, for context
             "frac_nominal": layer_roofline(cfg, n_active, NOMINAL_PEAKS)[2] * 1e3 / ms_step}
    return roof, layer


def other_workload(name, a, D, dev, uuid, shared_weights):
    """Device-timed measurement of one more workload (N=1): about a second of
    timed steps, with the same per-kernel events and clock samples."""
    cfg = inputs.CONFIGS[name]
    S = Setup(cfg, dev, w=shared_weights)
    n_active, routing = S.routing()
    # size the timed loop to about a second (at least --steps)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(S.stream)
    for _ in range(3):
        S.step()
    t1.record(S.stream)
    torch.cuda.synchronize()
    est = t0.elapsed_time(t1) / 3
    steps = int(min(2000, max(a.steps, 1000.0 / max(est, 1e-3))))
    ms, per_kernel_ms, rec, ck = device_timed(S, D, steps, a.warmup, uuid, True)
    ms_step = ms / steps
    roof, layer = rooflines(cfg, n_active, ms_step, per_kernel_ms, ms > 1000.0)
    del S
    return {"config": config_dict(cfg, D.world, a.expert_kernel, l2_note(cfg, n_active)),
            "steps": steps, "warmup": a.warmup, "ms_per_step": ms_step,
            "value": cfg.T * steps / (ms / 1e3), "unit": UNIT, "roofline": roof,
            "layer_roofline": layer, "kernels_ms": per_kernel_ms,
            "kernels_ms_steps": rec,
            "dominant_kernel": max(per_kernel_ms, key=per_kernel_ms.get), "routing": routing,
            "clocks": ck}


def ours_arm(a, D):
    from mixture_experts_layer_42_b200 import binding as M
    cfg = workload(a)
    dev = torch.device("cuda", torch.cuda.current_device())
    M.moe_select_expert_kernel({"auto": M.MOE_EXPERT_KERNEL_AUTO, "simt": M.MOE_EXPERT_KERNEL_SIMT,
                                "one_cta": M.MOE_EXPERT_KERNEL_TCGEN05,
                                "pair": M.MOE_EXPERT_KERNEL_TCGEN05_PAIR}[a.expert_kernel])
    M.moe_select_fp8_kernel({"auto": M.MOE_FP8_KERNEL_AUTO, "tokens_on_n": M.MOE_FP8_KERNEL_TOKENS_ON_N,
                             "tokens_on_m": M.MOE_FP8_KERNEL_TOKENS_ON_M}[a.fp8_kernel])
    S = Setup(cfg, dev)
    T = cfg.T
    launches = M.moe_forward_launch_count(cfg, T)
    n_active, routing = S.routing()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except AttributeError:
        pass

    # ------------------------------------------------------------ device-timed loop
    ms, per_kernel_ms, rec, ck = device_timed(S, D, a.steps, a.warmup, uuid, D.rank == 0)

    # ------------------------------------------------------------ end to end (host buffers)
    # Each step copies its x in from pinned host memory and its y back out.
    # A serving loop overlaps them: the H2D of step i+1 (copy stream) and the
    # D2H of step i (a second copy stream) run under the compute of the
    # neighbouring steps, with double-buffered device x and y.
    stream = S.stream
    x_h = S.x_cpu.pin_memory()
    y_h = [torch.empty(T, cfg.dim, dtype=cfg.torch_dtype).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(S.x) for _ in range(2)]
    y_d = [torch.empty_like(S.y) for _ in range(2)]
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
            S.step(xin=x_d[b], y=y_d[b])
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
    if not torch.equal(y_h[(a.steps - 1) & 1], S.y.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")

    N = D.world
    value = N * T * a.steps / (ms / 1e3)
    e2e = N * T * a.steps / (ms_e2e / 1e3)
    ms_step = ms / a.steps
    roof, layer = rooflines(cfg, n_active, ms_step, per_kernel_ms, ms > 1000.0)

    cpu = None
    if D.rank == 0 and N == 1 and not a.no_cpu_baseline:
        n_tok = a.cpu_tokens or (12 if cfg.dim >= 4096 else 96)
        rate, n, n_used, _ = oracle_rate(cfg, S.x_cpu, S.w_r_cpu, S.bias_cpu, S.w, n_tok)
        cpu = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{n} seeded tokens of the {cfg.name} batch ({n_used} experts): their routing "
                         f"and expert math in the fp64 numpy oracle, one run"}

    # ------------------------------------------------------------ the other workloads (N=1)
    others = None
    if N == 1 and not a.no_workloads and not a.tokens and not a.experts:
        others = {}
        for name in ("v3_prefill", "v3_zipf", "softmax_nogroup", "v3_decode_fp8", "v3_prefill_fp8"):
            if name == cfg.name:
                continue
            o = inputs.CONFIGS[name]
            # workloads of the same expert shapes and seed draw the same expert
            # weights (inputs.expert_weights): reuse the resident ones
            same = all(getattr(o, f) == getattr(cfg, f) for f in
                       ("dim", "n_routed", "moe_inter", "n_shared", "dtype", "seed"))
            others[name] = other_workload(name, a, D, dev, uuid, S.w if same else None)
            torch.cuda.empty_cache()

    if D.rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": N, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": config_dict(cfg, N, a.expert_kernel, l2_note(cfg, n_active)),
            "e2e": {"value": e2e, "unit": UNIT, "h2d_bytes_per_step": S.x.numel() * S.x.element_size(),
                    "d2h_bytes_per_step": S.y.numel() * S.y.element_size()},
            "gpu_launches": launches * a.steps * N,
            "roofline": roof,
            "layer_roofline": layer,
            "kernels_ms": per_kernel_ms, "kernels_ms_steps": rec,
            "dominant_kernel": max(per_kernel_ms, key=per_kernel_ms.get), "active_experts": n_active,
            "routing": routing,
            "cpu_baseline": cpu, "clocks": ck,
        }
        if others is not None:
            line["workloads"] = others
        print(json.dumps(line), flush=True)


def routing_only(a):
    """The layer's non-expert kernels -- router (moe_gate), dispatch
    (moe_dispatch, indices only, as moe_forward runs it) and combine
    (moe_combine) -- on a workload's shapes, without allocating any expert
    weights. A zeroed [T*k, D] buffer stands in for the expert outputs
    (combine reads rows of the same size and layout through pos), and x
    stands in for the shared expert's output. Each iteration launches the
    kernels once, in layer order, on one stream."""
    from mixture_experts_layer_42_b200 import binding as M
    cfg = workload(a)
    T, k, D, E = cfg.T, cfg.topk, cfg.dim, cfg.n_routed
    dev = torch.device("cuda")
    x, w_r, bias = inputs.routing_inputs(cfg, T)
    x, w_r = x.to(dev), w_r.to(dev)
    bias = None if bias is None else bias.to(dev)
    wts = torch.empty(T, k, dtype=torch.float32, device=dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    y_perm = torch.zeros(T * k, D, dtype=x.dtype, device=dev)
    s = x if cfg.shared_inter > 0 else None
    y = torch.empty_like(x)
    ws = M.alloc_workspace(cfg, T, dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    for _ in range(a.iters):
        M.moe_gate(cfg, x, w_r, bias, wts, idx, ws, stream=stream)
        M.moe_dispatch(cfg, idx, None, counts, offsets, src, pos, None, ws, stream=stream)
        M.moe_combine(cfg, y_perm, pos, wts, s, y, ws, stream=stream)
    stream.synchronize()
    st = M.moe_check_error(ws, stream=stream)
    if st != M.MOE_OK:
        raise SystemExit(f"device error word: {M.status_string(st)}")
    print(f"{cfg.name}: T={T} D={D} E={E} k={k}: {a.iters} x (gate, dispatch, combine) done; "
          f"active experts {int((counts > 0).sum())}, max count {int(counts.max())}", flush=True)


def main(argv=None):
    a = parse(argv)
    if a.routing_only:
        routing_only(a)
        return
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
