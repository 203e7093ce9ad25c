"""The benchmark's command-line contract on the CPU: the reference arm (the
CPU oracle timed on the host cores) prints exactly one JSON line with the
contract's keys, alone and as two torchrun ranks of which rank 0 alone
prints. The GPU arm's line is checked by running bench.py on a GPU."""

import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _json_lines(out: str):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check_reference_line(d, n_gpus):
    assert d["impl"] == "reference"
    assert d["metric"].startswith("MoE-layer tokens/sec")
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == n_gpus and d["steps"] == 2 and d["warmup"] == 1
    assert d["config"]["workload"] == "tiny_fp32"
    # the same config object the GPU arm prints for this workload
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_42_b200 import inputs
    cfg = inputs.CONFIGS["tiny_fp32"]
    assert d["config"] == bench.config_dict(cfg, n_gpus, "auto", bench.l2_note(cfg, cfg.n_routed))
    # ms_per_step is the measured time of one step of the sample, not T / value
    assert d["ms_per_step"] * 1e-3 * d["value"] <= cfg.T
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny_fp32",
                        "--steps", "2", "--warmup", "1"], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_reference_line(lines[0], 1)


def test_reference_arm_under_torchrun_prints_on_rank_0_only():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
                        "--impl", "reference", "--gpus", "2", "--config", "tiny_fp32", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_reference_line(lines[0], 2)


def test_gpu_count_must_match_the_launch():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--config",
                        "tiny_fp32", "--steps", "1", "--warmup", "0"], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0 and "--gpus 2" in r.stderr


def test_roofline_objects_and_the_note_above_one():
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_42_b200 import inputs
    cfg = inputs.CONFIGS["v3_decode"]
    up_f, up_b = bench.up_kernel_work(cfg, 158)
    pk, _ = bench.peaks()
    # a launch at exactly the HBM peak, then one faster than the copy peak
    t = up_b / (pk["hbm_gbs"] * 1e9) * 1e3
    roof, layer = bench.rooflines(cfg, 158, 2.2, {"experts_up": t}, False)
    assert roof["bound"] == "hbm" and abs(roof["frac"] - 1.0) < 1e-9 and "note" not in roof
    assert abs(roof["frac_nominal"] - pk["hbm_gbs"] / 8000.0) < 1e-9
    roof, _ = bench.rooflines(cfg, 158, 2.2, {"experts_up": 0.9 * t}, False)
    assert roof["frac"] > 1.0 and "note" in roof
    assert layer["bound"] == "hbm" and 0 < layer["frac_nominal"] < layer["frac"]
    # prefill is bound by the tensor cores
    p = inputs.CONFIGS["v3_prefill"]
    roof, layer = bench.rooflines(p, 256, 8.0, {"experts_up": 5.0}, True)
    assert roof["bound"] == "tensor" and roof["peak_source"].endswith("(sustained)")
    assert layer["bound"] == "tensor" and layer["frac_sustained"] > layer["frac"]


def test_l2_note_states_how_the_timed_loop_meets_l2():
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_42_b200 import inputs
    big = bench.l2_note(inputs.CONFIGS["v3_decode"], 158)
    assert big.startswith("inputs larger than L2") and "14.0 GB" in big   # 158 experts + shared
    small = bench.l2_note(inputs.CONFIGS["tiny_fp32"], 16)
    assert small.startswith("inputs fit in L2")
    # the rest of the roofline inputs the GPU arm builds its line from
    flops, byts, t, bound = bench.layer_roofline(inputs.CONFIGS["v3_decode"], 158, bench.NOMINAL_PEAKS)
    assert bound == "hbm" and t > 0


def test_fp8_rooflines_use_twice_the_bf16_peak_and_name_the_form():
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_42_b200 import inputs
    pk, _ = bench.peaks()
    dec, pre = inputs.CONFIGS["v3_decode_fp8"], inputs.CONFIGS["v3_prefill_fp8"]
    # the form the library picks: tokens on M above 16 rows per expert on average
    assert not bench.fp8_tokens_on_m(dec) and bench.fp8_tokens_on_m(pre)
    assert bench.config_dict(dec, 1, "auto", "")["fp8_gemm"] == "tokens on N"
    assert bench.config_dict(pre, 1, "auto", "")["fp8_gemm"] == "tokens on M"
    # e4m3 products at twice the bf16 peak, weights at one byte (and a scale per block)
    f16, b16, t16, _ = bench.layer_roofline(inputs.CONFIGS["v3_prefill"], 229, pk)
    f8, b8, t8, bound = bench.layer_roofline(pre, 229, pk)
    assert f8 == f16 and bound == "tensor" and b8 < 0.55 * b16
    t_router = 2 * pre.T * pre.dim * pre.n_routed / (pk["bf16_tflops"] * 1e12)   # stays bf16
    assert abs(t8 - (t_router + (t16 - t_router) / 2)) < 1e-12
    up_f, _ = bench.up_kernel_work(pre, 229)
    roof, _ = bench.rooflines(pre, 229, 5.6, {"experts_up": 3.0}, False)
    assert roof["bound"] == "tensor" and roof["peak"] == 2 * pk["bf16_tflops"]
    assert abs(roof["achieved"] - up_f / 3e-3 / 1e12) < 1e-6
    assert roof["kernel"] == "experts_up (grouped_fp8m_kernel<UP>)"
    roof, _ = bench.rooflines(dec, 158, 1.13, {"experts_up": 0.72}, False)
    assert roof["bound"] == "hbm" and roof["kernel"] == "experts_up (grouped_fp8_kernel<UP>)"
