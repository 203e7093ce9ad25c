"""Planted mistakes: each case edits a copy of the oracle's source to plant one
plausible error (a dropped term, a wrong sign, a swapped operand, a wrong
index or order), loads the copy as a separate module on the CPU, and checks
that at least one of the oracle's pins fails on it. This shows the pins are
sharp enough to catch that class of error."""

import importlib.util
import inspect
import os
import types

import pytest

from oracle import moe_oracle
from tests import test_oracle_ep as TEP
from tests import test_oracle_experts as TE
from tests import test_oracle_fp8 as TF8
from tests import test_oracle_routing as TR

SRC = inspect.getsource(moe_oracle)

# (name, original text, planted text, pins that must catch it)
MUTATIONS = [
    ("group score max instead of top-2 sum", "gscore = top2.sum(axis=-1)", "gscore = top2[:, :, 0]",
     [TR.test_golden_sigmoid_groups]),
    ("weights from biased scores", "w = np.take_along_axis(s, idx, axis=-1)",
     "w = np.take_along_axis(np.where(np.isinf(b), 0, b), idx, axis=-1)",
     [TR.test_golden_sigmoid_groups]),
    ("no renormalisation", "w = w / w.sum(axis=-1, keepdims=True)", "w = w",
     [TR.test_golden_sigmoid_groups]),
    ("route_scale dropped", "w = w * route_scale", "w = w",
     [TR.test_golden_sigmoid_groups]),
    ("no group mask", "b = np.where(np.repeat(masked, per, axis=-1), -np.inf, b)", "b = b",
     [TR.test_golden_sigmoid_groups]),
    ("strided instead of contiguous groups", "blocks = b.reshape(T, n_groups, per)",
     "blocks = b.reshape(T, per, n_groups).transpose(0, 2, 1)",
     [TR.test_golden_sigmoid_groups]),
    ("bias ignored for selection",
     "b = s + np.asarray(bias, dtype=np.float64)[None, :] if bias is not None else s.copy()",
     "b = s.copy()", [TR.test_golden_sigmoid_groups]),
    ("sigmoid sign flipped", "return 1.0 / (1.0 + np.exp(-z))", "return 1.0 / (1.0 + np.exp(z))",
     [TR.test_golden_sigmoid_groups]),
    ("softmax over the wrong axis", "m = z.max(axis=-1, keepdims=True)\n    p = np.exp(z - m)\n    return p / p.sum(axis=-1, keepdims=True)",
     "m = z.max(axis=0, keepdims=True)\n    p = np.exp(z - m)\n    return p / p.sum(axis=0, keepdims=True)",
     [TR.test_golden_softmax]),
    ("ties go to the higher index", 'return np.argsort(-v, axis=-1, kind="stable")',
     'return v.shape[-1] - 1 - np.argsort(-v[..., ::-1], axis=-1, kind="stable")',
     [TR.test_zero_router_softmax_ties_to_lowest_index]),
    ("dispatch order reversed within an expert", "for q in range(T * k):", "for q in reversed(range(T * k)):",
     [TR.test_golden_dispatch]),
    ("exclusive scan off by one", "offsets[1:] = np.cumsum(counts)", "offsets[1:] = np.cumsum(counts) - counts",
     [TR.test_golden_dispatch]),
    ("silu replaced by sigmoid", "return u / (1.0 + np.exp(-u))", "return 1.0 / (1.0 + np.exp(-u))",
     [TE.test_identity_expert_closed_form]),
    ("w1 and w3 swapped", "a = xr @ to_f64(w1).T\n    c = xr @ to_f64(w3).T",
     "a = xr @ to_f64(w3).T\n    c = xr @ to_f64(w1).T", [TE.test_single_expert_is_dense_swiglu]),
    ("w2 transposed", "h @ to_f64(w2).T", "h @ to_f64(w2)[:h.shape[1], :h.shape[1]]",
     [TE.test_layer_matches_library_per_token]),
    ("combine uses slot 0's weight", "y[r] += out * ws[r, j][:, None]", "y[r] += out * ws[r, 0][:, None]",
     [TE.test_identity_expert_closed_form]),
    ("shared expert subtracted", "y += swiglu(xs, ws1, ws3, ws2", "y -= swiglu(xs, ws1, ws3, ws2",
     [TE.test_zero_w1_gives_shared_only]),
    ("bf16 keeps 7 bits", "np.round(m * 256.0) / 256.0", "np.round(m * 128.0) / 128.0",
     [TR.test_round_bf16_matches_torch]),
    ("bf16 truncates", "np.round(m * 256.0) / 256.0", "np.trunc(m * 256.0) / 256.0",
     [TR.test_round_bf16_matches_torch]),
    ("fp32 rounding skipped",
     "return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)",
     "return np.asarray(v, dtype=np.float64)", [TR.test_round_f32_known_values]),
    ("fp32 rounding to half precision", "astype(np.float32).astype(np.float64)",
     "astype(np.float16).astype(np.float64)", [TR.test_round_f32_known_values]),
    ("margin ignores the group gap",
     "margin = np.minimum(margin, gs[:, topk_groups - 1] - gs[:, topk_groups])", "margin = margin",
     [TR.test_golden_group_gap_decides_margin, TR.pin_brute_force_margins]),
    ("margin reaches the (k+2)-th expert", "order[:, :min(topk + 1, E)]", "order[:, :min(topk + 2, E)]",
     [TR.pin_brute_force_margins]),
    ("margin skips the best expert left out", "order[:, :min(topk + 1, E)]", "order[:, :topk]",
     [TR.test_golden_softmax, TR.pin_brute_force_margins]),
    ("margin from unbiased scores", "ranked = np.take_along_axis(b, order", "ranked = np.take_along_axis(s, order",
     [TR.test_golden_sigmoid_groups, TR.pin_brute_force_margins]),
    ("expert block drops its last expert",
     "per = n_experts // world_size\n    return range(rank * per, (rank + 1) * per)",
     "per = n_experts // world_size\n    return range(rank * per, (rank + 1) * per - 1)",
     [TEP.pin_ep_partials]),
    ("every rank adds the whole shared MLP",
     "y += swiglu(xs, np.asarray(ws1)[f], np.asarray(ws3)[f], np.asarray(ws2)[:, f],",
     "y += swiglu(xs, np.asarray(ws1), np.asarray(ws3), np.asarray(ws2),", [TEP.pin_ep_partials]),
    ("shared slice takes rows of ws2", "np.asarray(ws2)[:, f]", "np.asarray(ws2)[f, :].T",
     [TEP.pin_ep_partials]),
    ("e4m3 keeps 4 mantissa bits", "normal = np.ldexp(np.round(m * 16.0) / 16.0, e)",
     "normal = np.ldexp(np.round(m * 32.0) / 32.0, e)", [TF8.pin_fp8]),
    ("e4m3 subnormal step 2^-8", "sub = np.round(v * 512.0) / 512.0", "sub = np.round(v * 256.0) / 256.0",
     [TF8.pin_fp8]),
    ("fp8 scale one step too large", "s = np.maximum(e - 9 + (2.0 * m > 1.75)", "s = np.maximum(e - 8 + (2.0 * m > 1.75)",
     [TF8.pin_fp8]),
    ("fp8 scale ignores the 1.75 boundary", "s = np.maximum(e - 9 + (2.0 * m > 1.75)",
     "s = np.maximum(e - 9 + (2.0 * m > 1.5)", [TF8.pin_fp8]),
    ("fp8 scale below the UE8M0 range", "SCALE_EXP_MIN = -127 ", "SCALE_EXP_MIN = -150 ", [TF8.pin_fp8]),
    ("h not quantized before w2", "h = fp8_act(silu(a) * c)", "h = silu(a) * c", [TF8.pin_fp8]),
    ("activations quantized per 128 x 128", "q, s = quantize_blocks(a, 1, 128)",
     "q, s = quantize_blocks(a, 128, 128)", [TF8.pin_fp8]),
    ("group gap taken one group too deep", "gs[:, topk_groups - 1] - gs[:, topk_groups]",
     "gs[:, topk_groups] - gs[:, min(topk_groups + 1, n_groups - 1)]",
     [TR.test_golden_group_gap_decides_margin, TR.pin_brute_force_margins]),
]


def _load_mutant(src: str) -> types.ModuleType:
    spec = importlib.util.spec_from_loader("moe_oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src, "<moe_oracle_mutant>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,orig,planted,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, orig, planted, pins, monkeypatch):
    assert SRC.count(orig) == 1, f"mutation anchor not found once: {orig!r}"
    mutant = _load_mutant(SRC.replace(orig, planted))
    caught = []
    for pin in pins:
        monkeypatch.setattr(inspect.getmodule(pin), "O", mutant)
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
        monkeypatch.undo()
    assert caught, f"no pin caught the planted mistake: {name}"


def test_unmutated_oracle_passes_pins():
    for _, _, _, pins in MUTATIONS:
        for pin in pins:
            pin()
