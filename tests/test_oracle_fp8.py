"""Pins for the oracle's FP8 (e4m3, block-scaled) numbers and expert (CPU only).

The layout is this library's (the pages give none): e4m3 values with one
power-of-two scale per block, 128 x 128 for weights and 1 x 128 for
activations, the smallest scale that keeps the block's largest magnitude
within 448. Pinned by: known e4m3 roundings worked from the format, torch's
own float8_e4m3fn conversion, the scale's minimality, the quantizer's error
bound, exact round trips of representable blocks, and a restatement of the
FP8 SwiGLU with torch's float8 rounding and torch.nn.functional."""

import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def test_round_e4m3_known_values():
    cases = [
        (448.0, 448.0),                  # the largest finite value
        (464.0, 448.0),                  # halfway to the next step (480): saturates
        (1.0 + 1 / 16, 1.0),             # halfway between 1 and 1.125: to even (1)
        (1.0 + 3 / 16, 1.25),            # halfway between 1.125 and 1.25: to even (1.25)
        (1.0 + 1 / 16 + 2 ** -20, 1.125),
        (0.3, 0.3125),                   # 0.6 * 2^-1 -> 10/16 * 2^-1
        (-0.1, -0.1015625),              # 13/128
        (2.0 ** -9, 2.0 ** -9),          # smallest subnormal
        (2.0 ** -10, 0.0),               # halfway to 0: to even (0)
        (3 * 2.0 ** -11, 2.0 ** -9),     # 0.75 of the subnormal step
        (2.0 ** -6, 2.0 ** -6),          # smallest normal
        (2.0 ** -6 - 2.0 ** -9, 7 * 2.0 ** -9),   # largest subnormal
        (0.0, 0.0),
    ]
    v = np.array([c[0] for c in cases])
    np.testing.assert_array_equal(O.round_e4m3(v), np.array([c[1] for c in cases]))


def test_round_e4m3_matches_torch_float8():
    rng = np.random.default_rng(0)
    v = rng.standard_normal(200000) * 10.0 ** rng.integers(-5, 3, 200000)
    v = np.clip(v, -448, 448).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(v).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_e4m3(v), ref)


def test_block_exponent_is_the_smallest_that_fits():
    rng = np.random.default_rng(1)
    amax = np.abs(rng.standard_normal(50000)) * 10.0 ** rng.integers(-8, 6, 50000)
    amax = np.concatenate([amax, [448.0, 224.0, 1.75, 2.0 ** -20, 896.0]])
    s = O.block_exponent(amax)
    assert np.all(amax <= 448.0 * np.ldexp(1.0, s))
    assert np.all(amax > 448.0 * np.ldexp(1.0, s - 1))
    assert O.block_exponent(np.array([0.0]))[0] == 0


def test_block_exponent_stops_at_the_smallest_ue8m0_scale():
    # 448 * 2^-127 is the largest magnitude the scale 2^-127 serves exactly;
    # anything smaller keeps 2^-127 (a UE8M0 byte encodes 2^-127 .. 2^127)
    edge = 448.0 * 2.0 ** -127
    amax = np.array([edge, edge * (1 + 2 ** -20), edge / 2, 2.0 ** -120, 2.0 ** -140, 2.0 ** -1074])
    np.testing.assert_array_equal(O.block_exponent(amax), [-127, -126, -127, -127, -127, -127])
    # above the limit the rule is unchanged: 448 * 2^-126 needs exactly -126
    assert O.block_exponent(np.array([448.0 * 2.0 ** -126]))[0] == -126
    # the largest bf16 value needs 2^120, well inside the range
    assert O.block_exponent(np.array([3.3895313892515355e38]))[0] == 120


@pytest.mark.parametrize("br,bc,shape", [(128, 128, (300, 200)), (1, 128, (7, 300)), (128, 128, (128, 128))])
def test_quantize_blocks_properties(br, bc, shape):
    rng = np.random.default_rng(2)
    a = rng.standard_normal(shape) * np.exp(rng.standard_normal((shape[0], 1)))
    q, sc = O.quantize_blocks(a, br, bc)
    assert sc.shape == (math.ceil(shape[0] / br), math.ceil(shape[1] / bc))
    m, _ = np.frexp(sc)
    assert np.all(m == 0.5)                                  # powers of two
    # every value is an e4m3 value; the scale is minimal: each block's largest
    # magnitude over its scale lies in (224, 448] (so the largest code in
    # [224, 448] once rounded)
    np.testing.assert_array_equal(q, O.round_e4m3(q))
    for i in range(sc.shape[0]):
        for j in range(sc.shape[1]):
            sl = np.s_[i * br:(i + 1) * br, j * bc:(j + 1) * bc]
            assert 224.0 < np.abs(a[sl]).max() / sc[i, j] <= 448.0
            assert 224.0 <= np.abs(q[sl]).max() <= 448.0
    # round to nearest: within half a step of the e4m3 grid
    d = O.dequantize_blocks(q, sc, br, bc)
    full = np.repeat(np.repeat(sc, br, 0), bc, 1)[:shape[0], :shape[1]]
    step = np.where(np.abs(a / full) >= 2.0 ** -6,
                    np.ldexp(1.0, np.frexp(a / full)[1] - 4), 2.0 ** -9) * full
    assert np.all(np.abs(d - a) <= step / 2 * (1 + 1e-12))


def test_representable_blocks_round_trip_exactly():
    rng = np.random.default_rng(3)
    codes = O.round_e4m3(rng.uniform(-448, 448, (128, 256)))
    codes[0, 0], codes[0, 128] = 448.0, -448.0                # amax pins the scale
    a = codes * np.repeat([2.0 ** -10, 2.0 ** 3], 128)[None, :]
    q, sc = O.quantize_blocks(a, 128, 128)
    np.testing.assert_array_equal(sc, [[2.0 ** -10, 2.0 ** 3]])
    np.testing.assert_array_equal(O.dequantize_blocks(q, sc, 128, 128), a)


def test_zero_block():
    q, sc = O.quantize_blocks(np.zeros((1, 128)), 1, 128)
    assert (q == 0).all() and sc[0, 0] == 1.0


def _torch_fp8_rows(a: torch.Tensor) -> torch.Tensor:
    """Restatement with torch: per 1 x 128 block, scale 2^ceil(log2(amax/448))
    (checked and corrected to be the smallest that fits), values through
    torch's float8_e4m3fn."""
    out = torch.empty_like(a)
    for c0 in range(0, a.shape[1], 128):
        blk = a[:, c0:c0 + 128]
        amax = blk.abs().amax(dim=1, keepdim=True)
        s = torch.ceil(torch.log2(torch.clamp(amax, min=1e-300) / 448.0))
        s = torch.where(amax > 448.0 * torch.exp2(s), s + 1, s)
        s = torch.where(amax <= 448.0 * torch.exp2(s - 1), s - 1, s)
        scale = torch.where(amax > 0, torch.exp2(s), torch.ones_like(amax))
        q = (blk / scale).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64)
        out[:, c0:c0 + 128] = q * scale
    return out


def test_swiglu_fp8_matches_torch_restatement():
    rng = np.random.default_rng(4)
    D, I, n = 256, 384, 12
    x = torch.from_numpy(rng.standard_normal((n, D)).astype(np.float32).astype(np.float64))
    w1 = torch.from_numpy(rng.standard_normal((I, D)) / 16)
    w3 = torch.from_numpy(rng.standard_normal((I, D)) / 16)
    w2 = torch.from_numpy(rng.standard_normal((D, I)) / 20)
    xq = _torch_fp8_rows(x)
    h = torch.nn.functional.silu(xq @ w1.T) * (xq @ w3.T)
    ref = _torch_fp8_rows(h) @ w2.T
    got = O.swiglu_fp8(x.numpy(), w1.numpy(), w3.numpy(), w2.numpy())
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def pin_fp8():
    """The FP8 pins in one call (used by the planted-mistake tests)."""
    test_round_e4m3_known_values()
    test_block_exponent_is_the_smallest_that_fits()
    test_block_exponent_stops_at_the_smallest_ue8m0_scale()
    for case in [(128, 128, (300, 200)), (1, 128, (7, 300))]:
        test_quantize_blocks_properties(*case)
    test_swiglu_fp8_matches_torch_restatement()
