"""Pins of the oracle's FP8 window rows (one fp32 scale per row, signed E4M3
codes; "DeepSeek V1 到 V4.1-Flash ..." part 4 "P4 main KV": the SWA KV stays
FP8).

- Rows made of exactly representable values (the row maximum at 448 s) code
  and decode without error.
- Codes equal torch's own round-to-nearest-even float8_e4m3fn conversion of
  x / s (a library cast, independent of the oracle's search), with -0 stored
  as +0.
- Every decoded element is within half a unit in the last place of E4M3
  (relative 2^-4 for normals, 2^-10 s below the normal range).
- A zero row has scale 0 and zero codes; a non-finite element is reported,
  coded 0 and left out of the maximum.
"""
import numpy as np
import torch


def _e4m3_values():
    return torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()


def test_representable_rows_round_trip(orc):
    rng = np.random.default_rng(0)
    vals = _e4m3_values()
    for s in (1.0, 0.5, 0.0078125, 3.0):
        mag = rng.choice(vals, (4, 96))
        sign = rng.choice([-1.0, 1.0], (4, 96))
        rows = (mag * sign * s).astype(np.float32)
        rows[:, 0] = 448.0 * s
        codes, scales, bad = orc.window_fp8(rows)
        assert bad == 0 and np.all(scales == np.float32(s))
        assert np.array_equal(orc.window_fp8_dequant(codes, scales), rows)


def test_codes_match_torch_rne(orc):
    rng = np.random.default_rng(1)
    rows = (rng.standard_normal((64, 576)) * rng.choice([0.01, 1, 30], (64, 1))).astype(np.float32)
    codes, scales, bad = orc.window_fp8(rows)
    assert bad == 0
    q = torch.from_numpy(rows / scales[:, None].astype(np.float32))
    t = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    t[(t & 0x7F) == 0] = 0  # magnitude zero stored as +0
    assert np.array_equal(codes, t)


def test_error_bound(orc):
    rng = np.random.default_rng(2)
    rows = (rng.standard_normal((32, 576)) * 10).astype(np.float32)
    codes, scales, _ = orc.window_fp8(rows)
    deq = orc.window_fp8_dequant(codes, scales).astype(np.float64)
    x = rows.astype(np.float64)
    s = scales.astype(np.float64)[:, None]
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(deq - x) <= bound)


def test_zero_and_nonfinite_rows(orc):
    codes, scales, bad = orc.window_fp8(np.zeros((1, 64), np.float32))
    assert bad == 0 and scales[0] == 0 and not codes.any()
    row = np.linspace(-2, 2, 64).astype(np.float32)[None]
    row[0, 5] = np.nan
    row[0, 9] = np.inf
    codes, scales, bad = orc.window_fp8(row)
    assert bad == 1 and codes[0, 5] == 0 and codes[0, 9] == 0
    assert scales[0] == np.float32(2.0) / np.float32(448.0)
