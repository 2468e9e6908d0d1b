"""Pins for the FP8 (E4M3) gating oracle (CPU).

* the E4M3 decoding against torch's float8_e4m3fn conversion, all 256 codes;
* on inputs whose dequantized values are exact in bf16 (every finite E4M3
  value is, and power-of-two scales keep them so) the FP8 oracle must equal
  the pinned bf16 oracle bit for bit: same products, same summation order;
* with arbitrary scales, logits against numpy's fp64 matmul of the
  dequantized operands (scale per token on rows, per expert on columns);
* planted mistakes in copies of the oracle source each fail one of these.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def _decode_torch(codes):
    return torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _pin_decode(o):
    codes = np.arange(256, dtype=np.uint8)
    ref = _decode_torch(codes)
    got = np.array([o.e4m3_to_f64(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def _random_codes(rng, shape):
    codes = rng.integers(0, 256, size=shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    return codes


def _pin_matches_bf16_oracle(o, T=40, H=96, E=24, k=5, seed=0):
    rng = np.random.default_rng(seed)
    xq = _random_codes(rng, (T, H))
    wq = _random_codes(rng, (E, H))
    xs = np.ldexp(1.0, rng.integers(-12, -4, size=T)).astype(np.float32)
    ws = np.ldexp(1.0, rng.integers(-12, -4, size=E)).astype(np.float32)
    got = o.gating_fp8(xq, xs, wq, ws, k, want_logits=True)
    x = xs[:, None].astype(np.float64) * _decode_torch(xq)
    w = (ws[:, None].astype(np.float64) * _decode_torch(wq)).T          # [H, E]
    xb, wb = workloads.round_bf16(x), workloads.round_bf16(w)
    assert np.array_equal(workloads.bf16_to_f64(xb), x) and np.array_equal(workloads.bf16_to_f64(wb), w)
    ref = oracle.load().gating(xb, wb, k, want_logits=True)
    assert np.array_equal(got.logits, ref.logits)
    assert np.array_equal(got.ids, ref.ids)
    assert np.array_equal(got.scores64, ref.scores64)


def _pin_scales_numpy(o, T=30, H=64, E=40, k=6, seed=1):
    rng = np.random.default_rng(seed)
    xq = _random_codes(rng, (T, H))
    wq = _random_codes(rng, (E, H))
    xs = rng.uniform(0.001, 0.01, size=T).astype(np.float32)
    ws = rng.uniform(0.001, 0.01, size=E).astype(np.float32)
    got = o.gating_fp8(xq, xs, wq, ws, k, want_logits=True)
    ref = (xs[:, None].astype(np.float64) * _decode_torch(xq)) @ (ws[:, None].astype(np.float64) * _decode_torch(wq)).T
    assert np.allclose(got.logits, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    order = np.lexsort((np.broadcast_to(np.arange(E), ref.shape), -ref), axis=1)[:, :k]
    assert np.array_equal(got.ids, order)


PINS = [_pin_decode, _pin_matches_bf16_oracle, _pin_scales_numpy]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_fp8_oracle_pins(pin):
    pin(oracle.load())


def test_workload_quantization_round_trips():
    wl = workloads.RouterWorkload("q", 16, 256, 32, 4, seed=2)
    xq, xs, wq, ws = workloads.fp8_inputs(wl)
    assert xq.shape == (16, 256) and xs.shape == (16,) and wq.shape == (32, 256) and ws.shape == (32,)
    x = workloads.bf16_to_f64(wl.hidden())
    back = xs[:, None] * _decode_torch(xq)
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -4 + xs[:, None] * 2.0 ** -9)  # E4M3: 3 mantissa bits
    assert np.all(np.abs(_decode_torch(xq)).max(axis=1) == 448.0)


MUTANTS = {
    "exponent_bias": ("magnitude = ldexp(1.0 + (double)mantissa / 8.0, exponent - 7);",
                      "magnitude = ldexp(1.0 + (double)mantissa / 8.0, exponent - 8);"),
    "subnormal_scale": ("magnitude = ldexp((double)mantissa / 8.0, -6);", "magnitude = ldexp((double)mantissa / 8.0, -7);"),
    "hidden_scale_dropped": ("x[h] = (double)hidden_scale[t] * oracle_e4m3_to_f64", "x[h] = 1.0 * oracle_e4m3_to_f64"),
    "gate_scale_index": ("w[e * H + h] = (double)gate_scale[e] *", "w[e * H + h] = (double)gate_scale[h % E] *"),
    "gate_transposed": ("acc += x[h] * w[e * H + h];", "acc += x[h] * w[(h % E) * H + (e % H)];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(oracle.FP8_SOURCE).read()
    assert src.count(before) == 1, name
    mutant = tmp_path / "fp8_mutant.c"
    mutant.write_text(src.replace(before, after))
    o = oracle.Oracle(oracle.compile_oracle(oracle.SOURCE, str(tmp_path / "libm.so"), oracle.ROUTE_SOURCE, str(mutant)))
    caught = False
    for pin in PINS:
        try:
            pin(o)
        except AssertionError:
            caught = True
            break
    assert caught, f"fp8 mutant {name} passed every pin"
