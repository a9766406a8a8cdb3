"""Pins of the oracle's MXFP8 latent-cache route (CPU).

The element format, rounding and block scaling are checked against torch's float8_e4m3fn
conversion (a library routine) and against properties the format fixes (exact round trips of
representable values, the half-step error bound, the smallest fitting power-of-two scale);
the decode route is checked literal against weight-absorbed on the same stored bytes.
"""
import numpy as np
import pytest
import torch

from oracle import gdla_oracle as O
from tests.test_oracle_pins import tiny_weights


def fp8_cfg(window=0):
    # latent rows of kv_rank + d_rope = 64 values: two blocks of 32
    return O.OracleConfig(d_model=48, q_rank=24, kv_rank=60, n_signal=8, n_noise=2, n_kv_heads=2,
                          d_nope=8, d_rope=4, d_v=6, window=window)


def test_e4m3_values_match_torch_for_every_code():
    codes = np.arange(256)
    mine = O.e4m3_value(codes)
    ref = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(mine[~np.isnan(mine)], ref[~np.isnan(ref)])
    assert O.e4m3_value(0x7E) == 448.0 and O.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_rounding_matches_torch():
    pos = O.e4m3_value(np.arange(0x7F))
    mids = (pos[1:] + pos[:-1]) / 2                  # exact ties: to the even code
    x = np.concatenate([np.random.default_rng(0).uniform(-460, 460, 200000), pos, -pos, mids, -mids,
                        np.random.default_rng(1).uniform(-2.0 ** -6, 2.0 ** -6, 20000)])
    x = np.concatenate([x, [0.0, -0.0, -1e-5, 1e-5, -2.0 ** -10, 2.0 ** -10]])
    mine = O.e4m3_round(x)
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)                  # the codes, sign of zero included


def test_e4m3_saturates_at_448():
    x = np.array([448.0, 470.0, 1e6, -1e6, -449.0])
    assert np.array_equal(O.e4m3_value(O.e4m3_round(x)), [448.0, 448.0, 448.0, -448.0, -448.0])


def test_block_scale_is_the_smallest_power_of_two_that_fits():
    r = np.random.default_rng(2)
    amax = np.exp2(r.uniform(-100, 100, 5000)) * r.uniform(0.5, 1.0, 5000)
    k = O.mx_block_exponent(amax)
    assert np.all(amax <= 448.0 * np.exp2(k.astype(float)))
    assert np.all(amax > 448.0 * np.exp2((k - 1).astype(float)))
    # boundaries: amax = 448 * 2^j takes exactly k = j; zero takes -127
    j = np.arange(-20, 21)
    assert np.array_equal(O.mx_block_exponent(448.0 * np.exp2(j.astype(float))), j)
    assert O.mx_block_exponent(np.array([0.0]))[0] == -127


def test_round_trip_is_exact_for_representable_rows():
    r = np.random.default_rng(3)
    n = 576
    pos = O.e4m3_value(np.arange(0x7F))
    rows = np.empty((6, n))
    for i in range(6):
        for blk in range(n // 32):
            k = int(r.integers(-30, 30))
            v = r.choice(pos, 32) * r.choice([-1.0, 1.0], 32)
            v[r.integers(0, 32)] = 448.0              # the block's maximum fixes the scale at 2^k
            rows[i, 32 * blk: 32 * blk + 32] = v * 2.0 ** k
    stored = O.mxfp8_quantize_rows(rows)
    assert stored.shape == (6, 608) and stored.dtype == np.uint8
    assert np.all(stored[:, 594:] == 0)
    assert np.array_equal(O.mxfp8_dequantize_rows(stored, n), rows)


def test_quantization_error_is_within_half_a_step():
    r = np.random.default_rng(4)
    n = 576
    rows = r.standard_normal((20, n)) * np.exp2(r.integers(-40, 40, (20, 1)).astype(float))
    stored = O.mxfp8_quantize_rows(rows)
    back = O.mxfp8_dequantize_rows(stored, n)
    k = stored[:, n: n + 18].astype(np.int64) - 127
    step_floor = np.repeat(np.exp2((k - 10).astype(float)), 32, axis=1)   # half the subnormal step
    err = np.abs(back - rows)
    assert np.all(err <= np.abs(rows) * 2.0 ** -4 + step_floor)
    # and the scale byte is what the block maximum asks for
    amax = np.abs(rows).reshape(20, 18, 32).max(-1)
    assert np.array_equal(k, O.mx_block_exponent(amax))


@pytest.mark.parametrize("window", [0, 3])
def test_fp8_decode_literal_equals_absorbed(window):
    cfg = fp8_cfg(window)
    W = tiny_weights(cfg)
    lens = [0, 1, 5, 12]
    r = np.random.default_rng(5)
    n = cfg.kv_rank + cfg.d_rope
    cache = np.zeros((4, 14, n))
    for b, L in enumerate(lens):
        cache[b, :L] = r.normal(size=(L, n))
    cache8 = O.mxfp8_quantize_rows(cache.reshape(-1, n)).reshape(4, 14, -1)
    xn = r.normal(size=(4, cfg.d_model))
    a = O.gdla_decode_fp8(xn, W, cache8, lens, cfg, route="literal")
    b = O.gdla_decode_fp8(xn, W, cache8, lens, cfg, route="absorbed")
    np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-11)
    # two new tokens per sequence: the second sees the first's stored (quantized) row
    x2 = np.stack([xn, r.normal(size=(4, cfg.d_model))], axis=1)
    a2 = O.gdla_decode_fp8(x2, W, cache8, lens, cfg, route="literal", q_len=2)
    b2 = O.gdla_decode_fp8(x2, W, cache8, lens, cfg, route="absorbed", q_len=2)
    np.testing.assert_allclose(b2, a2, rtol=1e-10, atol=1e-11)
    # the first of two new tokens sees exactly what a single new token sees
    np.testing.assert_allclose(a2[:, 0], a, rtol=1e-12, atol=1e-13)


def test_fp8_decode_is_close_to_the_full_precision_decode():
    """The only difference is the cache's 8-bit rounding: the outputs stay within a few
    percent, far from what a wrong scale or a misplaced block would give."""
    cfg = fp8_cfg()
    W = tiny_weights(cfg, std=0.2)
    lens = [7, 12]
    r = np.random.default_rng(6)
    n = cfg.kv_rank + cfg.d_rope
    cache = np.zeros((2, 14, n))
    for b, L in enumerate(lens):
        cache[b, :L] = r.normal(size=(L, n))
    cache8 = O.mxfp8_quantize_rows(cache.reshape(-1, n)).reshape(2, 14, -1)
    xn = r.normal(size=(2, cfg.d_model))
    y8 = O.gdla_decode_fp8(xn, W, cache8, lens, cfg)
    y = O.gdla_decode(xn, W, cache, lens, cfg)
    rel = np.linalg.norm(y8 - y) / np.linalg.norm(y)
    assert 1e-4 < rel < 5e-2, rel
