"""GPU parity of the MXFP8 latent cache: the row conversions bit for bit against the oracle's
quantizer, and decode over an MXFP8 cache against the oracle's route that dequantizes the same
bytes."""
import numpy as np
import pytest
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from differential_latent_attention_fwd_b200 import synth
from oracle import gdla_oracle as O
from tests.gpu_helpers import check, to_np

pytestmark = pytest.mark.gpu


def _edge_rows(n_rows: int, seed: int) -> torch.Tensor:
    """bf16 latent rows over a wide range of block magnitudes, plus rows that reach the edges:
    zero blocks, a single nonzero value, the largest bf16 values, subnormals, and values that
    land exactly halfway between two E4M3 values after scaling."""
    g = torch.Generator().manual_seed(seed)
    rows = torch.randn(n_rows, 576, generator=g)
    rows *= torch.exp2(torch.randint(-40, 40, (n_rows, 18), generator=g).float()).repeat_interleave(32, 1)
    rows = rows.bfloat16()
    rows[0] = 0
    rows[1] = 0
    rows[1, 5] = -3.0
    rows[2] = torch.finfo(torch.bfloat16).max * torch.sign(torch.randn(576, generator=g))
    rows[3] = torch.randn(576, generator=g).bfloat16() * 1e-39           # bf16 subnormals
    pos = torch.tensor(O.e4m3_value(np.arange(0x7F)), dtype=torch.float32)
    mids = ((pos[1:] + pos[:-1]) / 2)[:31]
    rows[4, :32] = torch.cat([torch.tensor([448.0]), mids]).bfloat16()   # scale 2^0: ties
    rows[5] = rows[4] * -2.0 ** -7
    return rows


def test_quantize_matches_oracle_bit_for_bit(cuda_ok):
    cfg = gb.make_config(synth.GdlaShape())
    rows = _edge_rows(3000, 31)
    out = torch.full((rows.shape[0], gb.FP8_ROW_BYTES), 0xAB, dtype=torch.uint8, device="cuda")
    gb.gdla_quantize_latent_fp8(cfg, rows.cuda(), out)
    torch.cuda.synchronize()
    want = O.mxfp8_quantize_rows(rows.float().numpy())
    got = out.cpu().numpy()
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:5].tolist()}"


def test_dequantize_matches_oracle(cuda_ok):
    cfg = gb.make_config(synth.GdlaShape())
    rows = _edge_rows(1000, 32)
    stored = torch.tensor(O.mxfp8_quantize_rows(rows.float().numpy())).cuda()
    back = torch.empty(rows.shape, dtype=torch.bfloat16, device="cuda")
    gb.gdla_dequantize_latent_fp8(cfg, stored, back)
    torch.cuda.synchronize()
    want = O.mxfp8_dequantize_rows(stored.cpu().numpy(), 576)
    # a stored value has 4 significant bits, so bf16 holds it exactly inside its normal range;
    # the edge rows (beyond the largest bf16, below its smallest normal) round as bf16 rounds
    want_bf16 = torch.tensor(want).to(torch.bfloat16).float().numpy()
    got = back.float().cpu().numpy()
    assert np.array_equal(got, want_bf16)
    normal = (np.abs(want) >= 2.0 ** -126) & (np.abs(want) <= float(torch.finfo(torch.bfloat16).max))
    assert np.array_equal(got[normal].astype(np.float64), want[normal])


def _fp8_case(window, lens, cap, seed, q_len=1, tail_nan=False):
    """Decode inputs with the cache stored in MXFP8 (the oracle's quantizer of the bf16 rows)."""
    from differential_latent_attention_fwd_b200.layer import GdlaLayer
    shape = synth.GdlaShape(window=window)
    inp = synth.make_decode_inputs(shape, len(lens), lens, cap=cap, seed=seed)
    cache8 = O.mxfp8_quantize_rows(inp.cache.float().numpy().reshape(-1, 576)).reshape(len(lens), cap, -1)
    if tail_nan:
        for b, L in enumerate(lens):
            cache8[b, L:] = 0xFF                      # NaN codes and NaN scales past the written rows
    layer = GdlaLayer(shape, inp.weights, inp.g_q, inp.g_kv, device="cuda")
    g = torch.Generator().manual_seed(seed + 1)
    x = inp.x_new if q_len == 1 else torch.randn(len(lens), q_len, shape.d_model, generator=g).bfloat16()
    c8 = torch.tensor(cache8).cuda()
    y = layer.decode_fp8(x.cuda(), c8, inp.cache_len.cuda())
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    cfg = O.OracleConfig.from_shape(shape)
    yo = O.gdla_decode_fp8(x, inp.weights, cache8, inp.cache_len, cfg, g_q=inp.g_q, g_kv=inp.g_kv, q_len=q_len)
    return y, yo, c8, cache8, inp, layer


@pytest.mark.parametrize("window", [0, 64])
def test_fp8_decode_small_ragged(cuda_ok, window):
    lens = [0, 5, 63, 64, 130, 317]
    y, yo, c8, cache8, inp, _ = _fp8_case(window, lens, 330, 41)
    errs = []
    for b in range(len(lens)):
        check(f"fp8 decode y[b={b}] len={lens[b]} W={window}", to_np(y[b]), yo[b], errors=errs)
    assert not errs, "\n".join(errs)
    got = c8.cpu().numpy()
    for b, L in enumerate(lens):
        # cached rows untouched; the appended row holds the new token's latent values in MXFP8
        assert np.array_equal(got[b, :L], cache8[b, :L])
        new = O.mxfp8_dequantize_rows(got[b, L][None], 576)[0]
        cfg = O.OracleConfig.from_shape(synth.GdlaShape(window=window))
        cbar, kR = O.kv_latent(O.f64(inp.x_new[b][None]), O.f64(inp.weights["W_aKV"]), O.f64(inp.g_kv), [L], cfg)
        want = np.concatenate([cbar[0], kR[0]])
        assert np.all(np.abs(new - want) <= np.abs(want) * (2.0 ** -4 + 2.0 ** -7) + 1e-2), b


def test_fp8_decode_ignores_unwritten_tail(cuda_ok):
    lens = [0, 63, 64, 200, 317]
    y, yo, *_ = _fp8_case(0, lens, 330, 43, tail_nan=True)
    assert bool(torch.isfinite(y).all())
    errs = []
    for b in range(len(lens)):
        check(f"fp8 decode with a NaN tail, b={b}", to_np(y[b]), yo[b], errors=errs)
    assert not errs, "\n".join(errs)


def test_fp8_decode_multi_token(cuda_ok):
    lens = [3, 64, 200, 500]
    y, yo, *_ = _fp8_case(0, lens, 520, 45, q_len=3)
    errs = []
    for b in range(len(lens)):
        for i in range(3):
            check(f"fp8 decode b={b} token {i}", to_np(y[b, i]), yo[b, i], errors=errs)
    assert not errs, "\n".join(errs)


@pytest.mark.parametrize("window", [0, 2048])
def test_fp8_decode_long_cache(cuda_ok, window):
    """16 sequences of 32 768 cached positions (the decode workload's length)."""
    lens = [32768] * 16
    y, yo, *_ = _fp8_case(window, lens, 32769, 47)
    errs = []
    for b in range(len(lens)):
        check(f"fp8 decode L=32768 W={window} b={b}", to_np(y[b]), yo[b], errors=errs)
    assert not errs, "\n".join(errs)
