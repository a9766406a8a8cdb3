"""GPU decode parity (absorbed form through the C ABI) against the fp64 oracle, plus the
prefill -> decode hand-off and the bounded-wait error path."""
import numpy as np
import pytest
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from differential_latent_attention_fwd_b200 import synth
from differential_latent_attention_fwd_b200.layer import GdlaLayer
from oracle import gdla_oracle as O
from tests.gpu_helpers import check, oracle_prefill, prefill_case, to_np

pytestmark = pytest.mark.gpu


def _decode(inp, device="cuda"):
    layer = GdlaLayer(inp.shape, inp.weights, inp.g_q, inp.g_kv, device=device)
    cache = inp.cache.to(device)
    lens = inp.cache_len.to(device)
    y = layer.decode(inp.x_new.to(device), cache, lens)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    return y, cache


@pytest.mark.parametrize("window", [0, 64])
def test_decode_small_ragged(cuda_ok, window):
    shape = synth.GdlaShape(window=window)
    lens = [0, 5, 130, 300]
    inp = synth.make_decode_inputs(shape, 4, lens, cap=320, seed=21)
    y, cache = _decode(inp)
    cfg = O.OracleConfig.from_shape(shape)
    yo, parts = O.gdla_decode(inp.x_new, inp.weights, inp.cache, inp.cache_len, cfg,
                              g_q=inp.g_q, g_kv=inp.g_kv, return_parts=True)
    errs = []
    for b in range(4):
        check(f"decode y[b={b}] len={lens[b]} W={window}", to_np(y[b]), yo[b], errors=errs)
        row = to_np(cache[b, lens[b]])
        check(f"appended cache row b={b}", row, np.concatenate([parts["cbar_new"][b], parts["kR_new"][b]]),
              rel=4e-3, mabs=5e-2, errors=errs)
    assert not errs, "\n".join(errs)
    # rows other than the appended one are untouched
    for b in range(4):
        assert torch.equal(cache[b, : lens[b]].cpu(), inp.cache[b, : lens[b]])


@pytest.mark.parametrize("name", ["decode_b64_l32768_causal", "decode_b64_l32768_swa2048"])
def test_decode_workload(cuda_ok, name):
    wl = synth.WORKLOADS[name]
    shape = synth.GdlaShape(window=wl["window"])
    inp = synth.make_decode_inputs(shape, wl["B"], wl["L"], cap=wl["cap"], seed=wl["seed"])
    y, _ = _decode(inp)
    cfg = O.OracleConfig.from_shape(shape)
    yo = O.gdla_decode_absorbed(inp.x_new, inp.weights, inp.cache, inp.cache_len, cfg,
                                g_q=inp.g_q, g_kv=inp.g_kv)
    check(f"{name}: all 64 sequences", to_np(y), yo)


@pytest.mark.parametrize("window", [0, 64])
def test_decode_ignores_unwritten_cache_tail(cuda_ok, window):
    """Cache rows past each sequence's new token were never written by the caller: here they
    hold NaN and Inf.  The output must equal the oracle's, which never reads those rows."""
    shape = synth.GdlaShape(window=window)
    lens = [0, 63, 64, 200, 317]
    inp = synth.make_decode_inputs(shape, len(lens), lens, cap=320, seed=23)
    cache = inp.cache.clone()
    for b, L in enumerate(lens):
        cache[b, L + 1:, ::2] = float("nan")       # row L is the appended one
        cache[b, L + 1:, 1::2] = float("inf")
    layer = GdlaLayer(shape, inp.weights, inp.g_q, inp.g_kv, device="cuda")
    y = layer.decode(inp.x_new.cuda(), cache.cuda(), inp.cache_len.cuda())
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    cfg = O.OracleConfig.from_shape(shape)
    yo = O.gdla_decode(inp.x_new, inp.weights, inp.cache, inp.cache_len, cfg, g_q=inp.g_q, g_kv=inp.g_kv)
    errs = []
    for b in range(len(lens)):
        check(f"decode with a NaN/Inf tail b={b} len={lens[b]} W={window}", to_np(y[b]), yo[b], errors=errs)
    assert not errs, "\n".join(errs)


def test_decode_single_sequence_long_cache(cuda_ok):
    """One sequence over a long cache: its key tiles are spread over every SM (many segments of
    one row), then merged."""
    shape = synth.GdlaShape()
    inp = synth.make_decode_inputs(shape, 1, [20000], cap=20001, seed=25)
    y, _ = _decode(inp)
    cfg = O.OracleConfig.from_shape(shape)
    yo = O.gdla_decode_absorbed(inp.x_new, inp.weights, inp.cache, inp.cache_len, cfg,
                                g_q=inp.g_q, g_kv=inp.g_kv)
    check("B=1, L=20000", to_np(y), yo)


def test_prefill_then_decode_continues_sequence(cuda_ok):
    """Prefill T tokens into a cache, decode token T: equals row T of a (T+1)-token prefill."""
    T, cap = 200, 256
    shape, inp, layer, x = prefill_case(1, T + 1, 0, seed=9)
    cache = torch.zeros((1, cap, 576), dtype=torch.bfloat16, device="cuda")
    layer.prefill(x[:, :T].contiguous(), kv_cache_out=cache)
    lens = torch.tensor([T], dtype=torch.int32, device="cuda")
    yd = layer.decode(x[:, T].contiguous(), cache, lens)
    yp = layer.prefill(x)
    torch.cuda.synchronize()
    yo = oracle_prefill(inp, rows=[T])
    check("decode of token T vs oracle", to_np(yd[0]), yo[0, 0])
    check("decode of token T vs GPU prefill row T", to_np(yd[0]), to_np(yp[0, T]), rel=5e-3, mabs=2e-2)


def test_bounded_wait_expires_and_context_survives(cuda_ok):
    site = gb.gdla_selftest_wait_timeout(2_000_000)  # 2 ms bound on a wait nothing satisfies
    assert site == 0x401
    assert gb.gdla_device_error() == 0                 # the self-test cleared its report
    shape, inp, layer, x = prefill_case(1, 64, 0, seed=1)
    y = layer.prefill(x)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    check("prefill after the timeout self-test", to_np(y[0]), oracle_prefill(inp)[0])


@pytest.mark.parametrize("window", [0, 64])
def test_multi_token_decode(cuda_ok, window):
    """Three new tokens per sequence in one call (multi-token verification) against the oracle,
    including the three appended latent-cache rows."""
    from differential_latent_attention_fwd_b200 import synth as S
    shape = S.GdlaShape(window=window)
    lens, q = [0, 50, 300], 3
    inp = S.make_decode_inputs(shape, 3, lens, cap=320, seed=31)
    xm = torch.randn((3, q, shape.d_model), generator=torch.Generator().manual_seed(5)).bfloat16()
    layer = GdlaLayer(shape, inp.weights, inp.g_q, inp.g_kv, device="cuda")
    cache = inp.cache.cuda()
    y = layer.decode_multi(xm.cuda(), cache, inp.cache_len.cuda())
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    cfg = O.OracleConfig.from_shape(shape)
    yo = O.gdla_decode_multi(xm, inp.weights, inp.cache, inp.cache_len, cfg, g_q=inp.g_q, g_kv=inp.g_kv)
    errs = []
    for b in range(3):
        for i in range(q):
            check(f"multi-token decode b={b} token {i} (len {lens[b]}, W={window})", to_np(y[b, i]),
                  yo[b, i], errors=errs)
    # appended rows: the q new latent rows sit at cache_len .. cache_len + q - 1
    W64 = {k: O.f64(v) for k, v in inp.weights.items()}
    for b in range(3):
        cb, kr = O.kv_latent(O.f64(xm[b]), W64["W_aKV"], None, lens[b] + np.arange(q), cfg)
        check(f"appended rows b={b}", to_np(cache[b, lens[b]:lens[b] + q]), np.concatenate([cb, kr], -1),
              rel=4e-3, mabs=5e-2, errors=errs)
    assert not errs, "\n".join(errs)


def test_multi_token_decode_workload_size(cuda_ok):
    """B=64 sequences x 2 new tokens over a 32768-position cache (absorbed oracle)."""
    from differential_latent_attention_fwd_b200 import synth as S
    shape = S.GdlaShape()
    inp = S.make_decode_inputs(shape, 64, 32768, cap=32770, seed=4)
    xm = torch.randn((64, 2, shape.d_model), generator=torch.Generator().manual_seed(6)).bfloat16()
    layer = GdlaLayer(shape, inp.weights, inp.g_q, inp.g_kv, device="cuda")
    y = layer.decode_multi(xm.cuda(), inp.cache.cuda(), inp.cache_len.cuda())
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    cfg = O.OracleConfig.from_shape(shape)
    yo = O.gdla_decode_multi(xm, inp.weights, inp.cache, inp.cache_len, cfg, g_q=inp.g_q, g_kv=inp.g_kv,
                             route="absorbed")
    check("B64 x 2 tokens, L=32768", to_np(y).reshape(128, -1), yo.reshape(128, -1))
