"""GPU prefill parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerance of the layer output y: max-abs 2e-2 and relative L2 5e-3.  Intermediates are checked
stage by stage first, with a bound derived from the storage precision of each stage (one bf16
rounding ~1.6e-3 rms relative, fp16 ~2e-4), so that a failure names the kernel at fault.
"""
import numpy as np
import pytest
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from differential_latent_attention_fwd_b200 import synth
from tests.gpu_helpers import (MAX_ABS, REL_L2, WS_CQ, WS_D1, WS_DG, WS_G, WS_KV, WS_LAM,
                               WS_LATENT, WS_ONOISE, WS_QQ, check, oracle_prefill, prefill_case,
                               to_np, ws_view)

pytestmark = pytest.mark.gpu


def _run(layer, x, kv_cache_out=None):
    y = layer.prefill(x, kv_cache_out=kv_cache_out)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    return y


def test_stagewise_intermediates_t256(cuda_ok):
    """Every stage of the T=256 causal layer against the oracle's intermediates."""
    B, T = 1, 256
    shape, inp, layer, x = prefill_case(B, T, 0, seed=0)
    y = _run(layer, x)
    ws = layer._ws
    cfg = layer.cfg
    yo, parts = oracle_prefill(inp, parts=True)
    p = parts[0]
    nH = shape.n_heads
    errs = []
    # fp32 down-projection, before the norms
    x64 = to_np(inp.x[0])
    W = {k: to_np(v) for k, v in inp.weights.items()}
    d1 = to_np(ws_view(ws, cfg, B, T, 0, WS_D1, torch.float32, (T, 1664)))
    check("x W_aQ (fp32)", d1[:, :1024], x64 @ W["W_aQ"], rel=1e-4, mabs=1e-2, errors=errs)
    check("x W_aKV (fp32)", d1[:, 1024:1600], x64 @ W["W_aKV"], rel=1e-4, mabs=1e-2, errors=errs)
    check("x W_lambda (fp32)", d1[:, 1600:], x64 @ W["W_lambda"], rel=1e-4, mabs=1e-2, errors=errs)
    cq = to_np(ws_view(ws, cfg, B, T, 0, WS_CQ, torch.bfloat16, (T, 1024)))
    check("c^Q (bf16)", cq, p["cQ"], rel=4e-3, mabs=5e-2, errors=errs)
    lat = to_np(ws_view(ws, cfg, B, T, 0, WS_LATENT, torch.bfloat16, (T, 576)))
    check("c_bar^KV (bf16)", lat[:, :512], p["cbar"], rel=4e-3, mabs=5e-2, errors=errs)
    check("rotated k^R (bf16)", lat[:, 512:], p["kR"], rel=4e-3, mabs=5e-2, errors=errs)
    lam = to_np(ws_view(ws, cfg, B, T, 0, WS_LAM, torch.float32, (T, 64)))
    check("lambda (fp32)", lam, p["lam"], rel=1e-4, mabs=1e-4, errors=errs)
    qq = to_np(ws_view(ws, cfg, B, T, 0, WS_QQ, torch.float16, (T, nH * 192)))
    check("q^C (fp16)", qq[:, : nH * 128].reshape(T, nH, 128), p["qC"], rel=6e-3, mabs=5e-2, errors=errs)
    check("rotated q^R (fp16)", qq[:, nH * 128:].reshape(T, nH, 64), p["qR"], rel=6e-3, mabs=5e-2,
          errors=errs)
    g = to_np(ws_view(ws, cfg, B, T, 0, WS_G, torch.bfloat16, (T, 64, 128)))
    check("G (bf16)", g, p["G"], rel=6e-3, mabs=5e-2, errors=errs)
    kv = to_np(ws_view(ws, cfg, B, T, 0, WS_KV, torch.float16, (T, 16, 256)))
    check("K^C (fp16)", kv[..., :128], p["KC"], rel=6e-3, mabs=5e-2, errors=errs)
    check("V (fp16)", kv[..., 128:], p["V"], rel=6e-3, mabs=5e-2, errors=errs)
    dg = to_np(ws_view(ws, cfg, B, T, 0, WS_DG, torch.bfloat16, (T, 64, 128)))
    check("Dg (bf16)", dg, p["Dg"], rel=REL_L2, mabs=MAX_ABS, errors=errs)
    check("y (bf16)", to_np(y[0]), yo[0], errors=errs)
    assert not errs, "\n".join(errs)


@pytest.mark.parametrize("B,T,window", [
    (1, 1, 0), (1, 100, 0), (1, 129, 0), (1, 300, 0), (2, 200, 64), (1, 700, 128),
    (1, 384, 1), (1, 257, 256), (3, 130, 0),
    # a window at least as long as the sequence: every row sees its whole causal prefix
    (1, 100, 2048), (2, 300, 512), (1, 256, 256), (1, 513, 600),
])
def test_prefill_edge_shapes(cuda_ok, B, T, window):
    shape, inp, layer, x = prefill_case(B, T, window, seed=11)
    y = _run(layer, x)
    yo = oracle_prefill(inp)
    errs = []
    for b in range(B):
        check(f"y[b={b}] B={B} T={T} W={window}", to_np(y[b]), yo[b], errors=errs)
    assert not errs, "\n".join(errs)


def test_prefill_writes_latent_cache(cuda_ok):
    B, T, cap = 2, 150, 160
    shape, inp, layer, x = prefill_case(B, T, 0, seed=5)
    cache = torch.zeros((B, cap, 576), dtype=torch.bfloat16, device="cuda")
    _run(layer, x, kv_cache_out=cache)
    _, parts = oracle_prefill(inp, parts=True)
    for b in range(B):
        want = np.concatenate([parts[b]["cbar"], parts[b]["kR"]], -1)
        check(f"cache rows b={b}", to_np(cache[b, :T]), want, rel=4e-3, mabs=5e-2)
    assert float(cache[:, T:].abs().max()) == 0.0


def test_prefill_deterministic(cuda_ok):
    shape, inp, layer, x = prefill_case(1, 300, 0, seed=3)
    y1 = _run(layer, x).clone()
    y2 = _run(layer, x)
    assert torch.equal(y1, y2)


def _sampled_workload(name, n_rows=512):
    wl = synth.WORKLOADS[name]
    B, T, window, seed = wl["B"], wl["T"], wl["window"], wl["seed"]
    shape, inp, layer, x = prefill_case(B, T, window, seed)
    y = _run(layer, x)
    rows = synth.sample_rows(T, window, n_rows, seed)
    yo = oracle_prefill(inp, rows=rows)
    errs = []
    for b in range(B):
        check(f"{name} b={b} ({len(rows)} sampled rows)", to_np(y[b, rows]), yo[b], errors=errs)
    del layer, x, y
    torch.cuda.empty_cache()
    assert not errs, "\n".join(errs)


def test_workload_t256_causal_all_rows(cuda_ok):
    wl = synth.WORKLOADS["prefill_b1_t256_causal"]
    shape, inp, layer, x = prefill_case(wl["B"], wl["T"], wl["window"], wl["seed"])
    y = _run(layer, x)
    check("T=256 causal, all rows", to_np(y[0]), oracle_prefill(inp)[0])


def test_workload_b2_t8192_swa2048_sampled(cuda_ok):
    _sampled_workload("prefill_b2_t8192_swa2048")


def test_workload_t32768_causal_sampled(cuda_ok):
    _sampled_workload("prefill_b1_t32768_causal")


def test_workload_t262144_swa2048_sampled(cuda_ok):
    _sampled_workload("prefill_b1_t262144_swa2048")


def test_workload_t262144_causal_sampled(cuda_ok):
    _sampled_workload("prefill_b1_t262144_causal")


@pytest.mark.parametrize("window", [0, 128])
def test_packed_documents(cuda_ok, window):
    """Packed documents (ragged lengths incl. 1, exact multiples of 128/256 and a tail) against
    the oracle run per document, and the packed latent rows against the oracle's."""
    from oracle import gdla_oracle as O
    lens = [1, 100, 256, 513, 37, 300, 128]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    shape, inp, layer, x = prefill_case(1, total, window, seed=23)
    xp = x[0].contiguous()
    lat = torch.zeros((total, 576), dtype=torch.bfloat16, device="cuda")
    y = layer.prefill_packed(xp, torch.from_numpy(cu).cuda(), kv_latent_out=lat)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    cfg = O.OracleConfig.from_shape(shape)
    yo = O.gdla_prefill_packed(inp.x[0], cu, inp.weights, cfg, g_q=inp.g_q, g_kv=inp.g_kv)
    errs = []
    for d in range(len(lens)):
        a, b = int(cu[d]), int(cu[d + 1])
        check(f"doc {d} (len {lens[d]}, W={window})", to_np(y[a:b]), yo[a:b], errors=errs)
    assert not errs, "\n".join(errs)
    # the same documents run one by one through the batch entry point give the same rows
    for d in (2, 3):
        a, b = int(cu[d]), int(cu[d + 1])
        yd = layer.prefill(xp[a:b][None].contiguous())
        torch.cuda.synchronize()
        check(f"doc {d}: packed vs standalone GPU run", to_np(y[a:b]), to_np(yd[0]), rel=1e-6, mabs=1e-5)
    # latent rows: positions restart inside every document
    _, parts = O.gdla_prefill(inp.x[:, cu[3]:cu[4]], inp.weights, cfg, g_q=inp.g_q, g_kv=inp.g_kv,
                              return_parts=True)
    want = np.concatenate([parts[0]["cbar"], parts[0]["kR"]], -1)
    check("packed latent rows of doc 3", to_np(lat[cu[3]:cu[4]]), want, rel=4e-3, mabs=5e-2)


def test_packed_documents_reject_bad_offsets(cuda_ok):
    shape, inp, layer, x = prefill_case(1, 64, 0, seed=2)
    bad = torch.tensor([0, 40, 30, 64], dtype=torch.int32, device="cuda")   # decreasing offset
    layer.prefill_packed(x[0].contiguous(), bad)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0x602


def test_large_norm_gains_keep_fp16_operands_finite(cuda_ok):
    """RMSNorm gains of 50 on both latents: the fp16 attention operands grow about 50x and stay
    finite, and no range error is reported.  Gains of 50 also scale the logits by 2500, where
    the bf16 rounding of the latents alone moves the softmax by percents (measured: 4.9 % rel-L2
    at gains 50, 5.1e-3 at gains 4), so parity against the oracle is checked with gains of 2
    (operands x2, logits x4), at the layer bar."""
    from oracle import gdla_oracle as O
    from differential_latent_attention_fwd_b200.layer import GdlaLayer
    T, window = 200, 0
    shape = synth.GdlaShape(window=window)
    inp = synth.make_prefill_inputs(shape, 1, T, seed=13)
    nH = shape.n_heads
    for gain in (50.0, 2.0):
        gq = (torch.ones(shape.q_rank) * gain).bfloat16()
        gkv = (torch.ones(shape.kv_rank) * gain).bfloat16()
        layer = GdlaLayer(shape, inp.weights, gq, gkv, device="cuda")
        y = layer.prefill(inp.x.cuda())
        torch.cuda.synchronize()
        assert gb.gdla_device_error() == 0
        assert bool(torch.isfinite(y).all())
        qq = to_np(ws_view(layer._ws, layer.cfg, 1, T, 0, WS_QQ, torch.float16, (T, nH * shape.d_qk)))
        kv = to_np(ws_view(layer._ws, layer.cfg, 1, T, 0, WS_KV, torch.float16, (T, shape.n_kv_heads, 256)))
        amax = max(np.abs(qq).max(), np.abs(kv).max())
        assert gain / 2 < amax < 65504.0, (gain, amax)
        if gain == 2.0:
            cfg = O.OracleConfig.from_shape(shape)
            _, parts = O.gdla_prefill(inp.x, inp.weights, cfg, g_q=gq, g_kv=gkv, return_parts=True)
            dg = to_np(ws_view(layer._ws, layer.cfg, 1, T, 0, WS_DG, torch.bfloat16, (T, 64, 128)))
            # V (hence D and Dg) grows with the KV gain: the absolute bound scales with it
            check("Dg with gains x2 vs the oracle with the same gains", dg, parts[0]["Dg"], mabs=MAX_ABS * gain)


def test_fp16_operand_overflow_is_reported(cuda_ok):
    """A query-latent gain of 1e5 pushes q^C past the fp16 range: the values saturate at
    +-65504, the output stays finite, and the device error word reports site 0x701."""
    T = 64
    shape = synth.GdlaShape()
    inp = synth.make_prefill_inputs(shape, 1, T, seed=14)
    from differential_latent_attention_fwd_b200.layer import GdlaLayer
    gq = (torch.ones(shape.q_rank) * 1e5).bfloat16()
    layer = GdlaLayer(shape, inp.weights, gq, inp.g_kv, device="cuda")
    y = layer.prefill(inp.x.cuda())
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0x701
    assert bool(torch.isfinite(y).all())
    qq = ws_view(layer._ws, layer.cfg, 1, T, 0, WS_QQ, torch.float16, (T, shape.n_heads * shape.d_qk))
    assert float(qq.float().abs().max()) == 65504.0
    # the next call with ordinary gains reports nothing
    layer2 = GdlaLayer(shape, inp.weights, inp.g_q, inp.g_kv, device="cuda")
    layer2.prefill(inp.x.cuda())
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
