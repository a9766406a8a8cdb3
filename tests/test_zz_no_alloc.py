"""Allocation-free attention stage (gdla_attn_prefill_noalloc) against the workspace path.

Callers that cannot allocate device memory while they run -- an engine plugin handed only its
input and output buffers, a service whose footprint is fixed at start-up -- use
gdla_attn_prefill_noalloc, whose only scratch is a fixed array inside the library.  These tests
call it through the C ABI twice in a row and compare its output with the attention stage of
gdla_prefill_fwd (the Dg it leaves in its workspace) and with the fp64 oracle's attention stage
on the same inputs, within the parity tolerance, up to the largest size its scratch allows.
"""
import pytest
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from differential_latent_attention_fwd_b200 import synth
from oracle import gdla_oracle as O
from tests.gpu_helpers import (MAX_ABS, REL_L2, WS_DG, WS_G, WS_KR16, WS_KV, WS_LAM, WS_QQ, check,
                               prefill_case, to_np, ws_view)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,T,window", [(1, 300, 0), (2, 640, 256)])
def test_noalloc_attention_matches_workspace_path(cuda_ok, B, T, window):
    shape, inp, layer, x = prefill_case(B, T, window, seed=17)
    layer.prefill(x)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    ws, cfg = layer._ws, layer.cfg
    M, nH = B * T, shape.n_heads
    qq = ws_view(ws, cfg, B, T, 0, WS_QQ, torch.float16, (M, nH * shape.d_qk))
    kv = ws_view(ws, cfg, B, T, 0, WS_KV, torch.float16, (M, shape.n_kv_heads * 256))
    kr = ws_view(ws, cfg, B, T, 0, WS_KR16, torch.float16, (M, shape.d_rope))
    lam = ws_view(ws, cfg, B, T, 0, WS_LAM, torch.float32, (M, shape.n_signal))
    gate = ws_view(ws, cfg, B, T, 0, WS_G, torch.bfloat16, (M, shape.n_signal * shape.d_v))
    ref = ws_view(ws, cfg, B, T, 0, WS_DG, torch.bfloat16, (M, shape.n_signal * shape.d_v)).clone()
    for call in (1, 2):
        out = torch.full_like(ref, float("nan"))
        gb.gdla_attn_prefill_noalloc(cfg, qq, kv, kr, lam, gate, out, B, T)
        torch.cuda.synchronize()
        assert gb.gdla_device_error() == 0
        check(f"no-alloc Dg, call {call}, B={B} T={T} W={window}", to_np(out), to_np(ref),
              rel=REL_L2, mabs=MAX_ABS)


# (2, 2048, 256): B*T equals the scratch limit, so the last 32-row block of the array is used
@pytest.mark.parametrize("B,T,window", [(1, 300, 0), (2, 2048, 256)])
def test_noalloc_attention_matches_oracle(cuda_ok, B, T, window):
    shape = synth.GdlaShape(window=window)
    cfg_o = O.OracleConfig.from_shape(shape)
    g = torch.Generator().manual_seed(43 + T)
    M = B * T
    qq = torch.randn((M, 80 * 192), generator=g).half()
    kv = torch.randn((M, 16 * 256), generator=g).half()
    kr = torch.randn((M, 64), generator=g).half()
    lam = torch.rand((M, 64), generator=g) * 0.9 + 0.05
    gate = torch.randn((M, 64 * 128), generator=g).bfloat16()
    cfg = gb.make_config(shape)
    dev = [t.cuda() for t in (qq, kv, kr, lam, gate)]
    outs = []
    for call in (1, 2):
        out = torch.full((M, 64 * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        gb.gdla_attn_prefill_noalloc(cfg, *dev, out, B, T)
        torch.cuda.synchronize()
        assert gb.gdla_device_error() == 0
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    errs = []
    for b in range(B):
        r = slice(b * T, (b + 1) * T)
        kvb = O.f64(kv[r]).reshape(T, 16, 256)
        Dg_o, _ = O.attention_stage(O.f64(qq[r, : 80 * 128]).reshape(T, 80, 128),
                                    O.f64(qq[r, 80 * 128:]).reshape(T, 80, 64), kvb[..., :128],
                                    kvb[..., 128:], O.f64(kr[r]), O.f64(lam[r]),
                                    O.f64(gate[r]).reshape(T, 64, 128), cfg_o)
        check(f"no-alloc Dg vs oracle b={b} B={B} T={T} W={window}", to_np(outs[1][r]).reshape(T, 64, 128),
              Dg_o, errors=errs)
    assert not errs, "\n".join(errs)


def test_noalloc_limit_matches_header():
    """The binding's limit is the header's #define (read from include/gdla.h)."""
    import os
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "gdla.h")
    m = re.search(r"#define\s+GDLA_NOALLOC_MAX_TOKENS\s+(\d+)", open(hdr).read())
    assert m and int(m.group(1)) == gb.GDLA_NOALLOC_MAX_TOKENS


def test_noalloc_rejects_more_tokens_than_its_scratch(cuda_ok):
    shape, inp, layer, x = prefill_case(1, 16, 0, seed=2)
    layer.prefill(x)
    torch.cuda.synchronize()
    ws, cfg = layer._ws, layer.cfg
    t = ws[:16].view(torch.float16)
    too_many = gb.GDLA_NOALLOC_MAX_TOKENS + 1
    with pytest.raises(gb.GdlaError) as e:
        gb.gdla_attn_prefill_noalloc(cfg, t, t, t, ws[:16].view(torch.float32), ws[:16].view(torch.bfloat16),
                                     ws[16:32].view(torch.bfloat16), 1, too_many)
    assert e.value.status == -3   # GDLA_ERR_WORKSPACE_TOO_SMALL: nothing was launched
