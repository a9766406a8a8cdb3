"""Shared helpers of the GPU parity tests: seeded inputs, runs through the C ABI, oracle refs."""
from __future__ import annotations

import numpy as np
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from differential_latent_attention_fwd_b200 import synth
from differential_latent_attention_fwd_b200.layer import GdlaLayer
from oracle import gdla_oracle as O

# Parity bar of the layer output against the fp64 oracle.
MAX_ABS = 2e-2
REL_L2 = 5e-3

# workspace slots (gdla_workspace_offset)
WS_D1, WS_CQ, WS_LATENT, WS_LAM, WS_QQ, WS_G, WS_KV, WS_ONOISE, WS_DG, WS_KR16 = range(10)


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))


def max_abs(got, want) -> float:
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))))


def check(name, got, want, rel=REL_L2, mabs=MAX_ABS, errors=None):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    finite = bool(np.isfinite(got).all())
    r, m = rel_l2(got, want), max_abs(got, want)
    ok = finite and r <= rel and m <= mabs
    msg = f"{name}: rel_l2={r:.3e} (<= {rel:.1e}) max_abs={m:.3e} (<= {mabs:.1e}) finite={finite}"
    print(msg)     # shown with pytest -s: the measured errors beside their bounds
    if errors is not None:
        if not ok:
            errors.append(msg)
        return ok
    assert ok, msg
    return ok


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def ws_view(ws: torch.Tensor, cfg, B, T, mode, which, dtype, shape) -> torch.Tensor:
    off = gb.gdla_workspace_offset(cfg, B, T, mode, which)
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    return ws[off: off + n].view(dtype).view(*shape)


def prefill_case(B, T, window, seed, device="cuda"):
    shape = synth.GdlaShape(window=window)
    inp = synth.make_prefill_inputs(shape, B, T, seed)
    layer = GdlaLayer(shape, inp.weights, inp.g_q, inp.g_kv, device=device)
    x = inp.x.to(device)
    return shape, inp, layer, x


def oracle_prefill(inp, rows=None, parts=False):
    cfg = O.OracleConfig.from_shape(inp.shape)
    return O.gdla_prefill(inp.x, inp.weights, cfg, rows=rows, g_q=inp.g_q, g_kv=inp.g_kv,
                          return_parts=parts)
