"""Attention-stage backward on the GPU (saving forward + gdla_attn_bwd through the C ABI)
against the fp64 oracle's gradient, on seeded inputs of the stage itself (q, K, V, k^R,
lambda, gate logits and dL/dDg drawn directly)."""
import numpy as np
import pytest
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from differential_latent_attention_fwd_b200 import synth
from oracle import gdla_oracle as O
from tests.gpu_helpers import check, to_np

pytestmark = pytest.mark.gpu


def _stage_inputs(B, T, seed):
    g = torch.Generator().manual_seed(seed)
    nH, nS, nK = 80, 64, 16
    qq = torch.randn((B * T, nH * 192), generator=g).half()
    kv = torch.randn((B * T, nK * 256), generator=g).half()
    kr = torch.randn((B * T, 64), generator=g).half()
    lam = torch.rand((B * T, nS), generator=g) * 0.9 + 0.05
    gate = torch.randn((B * T, nS * 128), generator=g).bfloat16()
    d_dg = torch.randn((B * T, nS * 128), generator=g).bfloat16()
    return qq, kv, kr, lam, gate, d_dg


def _run_gpu(shape, B, T, qq, kv, kr, lam, gate, d_dg):
    cfg = gb.make_config(shape)
    dev = "cuda"
    t = [v.to(dev) for v in (qq, kv, kr, lam, gate, d_dg)]
    fwd_b, bwd_b = gb.gdla_attn_train_workspace_size(cfg, B, T)
    M = B * T
    dg = torch.empty((M, 64 * 128), dtype=torch.bfloat16, device=dev)
    h = torch.empty((M, 80, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((M, 80), dtype=torch.float32, device=dev)
    gb.gdla_attn_train_fwd(cfg, t[0], t[1], t[2], t[3], t[4], B, T, dg, h, lse,
                           torch.empty(fwd_b, dtype=torch.uint8, device=dev))
    outs = [torch.empty((M, 80 * 192), device=dev), torch.empty((M, 16 * 256), device=dev),
            torch.empty((M, 64), device=dev), torch.empty((M, 64), device=dev),
            torch.empty((M, 64 * 128), device=dev)]
    gb.gdla_attn_bwd(cfg, t[0], t[1], t[2], t[3], t[4], h, lse, t[5], B, T, *outs,
                     torch.empty(bwd_b, dtype=torch.uint8, device=dev))
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    return dg, h, outs


# T > 512 spans several 512-row query blocks (the window case with a key range that starts
# after row 0 in the later blocks)
@pytest.mark.parametrize("B,T,window", [(1, 300, 0), (2, 260, 64), (1, 700, 0), (1, 600, 100)])
def test_attention_backward_matches_oracle(cuda_ok, B, T, window):
    shape = synth.GdlaShape(window=window)
    cfg = O.OracleConfig.from_shape(shape)
    qq, kv, kr, lam, gate, d_dg = _stage_inputs(B, T, seed=41 + T)
    dg, h, (d_qq, d_kv, d_kr, d_lam, d_gate) = _run_gpu(shape, B, T, qq, kv, kr, lam, gate, d_dg)
    errs = []
    for b in range(B):
        r = slice(b * T, (b + 1) * T)
        qC = O.f64(qq[r, : 80 * 128]).reshape(T, 80, 128)
        qR = O.f64(qq[r, 80 * 128:]).reshape(T, 80, 64)
        kvb = O.f64(kv[r]).reshape(T, 16, 256)
        KC, V = kvb[..., :128], kvb[..., 128:]
        kR = O.f64(kr[r])
        lam_b = O.f64(lam[r])
        G = O.f64(gate[r]).reshape(T, 64, 128)
        dDg = O.f64(d_dg[r]).reshape(T, 64, 128)
        Dg_o, H_o = O.attention_stage(qC, qR, KC, V, kR, lam_b, G, cfg)
        check(f"b={b} forward Dg", to_np(dg[r]).reshape(T, 64, 128), Dg_o, errors=errs)
        check(f"b={b} saved H", to_np(h[r]), H_o, rel=6e-3, mabs=5e-2, errors=errs)
        gr = O.attention_stage_backward(qC, qR, KC, V, kR, lam_b, G, dDg, cfg)
        dqq = to_np(d_qq[r])
        dkv = to_np(d_kv[r]).reshape(T, 16, 256)
        for name, got, want in [
            ("dq^C", dqq[:, : 80 * 128].reshape(T, 80, 128), gr["dqC"]),
            ("dq^R", dqq[:, 80 * 128:].reshape(T, 80, 64), gr["dqR"]),
            ("dK^C", dkv[..., :128], gr["dKC"]),
            ("dV", dkv[..., 128:], gr["dV"]),
            ("dk^R", to_np(d_kr[r]), gr["dkR"]),
            ("dlambda", to_np(d_lam[r]), gr["dlam"]),
            ("dG", to_np(d_gate[r]).reshape(T, 64, 128), gr["dG"]),
        ]:
            check(f"b={b} {name}", got, want, rel=1e-2, mabs=np.abs(want).max() * 2e-2 + 1e-3, errors=errs)
    assert not errs, "\n".join(errs)


@pytest.mark.parametrize("window", [0, 2048])
def test_attention_backward_sampled_rows_t8192(cuda_ok, window):
    """T = 8192 (128 key blocks of the dK/dV kernel, 64 query blocks of the dq kernel): the
    gradients of KV group 5 (its noise head and four signal heads) at 48 sampled query rows and
    48 sampled key rows against the oracle, which forms the group's softmax statistics over the
    whole sequence."""
    B, T, j = 1, 8192, 5
    shape = synth.GdlaShape(window=window)
    cfg = O.OracleConfig.from_shape(shape)
    qq, kv, kr, lam, gate, d_dg = _stage_inputs(B, T, seed=77 + window)
    dg, h, (d_qq, d_kv, d_kr, d_lam, d_gate) = _run_gpu(shape, B, T, qq, kv, kr, lam, gate, d_dg)
    q_rows = synth.sample_rows(T, window, 48, seed=3)
    k_rows = synth.sample_rows(T, window, 48, seed=4)
    kvb = O.f64(kv).reshape(T, 16, 256)
    part = O.attention_stage_backward_group(
        O.f64(qq[:, : 80 * 128]).reshape(T, 80, 128), O.f64(qq[:, 80 * 128:]).reshape(T, 80, 64),
        kvb[..., :128], kvb[..., 128:], O.f64(kr), O.f64(lam), O.f64(gate).reshape(T, 64, 128),
        O.f64(d_dg).reshape(T, 64, 128), cfg, j, q_rows, k_rows)
    heads, sig = part["heads"], part["signals"]
    dqq = to_np(d_qq[q_rows]).reshape(len(q_rows), -1)
    got_qC = dqq[:, : 80 * 128].reshape(-1, 80, 128)[:, heads]
    got_qR = dqq[:, 80 * 128:].reshape(-1, 80, 64)[:, heads]
    dkv = to_np(d_kv[k_rows]).reshape(len(k_rows), 16, 256)[:, j]
    errs = []
    for name, got, want in [
        ("dq^C", got_qC, part["dqC"]), ("dq^R", got_qR, part["dqR"]),
        ("dK^C", dkv[:, :128], part["dKC"]), ("dV", dkv[:, 128:], part["dV"]),
        ("dlambda", to_np(d_lam[q_rows])[:, sig], part["dlam"]),
        ("dG", to_np(d_gate[q_rows]).reshape(-1, 64, 128)[:, sig], part["dG"]),
    ]:
        check(f"T={T} W={window} group {j} {name}", got, want, rel=1e-2, mabs=np.abs(want).max() * 2e-2 + 1e-3,
              errors=errs)
    assert not errs, "\n".join(errs)
