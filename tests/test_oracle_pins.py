"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties one part of oracle/gdla_oracle.py to something it does not compute itself:
values printed on the pages, a library routine (torch SDPA, torch rms_norm, complex
arithmetic), a closed form, an invariant the equations imply, or a brute-force loop.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import gdla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny_cfg(window=0, n_signal=8, n_noise=2, n_kv=2, noise_map="grouped"):
    return O.OracleConfig(d_model=48, q_rank=24, kv_rank=16, n_signal=n_signal, n_noise=n_noise,
                          n_kv_heads=n_kv, d_nope=8, d_rope=4, d_v=6, window=window,
                          noise_map=noise_map)


def tiny_weights(cfg, seed=0, std=0.3):
    r = np.random.default_rng(seed)
    nh = cfg.n_heads
    return {
        "W_aQ": r.normal(0, std, (cfg.d_model, cfg.q_rank)),
        "W_bQ": r.normal(0, std, (cfg.q_rank, nh * (cfg.d_nope + cfg.d_rope))),
        "W_aKV": r.normal(0, std, (cfg.d_model, cfg.kv_rank + cfg.d_rope)),
        "W_bKV": r.normal(0, std, (cfg.kv_rank, cfg.n_kv_heads * (cfg.d_nope + cfg.d_v))),
        "W_lambda": r.normal(0, std, (cfg.d_model, cfg.n_signal)),
        "W_G": r.normal(0, std, (cfg.q_rank, cfg.n_signal * cfg.d_v)),
        "W_O": r.normal(0, std, (cfg.n_signal * cfg.d_v, cfg.d_model)),
    }


def tiny_x(cfg, B, T, seed=1):
    return np.random.default_rng(seed).normal(0, 1, (B, T, cfg.d_model))


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if "=" in line:
                k, v = line.split("=", 1)
                vals[k.strip()] = np.array([float(t) for t in v.split()])
    return vals


# ---------------------------------------------------------------- printed worked example
def test_worked_example_combine_and_gate():
    g = _read_golden("worked_example.txt")
    tol = float(g["print_tolerance"][0])
    noise = g["repeat_input"]
    # Repeat_2 as printed = tiled order
    cfg = O.OracleConfig(1, 1, 1, n_signal=4, n_noise=2, n_kv_heads=2, d_nope=1, d_rope=2,
                         d_v=1, noise_map="tiled")
    nmap = O.noise_of_signal(cfg)
    np.testing.assert_allclose(noise[nmap], g["repeat_output"], atol=1e-12)
    lam = g["lambda_times_rep"] / g["repeat_output"]
    H_S = g["D"] + g["lambda_times_rep"]
    D, gated = O.differential_combine(H_S[:, None], noise[:, None], lam, g["gate"][:, None],
                                      nmap, gate_is_logit=False)
    np.testing.assert_allclose(D[:, 0], g["D"], atol=1e-12)
    np.testing.assert_allclose(gated[:, 0], g["gated"], atol=tol)
    # the printed gate values are post-sigmoid: feeding them as logits would not match
    _, as_logit = O.differential_combine(H_S[:, None], noise[:, None], lam, g["gate"][:, None],
                                         nmap, gate_is_logit=True)
    assert np.max(np.abs(as_logit[:, 0] - g["gated"])) > 3 * tol


def test_head_count_rule():
    # n_N = n_H / (g + 1), n_S = g n_N with the Motif 3 sizes (80 query heads, g = 4)
    cfg = O.OracleConfig(4096, 1024, 512, 64, 16, 16, 128, 64, 128)
    assert cfg.n_heads == 80 and cfg.g == 4 and cfg.n_noise == cfg.n_heads // (cfg.g + 1)
    kvh = O.kv_head_of(cfg)
    # every KV head serves exactly one noise head and its g signal heads (16 KV heads shared)
    for j in range(16):
        assert sorted(np.nonzero(kvh == j)[0].tolist()) == [4 * j, 4 * j + 1, 4 * j + 2,
                                                             4 * j + 3, 64 + j]
    assert (O.noise_of_signal(cfg) == np.arange(64) // 4).all()
    gda = O.OracleConfig(64, 32, 16, 4, 4, 4, 8, 4, 8)     # GDA: equal split, g = 1
    assert gda.g == 1 and (O.noise_of_signal(gda) == np.arange(4)).all()


# ---------------------------------------------------------------- library routines
def test_softmax_attention_is_sdpa():
    r = np.random.default_rng(3)
    q, k, v = r.normal(size=(5, 12)), r.normal(size=(33, 12)), r.normal(size=(33, 7))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        scale=0.37)[0].numpy()
    np.testing.assert_allclose(O.softmax_attention(q, k, v, 0.37), ref, rtol=1e-12, atol=1e-13)


def test_rms_norm_is_torch_rms_norm():
    r = np.random.default_rng(4)
    v, gain = r.normal(size=(9, 40)) * 3.0, r.normal(size=40)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(v), (40,), torch.from_numpy(gain),
                                       eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(v, gain, 1e-6), ref, rtol=1e-12)
    # unit gains -> unit RMS (up to eps)
    out = O.rms_norm(v, None, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, -1)), 1.0, rtol=1e-12)


def test_sigmoid_is_torch_sigmoid():
    z = np.linspace(-800, 800, 4001)
    np.testing.assert_allclose(O.sigmoid(z), torch.sigmoid(torch.from_numpy(z)).numpy(),
                               rtol=1e-14, atol=1e-300)


def test_rope_is_complex_rotation_and_relative():
    r = np.random.default_rng(5)
    d, theta = 16, 10000.0
    v = r.normal(size=(7, d))
    pos = np.array([0, 1, 5, 100, 4097, 65536, 262143])
    out = O.rope(v, pos, theta)
    # independent route: pair (i, i + d/2) as a complex number times e^{i pos theta^(-2i/d)}
    z = v[:, : d // 2] + 1j * v[:, d // 2:]
    w = np.exp(1j * pos[:, None] * theta ** (-np.arange(d // 2) * 2.0 / d))
    zr = z * w
    np.testing.assert_allclose(out, np.concatenate([zr.real, zr.imag], -1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.rope(v, np.zeros(7), theta), v, atol=0)       # pos 0 = identity
    np.testing.assert_allclose(np.linalg.norm(out, axis=-1), np.linalg.norm(v, axis=-1), rtol=1e-12)
    # scores depend on the position difference only
    a, b = r.normal(size=d), r.normal(size=d)
    s1 = O.rope(a, np.array(40), theta) @ O.rope(b, np.array(13), theta)
    s2 = O.rope(a, np.array(1027), theta) @ O.rope(b, np.array(1000), theta)
    assert abs(s1 - s2) < 1e-10


# ---------------------------------------------------------------- full layer vs SDPA
def _sdpa_heads(parts, cfg, T, window):
    """Per-head outputs of the full layer recomputed with torch SDPA from the oracle's q/k/v."""
    qC, qR, KC, kR, V = (parts[k] for k in ("qC", "qR", "KC", "kR", "V"))
    kvh = O.kv_head_of(cfg)
    t = np.arange(T)
    mask = t[None, :] <= t[:, None]
    if window:
        mask &= t[None, :] > t[:, None] - window
    H = np.empty((T, cfg.n_heads, cfg.d_v))
    for h in range(cfg.n_heads):
        j = kvh[h]
        q = torch.from_numpy(np.concatenate([qC[:, h], qR[:, h]], -1))
        k = torch.from_numpy(np.concatenate([KC[:, j], kR], -1))
        H[:, h] = torch.nn.functional.scaled_dot_product_attention(
            q[None], k[None], torch.from_numpy(V[:, j])[None], attn_mask=torch.from_numpy(mask)[None],
            scale=1 / math.sqrt(cfg.d_nope + cfg.d_rope))[0].numpy()
    return H


@pytest.mark.parametrize("window", [0, 4])
def test_full_layer_attention_matches_sdpa(window):
    cfg = tiny_cfg(window=window)
    W = tiny_weights(cfg)
    T = 11
    x = tiny_x(cfg, 1, T)
    y, parts = O.gdla_prefill(x, W, cfg, return_parts=True)
    p = parts[0]
    H = _sdpa_heads(p, cfg, T, window)
    nm = O.noise_of_signal(cfg)
    D = H[:, : cfg.n_signal] - p["lam"][:, :, None] * H[:, cfg.n_signal:][:, nm]
    Dg = torch.sigmoid(torch.from_numpy(p["G"])).numpy() * D
    np.testing.assert_allclose(p["Dg"], Dg, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(y[0], Dg.reshape(T, -1) @ W["W_O"], rtol=1e-11, atol=1e-11)


def test_lambda_zero_reduces_to_gated_mla():
    """lambda = 0: noise heads drop out; output = gated multi-head latent attention."""
    cfg = tiny_cfg()
    W = tiny_weights(cfg)
    T = 9
    x = tiny_x(cfg, 1, T)
    _, parts = O.gdla_prefill(x, W, cfg, return_parts=True)
    p = parts[0]
    H = _sdpa_heads(p, cfg, T, 0)
    for t in range(T):
        Hrow = O.attend_row(p["qC"][t], p["qR"][t], p["KC"], p["kR"], p["V"], 0, t, cfg)
        Dg0, _ = O.combine_row(Hrow, np.zeros(cfg.n_signal), p["G"][t], W["W_O"], cfg)
        qC2 = p["qC"][t].copy()
        qC2[cfg.n_signal:] += 5.0                         # perturb every noise query
        Hrow2 = O.attend_row(qC2, p["qR"][t], p["KC"], p["kR"], p["V"], 0, t, cfg)
        Dg1, _ = O.combine_row(Hrow2, np.zeros(cfg.n_signal), p["G"][t], W["W_O"], cfg)
        np.testing.assert_array_equal(Dg0, Dg1)
        mla = O.sigmoid(p["G"][t]) * H[t, : cfg.n_signal]
        np.testing.assert_allclose(Dg0, mla, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- closed forms / invariants
@pytest.mark.parametrize("window", [0, 1])
def test_single_key_gives_one_minus_lambda_times_v(window):
    cfg = tiny_cfg(window=window)
    W = tiny_weights(cfg)
    T = 7
    x = tiny_x(cfg, 1, T)
    _, parts = O.gdla_prefill(x, W, cfg, return_parts=True)
    p = parts[0]
    kv_s = O.kv_head_of(cfg)[: cfg.n_signal]
    rows = range(T) if window == 1 else [0]
    for t in rows:   # one visible key: both maps equal V_{j,t}, D_s = (1 - lambda_s) V
        want = O.sigmoid(p["G"][t]) * (1 - p["lam"][t])[:, None] * p["V"][t, kv_s]
        np.testing.assert_allclose(p["Dg"][t], want, rtol=1e-12, atol=1e-13)


def test_sliding_window_equals_truncated_causal():
    Wn = 5
    cfg_swa, cfg_full = tiny_cfg(window=Wn), tiny_cfg(window=0)
    W = tiny_weights(cfg_swa)
    T = 16
    x = tiny_x(cfg_swa, 1, T)
    y = O.gdla_prefill(x, W, cfg_swa)
    for t in [0, 3, 4, 5, 9, 15]:
        lo = max(0, t - Wn + 1)
        ref = O.gdla_prefill(x[:, lo: t + 1], W, cfg_full, pos_offset=lo)[0, -1]
        np.testing.assert_allclose(y[0, t], ref, rtol=1e-12, atol=1e-12)
        ref0 = O.gdla_prefill(x[:, lo: t + 1], W, cfg_full, pos_offset=0)[0, -1]
        np.testing.assert_allclose(y[0, t], ref0, rtol=1e-9, atol=1e-10)   # RoPE is relative


def test_causality():
    cfg = tiny_cfg()
    W = tiny_weights(cfg)
    T = 10
    x = tiny_x(cfg, 1, T)
    y = O.gdla_prefill(x, W, cfg)
    x2 = x.copy()
    x2[0, 6:] += np.random.default_rng(9).normal(size=(T - 6, cfg.d_model))
    y2 = O.gdla_prefill(x2, W, cfg)
    np.testing.assert_allclose(y2[0, :6], y[0, :6], rtol=0, atol=1e-14)
    assert np.abs(y2[0, 6:] - y[0, 6:]).min() > 0


def test_noise_map_orders_are_a_head_permutation():
    """grouped and tiled Repeat_g agree once signal heads are permuted in W_bQ, W_G, W_lambda, W_O."""
    cfg_g = tiny_cfg(n_signal=8, n_noise=2, n_kv=2)
    # a one-KV-head variant so that permuting signal heads does not change their KV head
    cfg_g = O.OracleConfig(**{**cfg_g.__dict__, "n_kv_heads": 1})
    cfg_t = O.OracleConfig(**{**cfg_g.__dict__, "noise_map": "tiled"})
    W = tiny_weights(cfg_g)
    x = tiny_x(cfg_g, 1, 6)
    g, nN = cfg_g.g, cfg_g.n_noise
    # tiled signal head s' pairs with noise s' % nN; grouped head s pairs with s // g.
    perm = np.array([(s % g) * nN + s // g for s in range(cfg_g.n_signal)])  # grouped s -> tiled s'
    assert (np.arange(cfg_g.n_signal) // g == perm % nN).all()
    inv = np.argsort(perm)
    Wt = dict(W)
    dq = cfg_g.d_nope
    nc = cfg_g.n_heads * dq
    qc = W["W_bQ"][:, :nc].reshape(-1, cfg_g.n_heads, dq)
    qr = W["W_bQ"][:, nc:].reshape(-1, cfg_g.n_heads, cfg_g.d_rope)
    sig_perm = np.concatenate([inv, np.arange(cfg_g.n_signal, cfg_g.n_heads)])
    Wt["W_bQ"] = np.concatenate([qc[:, sig_perm].reshape(cfg_g.q_rank, -1),
                                 qr[:, sig_perm].reshape(cfg_g.q_rank, -1)], 1)
    Wt["W_lambda"] = W["W_lambda"][:, inv]
    dv = cfg_g.d_v
    Wt["W_G"] = W["W_G"].reshape(cfg_g.q_rank, cfg_g.n_signal, dv)[:, inv].reshape(cfg_g.q_rank, -1)
    Wt["W_O"] = W["W_O"].reshape(cfg_g.n_signal, dv, -1)[inv].reshape(cfg_g.n_signal * dv, -1)
    np.testing.assert_allclose(O.gdla_prefill(x, Wt, cfg_t), O.gdla_prefill(x, W, cfg_g),
                               rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- decode routes
def _random_cache(cfg, B, cap, lens, seed=7):
    r = np.random.default_rng(seed)
    c = np.zeros((B, cap, cfg.kv_rank + cfg.d_rope))
    for b, L in enumerate(lens):
        c[b, :L] = r.normal(size=(L, cfg.kv_rank + cfg.d_rope))
    return c


@pytest.mark.parametrize("window", [0, 3])
def test_absorbed_decode_equals_literal(window):
    cfg = tiny_cfg(window=window)
    W = tiny_weights(cfg)
    lens = [0, 1, 5, 12]
    cache = _random_cache(cfg, 4, 13, lens)
    xn = np.random.default_rng(8).normal(size=(4, cfg.d_model))
    a = O.gdla_decode(xn, W, cache, lens, cfg)
    b = O.gdla_decode_absorbed(xn, W, cache, lens, cfg)
    np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("window", [0, 4])
def test_decode_continues_prefill(window):
    """Decoding token t over the latent rows prefill produced for tokens < t = prefill row t."""
    cfg = tiny_cfg(window=window)
    W = tiny_weights(cfg)
    T = 10
    x = tiny_x(cfg, 1, T)
    y, parts = O.gdla_prefill(x, W, cfg, return_parts=True)
    rows = np.concatenate([parts[0]["cbar"], parts[0]["kR"]], -1)
    for t in [0, 1, 6, 9]:
        cache = np.zeros((1, T, rows.shape[1]))
        cache[0, :t] = rows[:t]
        yd = O.gdla_decode(x[:, t], W, cache, [t], cfg)
        np.testing.assert_allclose(yd[0], y[0, t], rtol=1e-10, atol=1e-11)
        ya = O.gdla_decode_absorbed(x[:, t], W, cache, [t], cfg)
        np.testing.assert_allclose(ya[0], y[0, t], rtol=1e-10, atol=1e-11)


# ---------------------------------------------------------------- brute force
def _brute_prefill(x, W, cfg):
    """Scalar loops over every index; no numpy matmul, reshape or broadcasting."""
    T, d = x.shape
    nH, dn, dr, dv, nS = cfg.n_heads, cfg.d_nope, cfg.d_rope, cfg.d_v, cfg.n_signal
    kvh = [s // (nS // cfg.n_kv_heads) for s in range(nS)] + \
          [n // (cfg.n_noise // cfg.n_kv_heads) for n in range(cfg.n_noise)]

    def mv(vec, M):
        return [sum(vec[i] * M[i][o] for i in range(len(vec))) for o in range(len(M[0]))]

    def rms(v):
        m = math.sqrt(sum(e * e for e in v) / len(v) + cfg.rms_eps)
        return [e / m for e in v]

    def rot(v, p):
        h = len(v) // 2
        out = [0.0] * len(v)
        for i in range(h):
            a = p * cfg.rope_theta ** (-2.0 * i / len(v))
            out[i] = v[i] * math.cos(a) - v[i + h] * math.sin(a)
            out[i + h] = v[i + h] * math.cos(a) + v[i] * math.sin(a)
        return out

    Wl = {k: v.tolist() for k, v in W.items()}
    q, k, vv, lam, G = [], [], [], [], []
    for t in range(T):
        xt = x[t].tolist()
        cq = rms(mv(xt, Wl["W_aQ"]))
        qq = mv(cq, Wl["W_bQ"])
        q.append([qq[h * dn:(h + 1) * dn] + rot(qq[nH * dn + h * dr: nH * dn + (h + 1) * dr], t)
                  for h in range(nH)])
        ck = mv(xt, Wl["W_aKV"])
        cb = rms(ck[: cfg.kv_rank])
        kr = rot(ck[cfg.kv_rank:], t)
        kvf = mv(cb, Wl["W_bKV"])
        blk = dn + dv
        k.append([kvf[j * blk: j * blk + dn] + kr for j in range(cfg.n_kv_heads)])
        vv.append([kvf[j * blk + dn: (j + 1) * blk] for j in range(cfg.n_kv_heads)])
        lam.append([1 / (1 + math.exp(-z)) for z in mv(xt, Wl["W_lambda"])])
        G.append(mv(cq, Wl["W_G"]))
    y = []
    for t in range(T):
        lo = 0 if cfg.window == 0 else max(0, t - cfg.window + 1)
        H = []
        for h in range(nH):
            j = kvh[h]
            sc = [sum(a * b for a, b in zip(q[t][h], k[s][j])) / math.sqrt(dn + dr)
                  for s in range(lo, t + 1)]
            m = max(sc)
            e = [math.exp(v - m) for v in sc]
            z = sum(e)
            H.append([sum(e[i] / z * vv[lo + i][j][c] for i in range(len(e))) for c in range(dv)])
        flat = []
        for s in range(nS):
            n = s // cfg.g
            for c in range(dv):
                dval = H[s][c] - lam[t][s] * H[nS + n][c]
                flat.append(dval / (1 + math.exp(-G[t][s * dv + c])))
        y.append(mv(flat, Wl["W_O"]))
    return np.array(y)


@pytest.mark.parametrize("window", [0, 3])
def test_brute_force_tiny(window):
    cfg = tiny_cfg(window=window)
    W = tiny_weights(cfg, seed=11)
    x = tiny_x(cfg, 1, 6, seed=12)
    np.testing.assert_allclose(O.gdla_prefill(x, W, cfg)[0], _brute_prefill(x[0], W, cfg),
                               rtol=1e-11, atol=1e-12)


def test_masked_softmax_attention_is_sdpa_with_mask():
    r = np.random.default_rng(13)
    q, k, v = r.normal(size=(6, 3, 10)), r.normal(size=(17, 10)), r.normal(size=(17, 4))
    allowed = r.random((6, 17)) < 0.6
    allowed[:, 0] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(0, 1), torch.from_numpy(k)[None].expand(3, 17, 10),
        torch.from_numpy(v)[None].expand(3, 17, 4), attn_mask=torch.from_numpy(allowed)[None],
        scale=0.29).transpose(0, 1).numpy()
    np.testing.assert_allclose(O.masked_softmax_attention(q, k, v, 0.29, allowed), ref,
                               rtol=1e-12, atol=1e-13)


def test_prefill_row_subsets_and_order_agree():
    """Sampled rows (any order, any chunking) equal the same rows of the all-rows run."""
    for window in (0, 5):
        cfg = tiny_cfg(window=window)
        W = tiny_weights(cfg)
        x = tiny_x(cfg, 2, 40)
        full = O.gdla_prefill(x, W, cfg)
        rows = [39, 3, 17, 0, 25, 26, 8]
        sub = O.gdla_prefill(x, W, cfg, rows=rows)
        np.testing.assert_allclose(sub, full[:, rows], rtol=1e-12, atol=1e-13)


def test_packed_documents_do_not_interact():
    """Packed prefill: perturbing one document changes no other document's rows, and a
    document's rows equal a standalone run of that document."""
    cfg = tiny_cfg(window=3)
    W = tiny_weights(cfg)
    x = tiny_x(cfg, 1, 17)[0]
    cu = [0, 5, 6, 13, 17]
    y = O.gdla_prefill_packed(x, cu, W, cfg)
    x2 = x.copy()
    x2[6:13] += 1.0
    y2 = O.gdla_prefill_packed(x2, cu, W, cfg)
    np.testing.assert_array_equal(y2[:6], y[:6])
    np.testing.assert_array_equal(y2[13:], y[13:])
    assert np.abs(y2[6:13] - y[6:13]).min() > 0
    np.testing.assert_allclose(y[13:17], O.gdla_prefill(x[None, 13:17], W, cfg)[0], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("window", [0, 3])
def test_multi_token_decode_continues_prefill(window):
    """q_len tokens decoded at once over prefill's latent rows of the earlier tokens equal the
    prefill rows of those tokens (literal and absorbed routes)."""
    cfg = tiny_cfg(window=window)
    W = tiny_weights(cfg)
    T = 11
    x = tiny_x(cfg, 1, T)
    y, parts = O.gdla_prefill(x, W, cfg, return_parts=True)
    rows = np.concatenate([parts[0]["cbar"], parts[0]["kR"]], -1)
    t0, q = 7, 4
    cache = np.zeros((1, T, rows.shape[1]))
    cache[0, :t0] = rows[:t0]
    for route in ("literal", "absorbed"):
        ym = O.gdla_decode_multi(x[:, t0:t0 + q], W, cache, [t0], cfg, route=route)
        np.testing.assert_allclose(ym[0], y[0, t0:t0 + q], rtol=1e-10, atol=1e-11)
