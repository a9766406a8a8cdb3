"""The oracle's attention-stage gradient against central finite differences of the oracle's
attention-stage forward (an independent check of every term of the chain rule)."""
import numpy as np
import pytest

from oracle import gdla_oracle as O

SMALL = dict(d_model=64, q_rank=32, kv_rank=16, n_signal=8, n_noise=2, n_kv_heads=2, d_nope=8,
             d_rope=4, d_v=8)


def _inputs(window, T=7, seed=5):
    from differential_latent_attention_fwd_b200 import synth
    cfg = O.OracleConfig.from_shape(synth.GdlaShape(window=window, **SMALL))
    r = np.random.default_rng(seed)
    x = dict(qC=r.normal(size=(T, cfg.n_heads, cfg.d_nope)), qR=r.normal(size=(T, cfg.n_heads, cfg.d_rope)),
             KC=r.normal(size=(T, cfg.n_kv_heads, cfg.d_nope)), V=r.normal(size=(T, cfg.n_kv_heads, cfg.d_v)),
             kR=r.normal(size=(T, cfg.d_rope)), lam=r.uniform(0.05, 0.95, size=(T, cfg.n_signal)),
             G=r.normal(size=(T, cfg.n_signal, cfg.d_v)))
    dDg = r.normal(size=(T, cfg.n_signal, cfg.d_v))
    return cfg, x, dDg


@pytest.mark.parametrize("window", [0, 3])
def test_backward_matches_finite_differences(window):
    cfg, x, dDg = _inputs(window)
    grads = O.attention_stage_backward(x["qC"], x["qR"], x["KC"], x["V"], x["kR"], x["lam"], x["G"], dDg, cfg)

    def loss(xx):
        Dg, _ = O.attention_stage(xx["qC"], xx["qR"], xx["KC"], xx["V"], xx["kR"], xx["lam"], xx["G"], cfg)
        return float(np.sum(dDg * Dg))

    r = np.random.default_rng(11)
    eps = 1e-6
    for name in ["qC", "qR", "KC", "V", "kR", "lam", "G"]:
        g = grads["d" + name]
        for _ in range(6):
            idx = tuple(int(r.integers(0, n)) for n in x[name].shape)
            xp = {k: v.copy() for k, v in x.items()}
            xm = {k: v.copy() for k, v in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            assert abs(fd - g[idx]) <= 1e-6 * (1 + abs(fd)), (name, idx, fd, g[idx])


def test_backward_of_first_row_only_touches_key_zero():
    """Row 0 sees only key 0: gradients of later keys come only from later rows."""
    cfg, x, dDg = _inputs(0)
    dDg[1:] = 0
    g = O.attention_stage_backward(x["qC"], x["qR"], x["KC"], x["V"], x["kR"], x["lam"], x["G"], dDg, cfg)
    assert np.abs(g["dKC"][1:]).max() == 0 and np.abs(g["dV"][1:]).max() == 0
    assert np.abs(g["dqC"][1:]).max() == 0
    # a single key: softmax is constant, so no gradient flows to q or K
    assert np.abs(g["dqC"][0]).max() < 1e-12 and np.abs(g["dKC"][0]).max() < 1e-12


@pytest.mark.parametrize("window", [0, 5])
def test_group_backward_equals_full_backward(window):
    """The group-restricted gradient at chosen rows (used at long lengths) equals the full
    oracle gradient's rows of that group, which the finite-difference test above pins."""
    cfg, x, dDg = _inputs(window, T=23, seed=8)
    full = O.attention_stage_backward(x["qC"], x["qR"], x["KC"], x["V"], x["kR"], x["lam"], x["G"], dDg, cfg)
    q_rows, k_rows = [0, 4, 11, 22], [0, 3, 17, 22]
    for j in range(cfg.n_kv_heads):
        part = O.attention_stage_backward_group(x["qC"], x["qR"], x["KC"], x["V"], x["kR"], x["lam"], x["G"],
                                                dDg, cfg, j, q_rows, k_rows, block=5)
        heads, sig = part["heads"], part["signals"]
        np.testing.assert_allclose(part["dqC"], full["dqC"][q_rows][:, heads], rtol=0, atol=1e-11)
        np.testing.assert_allclose(part["dqR"], full["dqR"][q_rows][:, heads], rtol=0, atol=1e-11)
        np.testing.assert_allclose(part["dKC"], full["dKC"][k_rows, j], rtol=0, atol=1e-11)
        np.testing.assert_allclose(part["dV"], full["dV"][k_rows, j], rtol=0, atol=1e-11)
        np.testing.assert_allclose(part["dlam"], full["dlam"][q_rows][:, sig], rtol=0, atol=1e-11)
        np.testing.assert_allclose(part["dG"], full["dG"][q_rows][:, sig], rtol=0, atol=1e-11)
