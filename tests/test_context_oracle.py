"""The oracle's prefix form (the unit of work of a context-parallel rank) against the whole-sequence
oracle: splitting a sequence at any point and handing the later part the latent rows of the
earlier tokens reproduces the whole sequence's rows (row t depends on tokens <= t only, and on
the earlier tokens only through their latent rows)."""
import numpy as np
import pytest

from differential_latent_attention_fwd_b200 import synth
from oracle import gdla_oracle as O

SMALL = dict(d_model=64, q_rank=32, kv_rank=16, n_signal=8, n_noise=2, n_kv_heads=2,
             d_nope=8, d_rope=4, d_v=8)


def _case(window, T=30, seed=7):
    shape = synth.GdlaShape(window=window, **SMALL)
    inp = synth.make_prefill_inputs(shape, 1, T, seed)
    cfg = O.OracleConfig.from_shape(shape)
    y, parts = O.gdla_prefill(inp.x, inp.weights, cfg, return_parts=True)
    lat = np.concatenate([parts[0]["cbar"], parts[0]["kR"]], -1)
    return inp, cfg, y[0], lat


@pytest.mark.parametrize("split", [0, 1, 11, 29])
def test_prefix_form_equals_whole_sequence_causal(split):
    inp, cfg, y, lat = _case(0)
    got = O.gdla_prefill_after_prefix(inp.x[0, split:], lat[:split] if split else None, split,
                                      inp.weights, cfg)
    np.testing.assert_allclose(got, y[split:], rtol=0, atol=1e-10)


@pytest.mark.parametrize("split", [3, 12, 25])
def test_prefix_form_window_needs_only_the_halo(split):
    W = 6
    inp, cfg, y, lat = _case(W)
    n = min(W - 1, split)
    got = O.gdla_prefill_after_prefix(inp.x[0, split:], lat[split - n: split], split, inp.weights, cfg)
    np.testing.assert_allclose(got, y[split:], rtol=0, atol=1e-10)
    # a longer prefix changes nothing
    got2 = O.gdla_prefill_after_prefix(inp.x[0, split:], lat[:split], split, inp.weights, cfg)
    np.testing.assert_allclose(got2, y[split:], rtol=0, atol=1e-10)


def test_prefix_form_positions_matter():
    """The query positions are pos_offset + t: a wrong offset changes the rotary scores."""
    inp, cfg, y, lat = _case(0)
    wrong = O.gdla_prefill_after_prefix(inp.x[0, 10:], lat[:10], 11, inp.weights, cfg)
    assert np.abs(wrong - y[10:]).max() > 1e-6
