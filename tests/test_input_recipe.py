"""The seeded synthetic inputs follow the stated recipe: one CPU generator per workload seed,
draws in a fixed order (x, then the seven weight matrices), standard normal scaled by 1 (x, cache)
or 0.02 (weights), rounded to bf16; decode caches hold exactly cache_len filled rows."""
import torch

from differential_latent_attention_fwd_b200 import synth

SHAPE = synth.GdlaShape()
WEIGHT_SHAPES = {"W_aQ": (4096, 1024), "W_bQ": (1024, 80 * 192), "W_aKV": (4096, 576), "W_bKV": (512, 16 * 256),
                 "W_lambda": (4096, 64), "W_G": (1024, 64 * 128), "W_O": (64 * 128, 4096)}


def test_prefill_inputs_are_seeded_and_follow_the_recipe():
    a = synth.make_prefill_inputs(SHAPE, 1, 128, seed=5)
    b = synth.make_prefill_inputs(SHAPE, 1, 128, seed=5)
    c = synth.make_prefill_inputs(SHAPE, 1, 128, seed=6)
    assert torch.equal(a.x, b.x) and not torch.equal(a.x, c.x)
    assert a.x.dtype == torch.bfloat16 and tuple(a.x.shape) == (1, 128, 4096)
    assert abs(float(a.x.float().std()) - 1.0) < 0.02
    for k, shp in WEIGHT_SHAPES.items():
        w = a.weights[k]
        assert tuple(w.shape) == shp and w.dtype == torch.bfloat16, k
        assert torch.equal(w, b.weights[k]), k
        assert abs(float(w.float().std()) - 0.02) < 0.002, k
    # the draw order is fixed: x comes first, so a longer sequence extends the same stream
    longer = synth.make_prefill_inputs(SHAPE, 1, 256, seed=5)
    assert torch.equal(longer.x[0, :128], a.x[0])


def test_decode_cache_has_exactly_cache_len_rows():
    d = synth.make_decode_inputs(SHAPE, 3, [0, 7, 16], 20, seed=4)
    assert d.cache.dtype == torch.bfloat16 and tuple(d.cache.shape) == (3, 20, 576)
    assert d.cache_len.tolist() == [0, 7, 16]
    for b, n in enumerate([0, 7, 16]):
        assert torch.count_nonzero(d.cache[b, n:]) == 0
        if n:
            assert torch.count_nonzero(d.cache[b, :n]) > 0.99 * n * 576
    e = synth.make_decode_inputs(SHAPE, 3, [0, 7, 16], 20, seed=4)
    assert torch.equal(d.cache, e.cache) and torch.equal(d.x_new, e.x_new)
