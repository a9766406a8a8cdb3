"""GPU context prefill (the per-rank unit of context parallelism) through the C ABI: a sequence
run as consecutive chunks, each after the latent rows of the tokens before it, against the
whole-sequence prefill on the GPU and against the fp64 oracle.  The chunks run one after the
other on one device (no rank waits on another)."""
import numpy as np
import pytest
import torch

from differential_latent_attention_fwd_b200 import binding as gb
from tests.gpu_helpers import check, oracle_prefill, prefill_case, to_np

pytestmark = pytest.mark.gpu


def _run_chunks(layer, x, lengths, window, halo_only=True):
    """y and latent rows of x [T, d] computed chunk by chunk; a window chunk gets only the last
    W - 1 latent rows before it when halo_only."""
    ys, lats, start = [], [], 0
    for L in lengths:
        xc = x[start: start + L].contiguous()
        lat = layer.latent(xc, start)
        if start == 0:
            prefix = None
        else:
            allp = torch.cat(lats, 0)
            n = start if (window == 0 or not halo_only) else min(window - 1, start)
            prefix = allp[start - n:].contiguous()
        lat_out = torch.empty_like(lat)
        ys.append(layer.prefill_context(xc, start, prefix, latent_out=lat_out))
        torch.cuda.synchronize()
        assert gb.gdla_device_error() == 0
        assert torch.equal(lat_out, lat), "latent rows of the context call differ from gdla_latent_fwd"
        lats.append(lat)
        start += L
    return torch.cat(ys, 0), torch.cat(lats, 0)


@pytest.mark.parametrize("window,lengths", [
    (0, [300, 256, 444]),
    (0, [1, 511, 512, 3]),
    (128, [200, 129, 1, 370]),
    (128, [100, 100, 100]),      # chunks shorter than W - 1: the prefix spans several chunks
])
def test_context_chunks_match_whole_sequence(cuda_ok, window, lengths):
    T = sum(lengths)
    shape, inp, layer, x = prefill_case(1, T, window, seed=13)
    cache = torch.zeros((1, T, 576), dtype=torch.bfloat16, device="cuda")
    y_full = layer.prefill(x, kv_cache_out=cache)
    y_cp, lat_cp = _run_chunks(layer, x[0], lengths, window)
    errs = []
    # latent rows: same kernels on the same rows
    check("latent rows, chunked vs whole", to_np(lat_cp), to_np(cache[0]), rel=4e-3, mabs=5e-2, errors=errs)
    # outputs: the prefix keys' rotary part is read back from bf16 rows (as in decode)
    check("y, chunked vs whole GPU prefill", to_np(y_cp), to_np(y_full[0]), rel=3e-3, mabs=1.5e-2, errors=errs)
    rows = sorted(set([0, T - 1] + list(np.cumsum(lengths)[:-1]) + list(np.cumsum(lengths)[:-1] - 1)
                      + list(np.linspace(0, T - 1, 24).astype(int))))
    yo = oracle_prefill(inp, rows=rows)
    check(f"y, chunked vs oracle ({len(rows)} rows)", to_np(y_cp[rows]), yo[0], errors=errs)
    assert not errs, "\n".join(errs)


def test_context_window_prefix_longer_than_halo_is_ignored(cuda_ok):
    """Passing every earlier latent row instead of the last W - 1 gives the same result (up to
    rounding: a longer prefix moves the 128-key tile boundaries the online softmax walks)."""
    shape, inp, layer, x = prefill_case(1, 700, 128, seed=17)
    a, _ = _run_chunks(layer, x[0], [300, 400], 128, halo_only=True)
    b, _ = _run_chunks(layer, x[0], [300, 400], 128, halo_only=False)
    check("window chunk: halo-only vs whole prefix", to_np(b), to_np(a), rel=3e-3, mabs=1.5e-2)


def test_context_chunks_t8192(cuda_ok):
    """Four 2048-token chunks of an 8192-token causal sequence (sampled oracle rows)."""
    lengths = [2048] * 4
    T = sum(lengths)
    shape, inp, layer, x = prefill_case(1, T, 0, seed=19)
    y_full = layer.prefill(x)
    y_cp, _ = _run_chunks(layer, x[0], lengths, 0)
    errs = []
    check("T=8192 chunked vs whole GPU prefill", to_np(y_cp), to_np(y_full[0]), rel=3e-3, mabs=1.5e-2, errors=errs)
    rows = sorted(set([0, 2047, 2048, 4095, 4096, 6143, 6144, T - 1] + list(np.linspace(0, T - 1, 40).astype(int))))
    yo = oracle_prefill(inp, rows=rows)
    check("T=8192 chunked vs oracle", to_np(y_cp[rows]), yo[0], errors=errs)
    assert not errs, "\n".join(errs)


def test_context_rejects_bad_offsets(cuda_ok):
    shape, inp, layer, x = prefill_case(1, 64, 0, seed=2)
    lat = layer.latent(x[0, :32].contiguous(), 0)
    with pytest.raises(gb.GdlaError):
        layer.prefill_context(x[0, 32:].contiguous(), 16, lat)     # 32 prefix rows before position 16


@pytest.mark.parametrize("window", [0, 128])
def test_context_chunk_after_fp8_prefix(cuda_ok, window):
    """The MXFP8 exchange of context parallelism on the GPU: the prefix rows are quantized and
    dequantized by the library, and the chunk after them matches the oracle's prefix form over
    the oracle's MXFP8 round trip of the (bf16) latent rows."""
    from oracle import gdla_oracle as O
    T0, T1 = 400, 300
    shape, inp, layer, x = prefill_case(1, T0 + T1, window, seed=19)
    lat0 = layer.latent(x[0, :T0].contiguous(), 0)
    n = T0 if window == 0 else window - 1
    stored = layer.quantize_latent_fp8(lat0[T0 - n:].contiguous())
    assert stored.shape == (n, 608) and stored.dtype == torch.uint8
    prefix = layer.dequantize_latent_fp8(stored)
    y1 = layer.prefill_context(x[0, T0:].contiguous(), T0, prefix)
    torch.cuda.synchronize()
    assert gb.gdla_device_error() == 0
    cfg = O.OracleConfig.from_shape(shape)
    cbar, kR = O.kv_latent(O.f64(inp.x[0, :T0]), O.f64(inp.weights["W_aKV"]), O.f64(inp.g_kv), np.arange(T0), cfg)
    rows_bf16 = torch.tensor(np.concatenate([cbar, kR], -1)[T0 - n:]).to(torch.bfloat16).double().numpy()
    pre_o = O.mxfp8_dequantize_rows(O.mxfp8_quantize_rows(rows_bf16), 576)
    rows = list(range(0, T1, 7)) + [T1 - 1]
    yo = O.gdla_prefill_after_prefix(inp.x[0, T0:], pre_o, T0, inp.weights, cfg, g_q=inp.g_q, g_kv=inp.g_kv)
    check(f"chunk after an MXFP8 prefix, W={window}", to_np(y1[rows]), yo[rows])
