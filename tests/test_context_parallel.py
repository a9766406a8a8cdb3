"""Context-parallel driver on CPU ranks (gloo): the exchange of latent rows and the per-rank
prefix calls reproduce the whole sequence.  The per-rank compute is the oracle's prefix form
here (the driver itself is device-agnostic; on GPUs the same calls go to the CUDA library)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from differential_latent_attention_fwd_b200 import synth
from differential_latent_attention_fwd_b200.context_parallel import cp_prefill
from oracle import gdla_oracle as O

SMALL = dict(d_model=64, q_rank=32, kv_rank=16, n_signal=8, n_noise=2, n_kv_heads=2,
             d_nope=8, d_rope=4, d_v=8)


class OracleLayer:
    """The two calls a rank makes, computed by the fp64 oracle."""

    def __init__(self, shape, weights):
        self.window = shape.window
        self.cfg = O.OracleConfig.from_shape(shape)
        self.w = weights
        self.W_aKV = O.f64(weights["W_aKV"])

    def latent(self, x, pos_offset):
        cbar, kR = O.kv_latent(O.f64(x), self.W_aKV, None, pos_offset + np.arange(x.shape[0]), self.cfg)
        return torch.from_numpy(np.concatenate([cbar, kR], -1))

    def prefill_context(self, x, pos_offset, prefix):
        pre = None if prefix is None else prefix.numpy()
        return torch.from_numpy(O.gdla_prefill_after_prefix(x, pre, pos_offset, self.w, self.cfg))

    def quantize_latent_fp8(self, latent):
        self.sent_bytes = int(latent.shape[0]) * O.fp8_row_bytes(latent.shape[1])
        return torch.from_numpy(O.mxfp8_quantize_rows(latent.numpy()))

    def dequantize_latent_fp8(self, stored):
        return torch.from_numpy(O.mxfp8_dequantize_rows(stored.numpy(), self.cfg.kv_rank + self.cfg.d_rope))


def _worker(rank, world, port, window, lengths, seed, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = synth.GdlaShape(window=window, **SMALL)
        inp = synth.make_prefill_inputs(shape, 1, sum(lengths), seed)
        start = sum(lengths[:rank])
        x = inp.x[0, start: start + lengths[rank]]
        y = cp_prefill(OracleLayer(shape, inp.weights), x)
        q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("window,lengths", [
    (0, [7, 13, 10]),        # full causal: all-gather of every rank's latent rows
    (6, [9, 8, 12]),         # window: point-to-point halo of the last W - 1 rows
    (9, [10, 3, 12]),        # a shard shorter than W - 1: all-gather of the tails
    (0, [16, 14]),
])
def test_cp_prefill_matches_whole_sequence(window, lengths):
    world = len(lengths)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, window, lengths, 3, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shape = synth.GdlaShape(window=window, **SMALL)
    inp = synth.make_prefill_inputs(shape, 1, sum(lengths), 3)
    y = O.gdla_prefill(inp.x, inp.weights, O.OracleConfig.from_shape(shape))[0]
    full = np.concatenate([got[r] for r in range(world)], 0)
    np.testing.assert_allclose(full, y, rtol=0, atol=1e-10)


def _worker_subgroup(rank, world, port, window, lengths, seed, q):
    """Ranks 1..world-1 of a world_size `world` job form the context-parallel group; rank 0 is
    outside it (it only takes part in creating the group)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        grp = dist.new_group(list(range(1, world)))
        if rank == 0:
            q.put((rank, None))
            return
        shape = synth.GdlaShape(window=window, **SMALL)
        inp = synth.make_prefill_inputs(shape, 1, sum(lengths), seed)
        gr = rank - 1
        start = sum(lengths[:gr])
        x = inp.x[0, start: start + lengths[gr]]
        y = cp_prefill(OracleLayer(shape, inp.weights), x, group=grp)
        q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("window,lengths", [(6, [9, 8, 12]), (0, [7, 13, 10])])
def test_cp_prefill_on_a_subgroup(window, lengths):
    """The sequence is split over ranks 1..3 of 4: the halo's point-to-point peers are the
    group's neighbours, addressed by their global ranks."""
    world = len(lengths) + 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_subgroup, args=(r, world, port, window, lengths, 3, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shape = synth.GdlaShape(window=window, **SMALL)
    inp = synth.make_prefill_inputs(shape, 1, sum(lengths), 3)
    y = O.gdla_prefill(inp.x, inp.weights, O.OracleConfig.from_shape(shape))[0]
    full = np.concatenate([got[r] for r in range(1, world)], 0)
    np.testing.assert_allclose(full, y, rtol=0, atol=1e-10)


# latent rows of 28 + 4 = 32 values: one MXFP8 block per row
SMALL8 = dict(SMALL, kv_rank=28)


def _worker_fp8(rank, world, port, window, lengths, seed, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = synth.GdlaShape(window=window, **SMALL8)
        inp = synth.make_prefill_inputs(shape, 1, sum(lengths), seed)
        start = sum(lengths[:rank])
        x = inp.x[0, start: start + lengths[rank]]
        lay = OracleLayer(shape, inp.weights)
        y = cp_prefill(lay, x, fp8=True)
        q.put((rank, y.numpy(), lay.sent_bytes))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("window,lengths", [(0, [7, 13, 10]), (6, [9, 8, 12])])
def test_cp_prefill_fp8_exchange(window, lengths):
    """Rows exchanged as MXFP8: each rank's result is the prefix computation over the
    dequantized rows of the ranks before it (its own rows at full precision), and stays close
    to the whole sequence."""
    world = len(lengths)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_fp8, args=(r, world, port, window, lengths, 5, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {r: (y, nb) for r, y, nb in (q.get(timeout=240) for _ in range(world))}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shape = synth.GdlaShape(window=window, **SMALL8)
    cfg = O.OracleConfig.from_shape(shape)
    inp = synth.make_prefill_inputs(shape, 1, sum(lengths), 5)
    x = O.f64(inp.x[0])
    T = sum(lengths)
    cbar, kR = O.kv_latent(x, O.f64(inp.weights["W_aKV"]), None, np.arange(T), cfg)
    rows = np.concatenate([cbar, kR], -1)
    stored = O.mxfp8_dequantize_rows(O.mxfp8_quantize_rows(rows), rows.shape[1])
    y_full = O.gdla_prefill(inp.x, inp.weights, cfg)[0]
    for r in range(world):
        start = sum(lengths[:r])
        lo = 0 if window == 0 else max(0, start - (window - 1))
        pre = stored[lo:start] if start > lo else None
        want = O.gdla_prefill_after_prefix(inp.x[0, start: start + lengths[r]], pre, start, inp.weights, cfg)
        y, nb = got[r]
        np.testing.assert_allclose(y, want, rtol=1e-9, atol=1e-10)
        assert nb == lengths[r] * O.fp8_row_bytes(32)      # 48 bytes a row instead of 64 in bf16
        rel = np.linalg.norm(y - y_full[start: start + lengths[r]]) / np.linalg.norm(y_full[start: start + lengths[r]])
        assert rel < 5e-2, rel
