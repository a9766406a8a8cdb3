"""Seeded synthetic inputs for one GDLA layer (shared by the tests, the bench and the oracle's callers).

This module only draws random numbers and holds shape constants; it contains none of the
layer's arithmetic.  Both the CUDA path and the CPU oracle are fed from here, so that they
see bit-identical bf16 inputs.

Recipe (Motif 3 Technical Report, hotpaper.ai page, "기술적 접근법" list: 80 query heads,
16 KV heads, latent ranks 1024/512, d_model 4096; head dims 128 nope + 64 rope and v 128,
the window 2048 and the value distributions are fixed by the workload definition, not by
the pages):

* a CPU ``torch.Generator`` seeded with ``seed`` draws, in this order,
  x, W_aQ, W_bQ, W_aKV, W_bKV, W_lambda, W_G, W_O  (then, for decode, the latent cache);
* every tensor is drawn as float32 standard normal, scaled (x and cache by 1, weights by
  0.02) and rounded to bf16;
* RMSNorm gains are ones.

Weights are stored the way the pages write the products ``x W``: row-major
``[in_features, out_features]``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class GdlaShape:
    """Layer dimensions (Motif 3 GDLA: d 4096, ranks 1024/512, 64 signal + 16 noise heads)."""

    d_model: int = 4096
    q_rank: int = 1024
    kv_rank: int = 512
    n_signal: int = 64
    n_noise: int = 16
    n_kv_heads: int = 16
    d_nope: int = 128
    d_rope: int = 64
    d_v: int = 128
    window: int = 0          # 0 = full causal, else sliding window of W keys (self included)
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6

    @property
    def n_heads(self) -> int:
        return self.n_signal + self.n_noise

    @property
    def group(self) -> int:
        return self.n_signal // self.n_noise

    @property
    def d_qk(self) -> int:
        return self.d_nope + self.d_rope

    @property
    def latent_row(self) -> int:
        """Width of one latent-cache row: normalised c^KV followed by the rotated k^R."""
        return self.kv_rank + self.d_rope

    def with_window(self, window: int) -> "GdlaShape":
        return GdlaShape(**{**self.__dict__, "window": window})


WEIGHT_NAMES = ("W_aQ", "W_bQ", "W_aKV", "W_bKV", "W_lambda", "W_G", "W_O")


def weight_shapes(s: GdlaShape) -> dict:
    """[in, out] shape of every projection, in draw order."""
    return {
        "W_aQ": (s.d_model, s.q_rank),
        "W_bQ": (s.q_rank, s.n_heads * (s.d_nope + s.d_rope)),
        "W_aKV": (s.d_model, s.kv_rank + s.d_rope),
        "W_bKV": (s.kv_rank, s.n_kv_heads * (s.d_nope + s.d_v)),
        "W_lambda": (s.d_model, s.n_signal),
        "W_G": (s.q_rank, s.n_signal * s.d_v),
        "W_O": (s.n_signal * s.d_v, s.d_model),
    }


def _normal_bf16(gen: torch.Generator, shape, std: float, chunk_rows: int = 1 << 14) -> torch.Tensor:
    """float32 N(0, std^2) rounded to bf16, drawn in row chunks to bound host memory."""
    shape = tuple(int(v) for v in shape)
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1, shape[-1]) if len(shape) > 1 else out.view(1, -1)
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        blk = torch.randn((r1 - r0, flat.shape[1]), generator=gen, dtype=torch.float32)
        if std != 1.0:
            blk.mul_(std)
        flat[r0:r1].copy_(blk)
    return out


@dataclass
class PrefillInputs:
    shape: GdlaShape
    x: torch.Tensor                       # [B, T, d] bf16
    weights: dict = field(default_factory=dict)   # name -> [in, out] bf16
    g_q: torch.Tensor | None = None       # [q_rank] bf16 (ones)
    g_kv: torch.Tensor | None = None      # [kv_rank] bf16 (ones)


def make_weights(gen: torch.Generator, s: GdlaShape, std: float = 0.02) -> dict:
    return {name: _normal_bf16(gen, shp, std) for name, shp in weight_shapes(s).items()}


def make_prefill_inputs(s: GdlaShape, B: int, T: int, seed: int, std_w: float = 0.02) -> PrefillInputs:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    x = _normal_bf16(gen, (B, T, s.d_model), 1.0)
    w = make_weights(gen, s, std_w)
    ones_q = torch.ones(s.q_rank, dtype=torch.bfloat16)
    ones_kv = torch.ones(s.kv_rank, dtype=torch.bfloat16)
    return PrefillInputs(s, x, w, ones_q, ones_kv)


@dataclass
class DecodeInputs:
    shape: GdlaShape
    x_new: torch.Tensor                   # [B, d] bf16
    weights: dict
    g_q: torch.Tensor
    g_kv: torch.Tensor
    cache: torch.Tensor                   # [B, cap, kv_rank + d_rope] bf16; rows >= cache_len are zero
    cache_len: torch.Tensor               # [B] int32, keys already cached (= position of the new token)


def make_decode_inputs(s: GdlaShape, B: int, cache_len, cap: int, seed: int,
                       std_w: float = 0.02) -> DecodeInputs:
    """Decode workload: x_new ~ N(0,1), weights ~ N(0, 0.02), cache rows ~ N(0,1).

    ``cache_len`` is an int (same for every sequence) or a list of B ints; cap must exceed
    every length so that the new token's row fits.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    x_new = _normal_bf16(gen, (B, s.d_model), 1.0)
    w = make_weights(gen, s, std_w)
    lens = [int(cache_len)] * B if isinstance(cache_len, int) else [int(v) for v in cache_len]
    assert len(lens) == B and max(lens) < cap
    cache = torch.zeros((B, cap, s.latent_row), dtype=torch.bfloat16)
    for b in range(B):
        if lens[b]:
            cache[b, : lens[b]] = _normal_bf16(gen, (lens[b], s.latent_row), 1.0)
    ones_q = torch.ones(s.q_rank, dtype=torch.bfloat16)
    ones_kv = torch.ones(s.kv_rank, dtype=torch.bfloat16)
    return DecodeInputs(s, x_new, w, ones_q, ones_kv, cache, torch.tensor(lens, dtype=torch.int32))


def sample_rows(T: int, window: int, n: int, seed: int) -> list:
    """Query rows checked at full size: first 32, last 16, 16 around t = W, rest uniform.

    Deterministic for (T, window, n, seed); returns sorted distinct row indices < T.
    """
    if T <= n:
        return list(range(T))
    rows = set(range(32))
    rows.update(range(T - 16, T))
    if window:
        rows.update(range(max(0, window - 8), min(T, window + 8)))
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed) + 1000)
    for r in torch.randint(0, T, (4 * n,), generator=gen).tolist():
        if len(rows) >= n:
            break
        rows.add(r)
    return sorted(rows)


# The five workloads (layer shapes as above; seeds and masks per workload).
WORKLOADS = {
    "prefill_b1_t256_causal": dict(kind="prefill", B=1, T=256, window=0, seed=0),
    "prefill_b2_t8192_swa2048": dict(kind="prefill", B=2, T=8192, window=2048, seed=1),
    "prefill_b1_t32768_causal": dict(kind="prefill", B=1, T=32768, window=0, seed=2),
    "prefill_b1_t262144_causal": dict(kind="prefill", B=1, T=262144, window=0, seed=3),
    "prefill_b1_t262144_swa2048": dict(kind="prefill", B=1, T=262144, window=2048, seed=3),
    "decode_b64_l32768_causal": dict(kind="decode", B=64, L=32768, cap=32769, window=0, seed=4),
    "decode_b64_l32768_swa2048": dict(kind="decode", B=64, L=32768, cap=32769, window=2048, seed=4),
}
