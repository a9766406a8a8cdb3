"""GdlaLayer: device-resident weights + caller-side buffers around the C ABI.

A convenience for Python users: it owns the layer's bf16 weights on one CUDA device, the
decode-ready absorbed weights, and a reusable workspace (allocated with torch, which is only
the memory/stream plumbing here), and forwards to the C entry points in ``binding``.
"""
from __future__ import annotations

import torch

from . import binding as gb
from .synth import GdlaShape, WEIGHT_NAMES


class GdlaLayer:
    def __init__(self, shape: GdlaShape, weights: dict, g_q=None, g_kv=None, device="cuda"):
        self.shape = shape
        self.window = shape.window        # 0 = full causal
        self.device = torch.device(device)
        self.w = {n: weights[n].to(self.device, torch.bfloat16).contiguous() for n in WEIGHT_NAMES}
        self.g_q = None if g_q is None else g_q.to(self.device, torch.bfloat16).contiguous()
        self.g_kv = None if g_kv is None else g_kv.to(self.device, torch.bfloat16).contiguous()
        self.cfg = gb.make_config(shape)
        self.cw = gb.make_weights(self.w, self.g_q, self.g_kv)
        self._ws = None
        self._absorbed = None
        self._absorbed_buf = None

    def workspace(self, B: int, T: int, mode: int) -> torch.Tensor:
        need = gb.gdla_workspace_size(self.cfg, B, T, mode)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def prefill(self, x: torch.Tensor, y: torch.Tensor | None = None,
                kv_cache_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        B, T, d = x.shape
        if y is None:
            y = torch.empty((B, T, d), dtype=torch.bfloat16, device=self.device)
        ws = self.workspace(B, T, gb.GDLA_MODE_PREFILL)
        cap = 0 if kv_cache_out is None else kv_cache_out.shape[1]
        gb.gdla_prefill_fwd(self.cfg, self.cw, x, y, ws, kv_cache_out, cap, stream)
        return y

    def prefill_packed(self, x: torch.Tensor, cu_seqlens: torch.Tensor, y: torch.Tensor | None = None,
                       kv_latent_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Independent documents packed row-wise in x [total, d]; cu_seqlens int32 [docs + 1]."""
        total, d = x.shape
        if y is None:
            y = torch.empty((total, d), dtype=torch.bfloat16, device=self.device)
        ws = self.workspace(1, total, gb.GDLA_MODE_VARLEN)
        gb.gdla_prefill_varlen_fwd(self.cfg, self.cw, x, cu_seqlens, y, ws, kv_latent_out, stream)
        return y

    def prefill_host(self, x_host: torch.Tensor, y_host: torch.Tensor | None = None, n_pieces: int = 8,
                     stream=None) -> torch.Tensor:
        """x_host [B, T, d] bf16 on the host (pinned for overlapped copies) -> y_host [B, T, d];
        returns once the work is enqueued: synchronise `stream` before reading y_host."""
        B, T, d = x_host.shape
        if y_host is None:
            y_host = torch.empty((B, T, d), dtype=torch.bfloat16, pin_memory=True)
        ws = self.workspace(B, T, gb.GDLA_MODE_HOST)
        gb.gdla_prefill_host_fwd(self.cfg, self.cw, x_host, y_host, ws, n_pieces, stream)
        return y_host

    def latent(self, x: torch.Tensor, pos_offset: int = 0, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        """Latent rows [T, kv_rank + d_rope] of tokens x [T, d] at positions pos_offset + t."""
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.cfg.kv_rank + self.cfg.d_rope), dtype=torch.bfloat16,
                              device=self.device)
        ws = self.workspace(1, T, gb.GDLA_MODE_PREFILL)
        gb.gdla_latent_fwd(self.cfg, self.cw, x, pos_offset, out, ws, stream)
        return out

    def prefill_context(self, x: torch.Tensor, pos_offset: int, prefix_latent: torch.Tensor | None,
                        y: torch.Tensor | None = None, latent_out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
        """Tokens x [T, d] at positions pos_offset + t, after the key prefix prefix_latent
        [n_prefix, kv_rank + d_rope] (the latent rows of the n_prefix tokens just before)."""
        T, d = x.shape
        if y is None:
            y = torch.empty((T, d), dtype=torch.bfloat16, device=self.device)
        n_prefix = 0 if prefix_latent is None else prefix_latent.shape[0]
        ws = self.workspace(1, T + n_prefix, gb.GDLA_MODE_CONTEXT)
        gb.gdla_prefill_context_fwd(self.cfg, self.cw, x, pos_offset, prefix_latent, y, ws,
                                    latent_out, stream)
        return y

    def absorbed(self, stream=None) -> gb.gdla_absorbed_t:
        if self._absorbed is None:
            n = gb.gdla_absorbed_size(self.cfg)
            self._absorbed_buf = torch.empty(n, dtype=torch.uint8, device=self.device)
            self._absorbed = gb.gdla_absorb_weights(self.cfg, self.cw, self._absorbed_buf, stream)
        return self._absorbed

    def decode(self, x_new: torch.Tensor, kv_cache: torch.Tensor, cache_len: torch.Tensor,
               y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        B, d = x_new.shape
        if y is None:
            y = torch.empty((B, d), dtype=torch.bfloat16, device=self.device)
        ws = self.workspace(B, kv_cache.shape[1], gb.GDLA_MODE_DECODE)
        gb.gdla_decode_fwd(self.cfg, self.absorbed(stream), x_new, kv_cache, cache_len, y, ws, stream)
        return y

    def decode_multi(self, x_new: torch.Tensor, kv_cache: torch.Tensor, cache_len: torch.Tensor,
                     y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """x_new [n_seq, q_len, d]: q_len consecutive new tokens per sequence in one call."""
        n_seq, q_len, d = x_new.shape
        if y is None:
            y = torch.empty((n_seq, q_len, d), dtype=torch.bfloat16, device=self.device)
        ws = self.workspace(n_seq * q_len, kv_cache.shape[1], gb.GDLA_MODE_DECODE)
        gb.gdla_decode_multi_fwd(self.cfg, self.absorbed(stream), x_new, kv_cache, cache_len, y, ws,
                                 stream)
        return y

    def decode_fp8(self, x_new: torch.Tensor, kv_cache8: torch.Tensor, cache_len: torch.Tensor,
                   y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Decode over an MXFP8 latent cache [n_seq, cap, 608] (uint8); x_new [n_seq, d] or
        [n_seq, q_len, d]."""
        if y is None:
            y = torch.empty(x_new.shape, dtype=torch.bfloat16, device=self.device)
        rows = x_new.shape[0] * (x_new.shape[1] if x_new.dim() == 3 else 1)
        ws = self.workspace(rows, kv_cache8.shape[1], gb.GDLA_MODE_DECODE)
        gb.gdla_decode_fp8_fwd(self.cfg, self.absorbed(stream), x_new, kv_cache8, cache_len, y, ws, stream)
        return y

    def quantize_latent_fp8(self, latent: torch.Tensor, stream=None) -> torch.Tensor:
        """bf16 latent rows [..., 576] -> MXFP8 rows [..., 608] (uint8)."""
        out = torch.empty(latent.shape[:-1] + (gb.FP8_ROW_BYTES,), dtype=torch.uint8, device=latent.device)
        gb.gdla_quantize_latent_fp8(self.cfg, latent, out, stream)
        return out

    def dequantize_latent_fp8(self, stored: torch.Tensor, stream=None) -> torch.Tensor:
        """MXFP8 rows [..., 608] (uint8) -> bf16 latent rows [..., 576]."""
        out = torch.empty(stored.shape[:-1] + (self.cfg.kv_rank + self.cfg.d_rope,), dtype=torch.bfloat16,
                          device=stored.device)
        gb.gdla_dequantize_latent_fp8(self.cfg, stored, out, stream)
        return out
