"""Context-parallel GDLA prefill: one long sequence split over the ranks of a process group.

The report trains 256K-token contexts by splitting each sequence over ranks and exchanging only
key/value information (paperglide.net summary, Figure 5 caption; section on the hierarchical
parallel layout): a sliding-window layer needs the trailing W tokens of the preceding shard (a
halo), a full-attention layer every preceding shard.  Here the exchanged rows are the 576-value
latent rows (RMSNorm'd c^KV | rotated k^R) from which every head's keys and values follow -
1152 bytes per token instead of per-head K/V.

Protocol for rank r holding tokens [start_r, start_r + T_r) of the sequence:
  1. all ranks learn every T_r (one small all-gather) and so their start positions;
  2. each rank computes the latent rows of its own tokens (`layer.latent`);
  3. exchange: full causal - all-gather of the latent rows (rank r keeps rows of ranks < r);
     window W - rank r sends its last W - 1 rows to rank r + 1 (point-to-point halo), or, when
     some shard is shorter than W - 1, an all-gather of every rank's last W - 1 rows;
  4. each rank runs its tokens after the received key prefix (`layer.prefill_context`).

`layer` needs `latent(x, pos_offset)`, `prefill_context(x, pos_offset, prefix_latent)` and
`window` (0 = full causal); GdlaLayer provides them on the GPU.  The collectives are those of
torch.distributed on the tensors' device (NCCL for CUDA tensors).

With fp8=True the rows cross the network as MXFP8 rows (the report's low-precision format,
paperglide.net summary, the low-precision paragraph and Figure 3: E4M3 values with one
power-of-two scale per 32; 608 bytes instead of 1152): each rank quantizes its rows before the
exchange (`layer.quantize_latent_fp8`) and the receiver dequantizes the prefix it gets
(`layer.dequantize_latent_fp8`); a rank's own rows stay bf16.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _lengths(T_local: int, device, group) -> list:
    t = torch.tensor([T_local], dtype=torch.int64, device=device)
    out = [torch.zeros_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(out, t, group=group)
    return [int(v.item()) for v in out]


def _all_gather_rows(rows: torch.Tensor, counts: list, group) -> list:
    """All-gather of per-rank row blocks of different lengths (padded to the longest)."""
    width = rows.shape[1]
    n = max(counts)
    buf = torch.zeros((n, width), dtype=rows.dtype, device=rows.device)
    buf[: rows.shape[0]] = rows
    out = [torch.empty_like(buf) for _ in counts]
    dist.all_gather(out, buf, group=group)
    return [o[:c] for o, c in zip(out, counts)]


def exchange_prefix(latent: torch.Tensor, lengths: list, rank: int, window: int, group=None):
    """The latent rows rank `rank` needs before its first token (None when it needs none)."""
    world = len(lengths)
    start = sum(lengths[:rank])
    if window <= 0:
        # full causal: every preceding token
        blocks = _all_gather_rows(latent, lengths, group)
        return torch.cat(blocks[:rank], 0) if rank > 0 and start > 0 else None
    need = min(window - 1, start)
    halo = window - 1
    if all(t >= halo for t in lengths[:-1]):
        # every shard but the last can serve the next one alone: one point-to-point halo.
        # P2POp takes the peer as a global rank, so the group's neighbours are mapped.
        def peer(r):
            return r if group is None else dist.get_global_rank(group, r)
        ops = []
        recv = None
        if rank + 1 < world and halo > 0:
            ops.append(dist.P2POp(dist.isend, latent[latent.shape[0] - halo:].contiguous(), peer(rank + 1), group))
        if rank > 0 and halo > 0:
            recv = torch.empty((halo, latent.shape[1]), dtype=latent.dtype, device=latent.device)
            ops.append(dist.P2POp(dist.irecv, recv, peer(rank - 1), group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
        return recv[halo - need:] if (recv is not None and need > 0) else None
    # short shards: everyone's last W - 1 rows, then the W - 1 rows just before this rank
    tails = [min(halo, t) for t in lengths]
    blocks = _all_gather_rows(latent[latent.shape[0] - tails[rank]:].contiguous(), tails, group)
    if need == 0:
        return None
    return torch.cat(blocks[:rank], 0)[-need:]


def cp_prefill(layer, x_local: torch.Tensor, group=None, fp8: bool = False) -> torch.Tensor:
    """y rows of this rank's tokens x_local [T_r, d] of a sequence split over the group."""
    rank = dist.get_rank(group)
    lengths = _lengths(x_local.shape[0], x_local.device, group)
    start = sum(lengths[:rank])
    latent = layer.latent(x_local, start)
    send = layer.quantize_latent_fp8(latent) if fp8 else latent
    prefix = exchange_prefix(send, lengths, rank, int(layer.window), group)
    if fp8 and prefix is not None:
        prefix = layer.dequantize_latent_fp8(prefix)
    return layer.prefill_context(x_local, start, prefix)
