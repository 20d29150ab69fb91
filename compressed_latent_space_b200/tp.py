"""Tensor parallelism by key/value group: one all-reduce per layer.

Every step of the layer before the up-projection is local to a key/value group: the
channel conv is per head, Q-K-Mean pairs a query head with its group's key head, and
attention reads only its group's keys and values (gist.science explainer, 5. Significance
and Implications, Scalability: compatible with tensor parallelism, with communication on the
compressed width).  So with R ranks, rank r holds query heads [r H/R, (r+1) H/R) and
key/value heads [r Hkv/R, (r+1) Hkv/R), computes them with the library's kernels (the
config's tp_size / tp_rank), and produces its share of the up-projection; the layer output is
the sum of the shares, one all-reduce of [tokens, E] over NCCL.

This module only cuts the weight tensors into the ranks' slices (a layout operation) and
issues the collective; all arithmetic of the layer runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from .layer import CCALayer


@dataclass(frozen=True)
class KVGroupSlice:
    """Index ranges of rank `rank`'s share of a layer's parameters."""
    q_rows: range          # rows of W_q (= query latent channels) and columns of W_o
    k_rows: range          # rows of W_k (= key latent channels)
    v_rows: range          # rows of W_v (= value latent channels)
    q_heads: range
    kv_heads: range


def kv_group_slice(n_heads: int, n_kv_heads: int, dl: int, tp_size: int, rank: int) -> KVGroupSlice:
    if n_kv_heads % tp_size:
        raise ValueError(f"n_kv_heads {n_kv_heads} is not a multiple of tp_size {tp_size}")
    if not 0 <= rank < tp_size:
        raise ValueError(f"rank {rank} outside [0, {tp_size})")
    hq, hk = n_heads // tp_size, n_kv_heads // tp_size
    return KVGroupSlice(q_rows=range(rank * hq * dl, (rank + 1) * hq * dl),
                        k_rows=range(rank * hk * dl, (rank + 1) * hk * dl),
                        v_rows=range(rank * hk * dl, (rank + 1) * hk * dl),
                        q_heads=range(rank * hq, (rank + 1) * hq),
                        kv_heads=range(rank * hk, (rank + 1) * hk))


def shard_weights(w_qkv, w_o, conv_seq, conv_chan, n_heads, n_kv_heads, dl, tp_size, rank):
    """Rank `rank`'s weights in the layout the library expects for tp_size > 1:
    w_qkv = [its W_q rows; its W_k rows; its W_v rows], w_o = its columns of W_o,
    conv_seq = [its query channels; its key channels], conv_chan = [its query heads; its key
    heads].  conv_seq / conv_chan may be None (CCA_NO_CONV layers)."""
    sl = kv_group_slice(n_heads, n_kv_heads, dl, tp_size, rank)
    n_q, n_kv = n_heads * dl, n_kv_heads * dl

    def rows(t, r, base=0):
        return t[base + r.start:base + r.stop]

    wq = rows(w_qkv, sl.q_rows)
    wk = rows(w_qkv, sl.k_rows, n_q)
    wv = rows(w_qkv, sl.v_rows, n_q + n_kv)
    local_qkv = torch.cat([wq, wk, wv], dim=0).contiguous()
    local_o = w_o[:, sl.q_rows.start:sl.q_rows.stop].contiguous()
    local_seq = None if conv_seq is None else torch.cat(
        [rows(conv_seq, sl.q_rows), rows(conv_seq, sl.k_rows, n_q)], dim=0).contiguous()
    local_chan = None if conv_chan is None else torch.cat(
        [conv_chan[sl.q_heads.start:sl.q_heads.stop],
         conv_chan[n_heads + sl.kv_heads.start:n_heads + sl.kv_heads.stop]], dim=0).contiguous()
    return local_qkv, local_o, local_seq, local_chan


def tp_all_reduce(y: torch.Tensor, tp_size: int, group=None) -> torch.Tensor:
    """Sums the ranks' shares of the layer output in place (the layer's one collective)."""
    if tp_size > 1:
        import torch.distributed as dist
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


class TPLayer:
    """One rank's share of a CCA / CCGQA layer split by key/value group.

    prefill() and decode() return the whole layer's output on every rank (the shares summed
    by one all-reduce over `group`); the rank's cache holds only its key/value heads."""

    def __init__(self, d_model, n_heads, n_kv_heads, compression, w_qkv, w_o, conv_seq, conv_chan,
                 tp_size, tp_rank, group=None, **kw):
        dl = d_model // n_heads // compression
        lw = shard_weights(w_qkv, w_o, conv_seq, conv_chan, n_heads, n_kv_heads, dl, tp_size,
                           tp_rank)
        self.tp_size, self.tp_rank, self.group = tp_size, tp_rank, group
        self.local = CCALayer(d_model, n_heads, n_kv_heads, compression, *lw, tp_size=tp_size,
                              tp_rank=tp_rank, **kw)

    @classmethod
    def from_workload(cls, w, inputs, tp_size, tp_rank, group=None, device="cuda"):
        no_conv = bool(w.flags & 16)
        return cls(w.d_model, w.n_heads, w.n_kv_heads, w.compression, inputs.w_qkv, inputs.w_o,
                   None if no_conv else inputs.conv_seq, None if no_conv else inputs.conv_chan,
                   tp_size, tp_rank, group, conv_kernel=w.conv_kernel, rope_base=w.rope_base,
                   flags=w.flags, dtype=w.dtype, device=device)

    def new_cache(self, batch, max_seq, stream=None):
        return self.local.new_cache(batch, max_seq, stream)

    def prefill_share(self, x, cache=None, out=None, stream=None):
        """This rank's share of y, before the all-reduce."""
        return self.local.prefill(x, cache=cache, out=out, stream=stream)

    def decode_share(self, x, cache, out=None, stream=None):
        return self.local.decode(x, cache, out=out, stream=stream)

    def prefill(self, x, cache=None, out=None, stream=None):
        return tp_all_reduce(self.prefill_share(x, cache, out, stream), self.tp_size, self.group)

    def decode(self, x, cache, out=None, stream=None):
        return tp_all_reduce(self.decode_share(x, cache, out, stream), self.tp_size, self.group)
