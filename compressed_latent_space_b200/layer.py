"""Convenience wrapper: one CCA / CCGQA layer whose parameters, workspace and caches are
torch CUDA tensors, driving the C ABI of libcca.  Holds memory only; every step of the
computation runs in the library's kernels."""
from __future__ import annotations

import torch

from . import (CCA_BF16, CCA_DEFAULT_FLAGS, CCA_F32, cca_backward, cca_backward_workspace_size,
               cca_cache_alloc, cca_decode_step,
               cca_decode_workspace_size, cca_prefill_forward, cca_prefill_workspace_size,
               make_config, make_weights)


class Cache:
    """A decode cache laid out by cca_cache_alloc inside one uint8 CUDA buffer, with torch
    views of its regions (k, v, conv_state, vshift_state, lengths)."""

    def __init__(self, layer: "CCALayer", batch: int, max_seq: int, stream=None):
        nbytes = cca_cache_alloc(layer.cfg, batch, max_seq)
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=layer.device)
        self.struct = cca_cache_alloc(layer.cfg, batch, max_seq, self.buf, stream)
        self.batch, self.max_seq = batch, max_seq
        base = self.buf.data_ptr()
        dt, es = layer.dtype, layer.esize

        def view(ptr, numel, dtype, esz, shape):
            off = ptr - base
            assert off % esz == 0
            return self.buf[off:off + numel * esz].view(dtype).view(*shape)

        c = layer.cfg
        dl = layer.dl
        hkv = layer.n_kv_heads_local
        self.k = view(self.struct.k, batch * hkv * max_seq * dl, layer.latent_dtype, es,
                      (batch, hkv, max_seq, dl))
        self.v = view(self.struct.v, batch * hkv * max_seq * dl, layer.latent_dtype, es,
                      (batch, hkv, max_seq, dl))
        kc1 = c.conv_kernel - 1
        if kc1 > 0:
            self.conv_state = view(self.struct.conv_state, batch * kc1 * (layer.n_q + layer.n_kv),
                                   torch.float32, 4, (batch, kc1, layer.n_q + layer.n_kv))
        else:
            self.conv_state = None
        half = layer.n_kv - layer.vshift_begin
        self.vshift_state = view(self.struct.vshift_state, batch * half, torch.float32, 4,
                                 (batch, half))
        self.lengths = view(self.struct.lengths, batch, torch.int32, 4, (batch,))


class CCALayer:
    def __init__(self, d_model, n_heads, n_kv_heads, compression, w_qkv, w_o, conv_seq, conv_chan,
                 conv_kernel=4, rope_base=10000.0, norm_eps=1e-6, flags=CCA_DEFAULT_FLAGS,
                 dtype="bf16", device="cuda", tp_size=1, tp_rank=0):
        """Global layer shape; with tp_size > 1 the weights are rank tp_rank's slices (see
        compressed_latent_space_b200.tp) and prefill / decode return its share of y."""
        self.dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        # latent q, k, v and the K/V cache: float16 in 16-bit layers, float32 otherwise
        self.latent_dtype = torch.float16 if dtype == "bf16" else torch.float32
        self.esize = 2 if dtype == "bf16" else 4
        self.device = torch.device(device)
        self.cfg = make_config(d_model, n_heads, n_kv_heads, compression, conv_kernel, 1, rope_base,
                               norm_eps, flags, CCA_BF16 if dtype == "bf16" else CCA_F32,
                               tp_size, tp_rank)
        tp = max(tp_size, 1)
        self.dl = d_model // n_heads // compression
        self.n_heads_local = n_heads // tp
        self.n_kv_heads_local = n_kv_heads // tp
        self.n_q = self.n_heads_local * self.dl
        self.n_kv = self.n_kv_heads_local * self.dl
        # first value channel of this rank taken from the previous token (the layer's split
        # at n_kv/2 of all key/value heads, in this rank's channel numbering)
        self.vshift_begin = min(max(n_kv_heads * self.dl // 2 - tp_rank * self.n_kv, 0), self.n_kv)
        self.w_qkv = w_qkv.to(self.device, self.dtype).contiguous()
        self.w_o = w_o.to(self.device, self.dtype).contiguous()
        # CCA_NO_CONV layers take no conv filters
        self.conv_seq = None if conv_seq is None else conv_seq.to(self.device, torch.float32).contiguous()
        self.conv_chan = None if conv_chan is None else conv_chan.to(self.device, torch.float32).contiguous()
        self.weights = make_weights(self.w_qkv, self.w_o, self.conv_seq, self.conv_chan)
        self._ws = None

    @classmethod
    def from_workload(cls, w, inputs, flags=None, device="cuda"):
        """flags None: the workload's own switches."""
        flags = w.flags if flags is None else flags
        no_conv = bool(flags & 16)
        return cls(w.d_model, w.n_heads, w.n_kv_heads, w.compression, inputs.w_qkv, inputs.w_o,
                   None if no_conv else inputs.conv_seq, None if no_conv else inputs.conv_chan,
                   conv_kernel=w.conv_kernel, rope_base=w.rope_base, flags=flags, dtype=w.dtype,
                   device=device)

    def workspace(self, nbytes: int) -> torch.Tensor:
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def new_cache(self, batch: int, max_seq: int, stream=None) -> Cache:
        return Cache(self, batch, max_seq, stream)

    def prefill(self, x: torch.Tensor, cache: Cache | None = None, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
        B, S, E = x.shape
        y = out if out is not None else torch.empty_like(x)
        ws = self.workspace(cca_prefill_workspace_size(self.cfg, B, S))
        cca_prefill_forward(self.cfg, self.weights, x, B, S, y,
                            cache.struct if cache is not None else None, ws, stream)
        return y

    def backward(self, x: torch.Tensor, dy: torch.Tensor, stream=None):
        """Gradients of sum(y * dy) for the prefill of x: (dx, dw_qkv, dw_o, dconv_seq,
        dconv_chan); weight gradients in float32."""
        B, S, E = x.shape
        dx = torch.empty_like(x)
        dw_qkv = torch.empty(self.w_qkv.shape, dtype=torch.float32, device=self.device)
        dw_o = torch.empty(self.w_o.shape, dtype=torch.float32, device=self.device)
        dconv_seq = torch.empty(self.conv_seq.shape, dtype=torch.float32, device=self.device)
        dconv_chan = torch.empty(self.conv_chan.shape, dtype=torch.float32, device=self.device)
        ws = self.workspace(cca_backward_workspace_size(self.cfg, B, S))
        cca_backward(self.cfg, self.weights, x, dy, B, S, dx, dw_qkv, dw_o, dconv_seq, dconv_chan,
                     ws, stream)
        return dx, dw_qkv, dw_o, dconv_seq, dconv_chan

    def decode(self, x: torch.Tensor, cache: Cache, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        y = out if out is not None else torch.empty_like(x)
        ws = self.workspace(cca_decode_workspace_size(self.cfg, cache.batch, cache.max_seq))
        cca_decode_step(self.cfg, self.weights, x, y, cache.struct, ws, stream)
        return y
