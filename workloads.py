"""Seeded synthetic inputs for the CCA / CCGQA layer.

This module holds shapes and random draws only: none of the method's arithmetic.  Both
the CUDA path's tests/benchmark and the CPU oracle take their inputs from here.

Recipe (every workload): ``torch.Generator('cpu').manual_seed(seed)`` draws, in this
order, x, W_q, W_k, W_v, W_o, conv_seq, conv_chan, and for the decode workload then the
key cache, value cache, conv state, value-shift state and the new tokens.  x and the
cache contents are N(0, 1); every weight (projections and conv filters) is N(0, 0.02^2)
unless a test overrides the conv scale.  x and the projection weights are rounded to the
workload's dtype, the K/V cache to its latent type (float16 for bf16 workloads), conv
filters and the conv / value-shift state stay float32; the oracle receives exactly these
values.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

WEIGHT_STD = 0.02


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq: int                 # prefill length, or cached context for decode
    d_model: int
    n_heads: int
    n_kv_heads: int
    compression: int
    conv_kernel: int = 4
    chan_conv_kernel: int = 1
    rope_base: float = 10000.0
    dtype: str = "bf16"      # "f32" or "bf16"
    decode: bool = False
    description: str = ""
    flags: int = 15          # CCA_* switches of the layer (16 = CCA_NO_CONV: identity convs)

    @property
    def head_dim(self) -> int:
        return self.d_model // self.n_heads

    @property
    def dl(self) -> int:
        return self.head_dim // self.compression

    @property
    def n_q(self) -> int:
        return self.n_heads * self.dl

    @property
    def n_kv(self) -> int:
        return self.n_kv_heads * self.dl

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def latent_dtype(self):
        """Storage type of the latent q, k, v and the K/V cache (float16 in 16-bit workloads)."""
        return torch.float32 if self.dtype == "f32" else torch.float16

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    w.name: w for w in [
        Workload("cca_tiny_fp32", 1, 128, 256, 4, 4, 4, dtype="f32",
                 description="CCA tiny fp32: B=1 S=128 E=256 H=4 Hkv=4 C=4 (d~=16)"),
        Workload("cca_prefill_4k", 4, 4096, 2048, 16, 16, 4,
                 description="CCA bf16 prefill: B=4 S=4096 E=2048 H=16 Hkv=16 C=4 (d~=32)"),
        Workload("ccgqa_prefill_16k", 2, 16384, 2048, 16, 4, 2,
                 description="CCGQA bf16 long prefill: B=2 S=16384 E=2048 H=16 Hkv=4 C=2 (d~=64)"),
        Workload("ccgqa_prefill_32k", 1, 32768, 4096, 32, 8, 4,
                 description="CCGQA bf16 large prefill: B=1 S=32768 E=4096 H=32 Hkv=8 C=4 (d~=32)"),
        Workload("ccgqa_decode_8k", 64, 8192, 2048, 16, 4, 4, decode=True,
                 description="CCGQA bf16 decode: B=64, 8192 cached tokens, E=2048 H=16 Hkv=4 C=4 (d~=32)"),
    ]
}

# The systems the pages compare CCA / CCGQA prefill against at 16k tokens, on the same
# d_model, heads and batch as ccgqa_prefill_16k: multi-head attention and grouped-query
# attention with 8 key/value heads (GQA-8), head width 128 (C = 1), RoPE only, no convs.
BASELINES = {
    w.name: w for w in [
        Workload("mha_prefill_16k", 2, 16384, 2048, 16, 16, 1, flags=8 | 16,
                 description="MHA bf16 prefill baseline: B=2 S=16384 E=2048 H=16 (hd=128), RoPE"),
        Workload("gqa8_prefill_16k", 2, 16384, 2048, 16, 8, 1, flags=8 | 16,
                 description="GQA-8 bf16 prefill baseline: B=2 S=16384 E=2048 H=16 Hkv=8 (hd=128), RoPE"),
    ]
}


@dataclass
class Inputs:
    """Host tensors (already rounded to the workload dtype) for one workload."""
    x: torch.Tensor                 # [B, S, E] prefill, or [B, E] new tokens for decode
    w_qkv: torch.Tensor             # [n_q + 2 n_kv, E]
    w_o: torch.Tensor               # [E, n_q]
    conv_seq: torch.Tensor          # [n_q + n_kv, k]          float32
    conv_chan: torch.Tensor         # [H + Hkv, d~, d~, k_c]    float32
    k_cache: torch.Tensor | None = None       # [B, Hkv, ctx, d~]
    v_cache: torch.Tensor | None = None       # [B, Hkv, ctx, d~]
    conv_state: torch.Tensor | None = None    # [B, k-1, n_q + n_kv] float32
    vshift_state: torch.Tensor | None = None  # [B, n_kv - n_kv/2] float32
    lengths: torch.Tensor | None = None       # [B] int32
    extra: dict = field(default_factory=dict)


def make_inputs(w: Workload, seed: int = 0, conv_std: float = WEIGHT_STD,
                identity_conv: bool = False, lengths=None) -> Inputs:
    """Draw one workload's inputs in the fixed order of the module docstring.

    ``conv_std`` lets a test give the conv filters O(1) weight so that the conv branch is
    visible next to the q-k-mean skip; ``identity_conv`` adds 1 to the current-token tap
    of every sequence filter and to the diagonal of every channel filter.  ``lengths``
    (decode only) overrides the per-sequence cached length (default: all equal to seq).
    """
    g = torch.Generator("cpu").manual_seed(seed)
    dt = w.torch_dtype
    E, nq, nkv, d = w.d_model, w.n_q, w.n_kv, w.dl

    def randn(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, dtype=torch.float32) * std)

    if not w.decode:
        x = randn(w.batch, w.seq, E).to(dt)
    w_q = randn(nq, E, std=WEIGHT_STD)
    w_k = randn(nkv, E, std=WEIGHT_STD)
    w_v = randn(nkv, E, std=WEIGHT_STD)
    w_o = randn(E, nq, std=WEIGHT_STD).to(dt)
    conv_seq = randn(nq + nkv, w.conv_kernel, std=conv_std)
    conv_chan = randn(w.n_heads + w.n_kv_heads, d, d, w.chan_conv_kernel, std=conv_std)
    if identity_conv:
        conv_seq[:, -1] += 1.0
        idx = torch.arange(d)
        conv_chan[:, idx, idx, -1] += 1.0
    w_qkv = torch.cat([w_q, w_k, w_v], dim=0).to(dt)
    inp = Inputs(x=None, w_qkv=w_qkv, w_o=w_o, conv_seq=conv_seq.contiguous(),
                 conv_chan=conv_chan.contiguous())
    if not w.decode:
        inp.x = x
        return inp
    B, ctx = w.batch, w.seq
    inp.k_cache = randn(B, w.n_kv_heads, ctx, d).to(w.latent_dtype)
    inp.v_cache = randn(B, w.n_kv_heads, ctx, d).to(w.latent_dtype)
    inp.conv_state = randn(B, w.conv_kernel - 1, nq + nkv)          # float32 state
    inp.vshift_state = randn(B, nkv - nkv // 2)
    inp.x = randn(B, E).to(dt)
    if lengths is None:
        inp.lengths = torch.full((B,), ctx, dtype=torch.int32)
    else:
        inp.lengths = torch.as_tensor(lengths, dtype=torch.int32)
    return inp

