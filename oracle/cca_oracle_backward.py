"""Plain, slow CPU oracle of the CCA / CCGQA layer's backward pass (gradients).

TEST INFRASTRUCTURE ONLY, like ``cca_oracle``: nothing in the product path imports it; the
tests, the smoke check and the benchmark's CPU leg may.  It shares no code with the CUDA path.

The layer is the one ``cca_oracle`` defines ([gist] §2 Core Mechanism: down-projection,
convolutional mixing, Q-K-Mean, Value-Shift, normalisation, RoPE, attention in the compressed
space, up-projection).  The pages measure its backward pass ([gist] §4 Experimental Results:
"Backward Pass: CCA is 1.3x faster than MHA") but print no formula for it; the gradients below
are the chain rule taken through the forward's steps in reverse order, each step written out
on its own in float64 with no fusion:

  9  y = o W_o^T                 do = dy W_o,            dW_o = dy^T o
  8  o = softmax(q k^T s) v      per head: dP = do v^T, dS = P * (dP - rowsum(P * dP)),
                                 dq = s dS k, dk += s dS^T q, dv += P^T do   (causal P)
  7  RoPE rotation R_t           d(before) = R_t^T d(after) = R_{-t} d(after)
  6  n = u / r, r = sqrt(mean(u^2) + eps)
                                 du = (dn - n * mean(dn * n)) / r
  5  value-shift                 dpv[t, c] = dv[t, c] (c < n_kv/2), dv[t+1, c] (c >= n_kv/2)
  4  q-k-mean                    db = du;  dpq_h += du_q,h / 2 + du_k,g / (2G);
                                           dpk_g += sum_h du_q,h / 2 + du_k,g / 2
  3  channel conv (pointwise)    da[t,h,:] = W_c[h]^T db[t,h,:];  dW_c[h] = sum_t db[t,h] a[t,h]^T
  2  causal sequence conv        dp[s,c] += sum_j w[c,j] da[s+k-1-j, c];
                                 dw[c,j] = sum_t da[t,c] p[t-(k-1)+j, c]
  1  p = x W^T                   dx = dp W,  dW = dp^T x

Pins (tests/test_oracle_backward_pins.py): central finite differences of the pinned oracle
forward for every input and parameter, in several switch settings and group sizes; the MHA
reduction against torch autograd of scaled_dot_product_attention; planted mistakes.
Requires chan_conv_kernel == 1 (the kernels' reading).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from .cca_oracle import (OracleConfig, OracleWeights, channel_conv, down_project, qk_mean,
                         rms_norm_heads, rope_heads, seq_conv, value_shift)


@dataclass
class OracleGrads:
    dx: np.ndarray          # [B, S, E]
    dw_qkv: np.ndarray      # [n_q + 2 n_kv, E]
    dw_o: np.ndarray        # [E, n_q]
    dconv_seq: np.ndarray   # [n_q + n_kv, k]
    dconv_chan: np.ndarray  # [H + Hkv, d~, d~, 1]


def _forward_saved(cfg: OracleConfig, w: OracleWeights, x):
    """The forward of one sequence with every intermediate the backward reads."""
    H, Hk, d = cfg.n_heads, cfg.n_kv_heads, cfg.dl
    s = x.shape[0]
    pq, pk, pv = down_project(x, w)
    pqk = np.concatenate([pq, pk], axis=1)
    a = seq_conv(pqk, w.conv_seq)
    b = channel_conv(a, w.conv_chan, H + Hk, d)
    bq, bk = b[:, :cfg.n_q], b[:, cfg.n_q:]
    uq, uk = qk_mean(bq, bk, pq, pk, cfg) if cfg.qk_mean else (bq, bk)
    v = value_shift(pv) if cfg.value_shift else pv.copy()
    nq = rms_norm_heads(uq, H, d, cfg.norm_eps) if cfg.qk_norm else uq
    nk = rms_norm_heads(uk, Hk, d, cfg.norm_eps) if cfg.qk_norm else uk
    pos = np.arange(s)
    q = rope_heads(nq, pos, H, d, cfg.rope_base) if cfg.rope else nq
    k = rope_heads(nk, pos, Hk, d, cfg.rope_base) if cfg.rope else nk
    return dict(pq=pq, pk=pk, pv=pv, pqk=pqk, a=a, uq=uq, uk=uk, nq=nq, nk=nk, q=q, k=k, v=v)


def _attention_backward(cfg: OracleConfig, q, k, v, do):
    """Causal softmax attention of every head, recomputed with its probabilities, and the
    gradients of q, k, v from do (the gradient of the attention output), all [S, width]."""
    H, Hk, G, d = cfg.n_heads, cfg.n_kv_heads, cfg.group, cfg.dl
    s = q.shape[0]
    scale = 1.0 / math.sqrt(d)
    mask = np.tril(np.ones((s, s), dtype=bool))
    o = np.zeros((s, H * d))
    dq = np.zeros((s, H * d))
    dk = np.zeros((s, Hk * d))
    dv = np.zeros((s, Hk * d))
    for h in range(H):
        g = h // G
        qh, kg, vg = q[:, h * d:(h + 1) * d], k[:, g * d:(g + 1) * d], v[:, g * d:(g + 1) * d]
        scores = np.where(mask, (qh @ kg.T) * scale, -np.inf)
        scores = scores - scores.max(axis=1, keepdims=True)
        e = np.exp(scores)
        p = e / e.sum(axis=1, keepdims=True)               # [S, S], zero above the diagonal
        o[:, h * d:(h + 1) * d] = p @ vg
        doh = do[:, h * d:(h + 1) * d]
        dp = doh @ vg.T
        ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
        dq[:, h * d:(h + 1) * d] = scale * (ds @ kg)
        dk[:, g * d:(g + 1) * d] += scale * (ds.T @ qh)
        dv[:, g * d:(g + 1) * d] += p.T @ doh
    return o, dq, dk, dv


def _norm_backward(u, n, dn, n_heads, dl, eps):
    """u -> n = u / sqrt(mean(u^2) + eps) per head vector: du from dn."""
    s = u.shape[0]
    u3, n3, dn3 = (t.reshape(s, n_heads, dl) for t in (u, n, dn))
    r = np.sqrt(np.mean(u3 * u3, axis=2, keepdims=True) + eps)
    du = (dn3 - n3 * np.mean(dn3 * n3, axis=2, keepdims=True)) / r
    return du.reshape(s, n_heads * dl)


def backward_sequence(cfg: OracleConfig, w: OracleWeights, x, dy):
    """Gradients of sum(y * dy) for one sequence x [S, E] (forward from position 0)."""
    assert cfg.chan_conv_kernel == 1, "the backward oracle covers the pointwise channel conv"
    H, Hk, G, d = cfg.n_heads, cfg.n_kv_heads, cfg.group, cfg.dl
    nq_w, nkv_w = cfg.n_q, cfg.n_kv
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    s = x.shape[0]
    f = _forward_saved(cfg, w, x)
    o, dq_r, dk_r, dv = _attention_backward(cfg, f["q"], f["k"], f["v"], dy @ w.w_o)
    # 9: up-projection
    dw_o = dy.T @ o
    # 7: RoPE (the transpose of a rotation by angle t*theta is the rotation by -t*theta)
    pos = np.arange(s)
    dnq = rope_heads(dq_r, -pos, H, d, cfg.rope_base) if cfg.rope else dq_r
    dnk = rope_heads(dk_r, -pos, Hk, d, cfg.rope_base) if cfg.rope else dk_r
    # 6: normalisation
    duq = _norm_backward(f["uq"], f["nq"], dnq, H, d, cfg.norm_eps) if cfg.qk_norm else dnq
    duk = _norm_backward(f["uk"], f["nk"], dnk, Hk, d, cfg.norm_eps) if cfg.qk_norm else dnk
    # 4: q-k-mean (the post-conv terms pass straight through; the skip reaches the projections)
    dpq = np.zeros((s, nq_w))
    dpk = np.zeros((s, nkv_w))
    if cfg.qk_mean:
        duq3, duk3 = duq.reshape(s, H, d), duk.reshape(s, Hk, d)
        dpq += (0.5 * duq3 + np.repeat(duk3, G, axis=1) / (2.0 * G)).reshape(s, nq_w)
        dpk += (0.5 * duq3.reshape(s, Hk, G, d).sum(axis=2) + 0.5 * duk3).reshape(s, nkv_w)
    db = np.concatenate([duq, duk], axis=1)                # [S, n_q + n_kv]
    # 3: channel conv, one d~ x d~ matrix per head (pointwise in time)
    wc = w.conv_chan[:, :, :, 0]                           # [heads, out i, in j]
    db3 = db.reshape(s, H + Hk, d)
    a3 = f["a"].reshape(s, H + Hk, d)
    da = np.einsum("hij,shi->shj", wc, db3).reshape(s, nq_w + nkv_w)
    dconv_chan = np.einsum("shi,shj->hij", db3, a3)[:, :, :, None]
    # 2: causal sequence conv (tap j of output t reads input t - (k-1) + j)
    kk = w.conv_seq.shape[1]
    p = f["pqk"]
    dp_conv = np.zeros_like(p)
    dconv_seq = np.zeros_like(w.conv_seq)
    for j in range(kk):
        lag = (kk - 1) - j                                 # output t reads input t - lag
        if lag < s:
            dp_conv[:s - lag] += w.conv_seq[:, j][None, :] * da[lag:]
            dconv_seq[:, j] = np.sum(da[lag:] * p[:s - lag], axis=0)
    dpq += dp_conv[:, :nq_w]
    dpk += dp_conv[:, nq_w:]
    # 5: value-shift
    dpv = dv.copy()
    if cfg.value_shift:
        half = nkv_w // 2
        dpv[:, half:] = 0.0
        dpv[:-1, half:] = dv[1:, half:]
    # 1: down-projection
    dp_all = np.concatenate([dpq, dpk, dpv], axis=1)       # [S, n_q + 2 n_kv]
    w_qkv = np.concatenate([w.w_q, w.w_k, w.w_v], axis=0)
    dx = dp_all @ w_qkv
    dw_qkv = dp_all.T @ x
    return dx, dw_qkv, dw_o, dconv_seq, dconv_chan


def backward(cfg: OracleConfig, w: OracleWeights, x, dy) -> OracleGrads:
    """Batched: x, dy [B, S, E]; weight gradients summed over the sequences."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    outs = [backward_sequence(cfg, w, x[b], dy[b]) for b in range(x.shape[0])]
    return OracleGrads(dx=np.stack([o[0] for o in outs]),
                       dw_qkv=sum(o[1] for o in outs), dw_o=sum(o[2] for o in outs),
                       dconv_seq=sum(o[3] for o in outs), dconv_chan=sum(o[4] for o in outs))
