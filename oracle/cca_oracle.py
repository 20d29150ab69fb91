"""Plain, slow CPU oracle for Compressed Convolutional Attention (CCA) and CCGQA.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links this
module; only the test suite, the smoke check and the benchmark's CPU-baseline leg do.
It shares no code with the CUDA path: no kernels, headers, tables or helpers.

Every step is written out in float64 numpy, in the order the pages give it, with no
tiling, no online softmax and no fusion.  Library primitives used as single steps:
``numpy`` matrix products and ``numpy.exp``.

Sources (titles of the pages that describe the method, arXiv 2510.04476):
  [gist]   "Compressed Convolutional Attention: Efficient Attention in a Compressed
           Latent Space" (gist.science explainer), §2 Methodology -- Core Mechanism,
           and "Extension: CCGQA".
  [gistde] the German edition of the same explainer, §2 Methodik.
  [abs]    the arXiv abstract as reprinted on mlsanity.com.
  [blog]   "Boosting Transformer Efficiency with Compressed Convolutional Attention"
           (edgentiq), "How Compressed Convolutional Attention Works".

Readings taken where the pages are silent or ambiguous (each is a switch in
``OracleConfig`` so a different reading costs one flag):
  * channel conv: grouped per head (groups = n_heads + n_kv_heads), mixing all
    latent channels of a head, kernel ``chan_conv_kernel`` along the sequence (1 =
    pointwise); applied after the causal depthwise sequence conv; no biases.
  * q-k-mean: add half of (pre-conv q + pre-conv k) to both post-conv q and k.  Under
    CCGQA a query head pairs with its group's key head, and a key head uses the mean of
    its group's pre-conv query heads.
  * value-shift: the upper half of the value channels of token t come from token t-1
    (zero at t = 0), which is "half of the heads" whenever n_kv_heads is even.
  * normalisation: RMS over each latent head vector, eps 1e-6, no learned weight, on q
    and k; then rotate-half RoPE over the full latent head width, base 10000, absolute
    positions from 0; softmax scale 1/sqrt(latent head dim).

Parity status: every step is pinned by tests (library routines, closed forms, brute
force, invariants).  The four readings above are "parity unpinned" as readings: the
pages print no formula or example that tells them apart from the alternatives.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class OracleConfig:
    """Shape and switches of one CCA / CCGQA attention layer.

    [gist] §2 Core Mechanism: queries, keys and values are projected from the residual
    width E to e~ = E/C; [gist] "Extension: CCGQA": key/value heads are shared by groups
    of query heads.  With H query heads of width hd = E/H, every latent head has width
    d~ = hd/C, so the query latent width is H*d~ = E/C and the key/value latent width is
    n_kv_heads*d~.
    """

    d_model: int
    n_heads: int
    n_kv_heads: int
    compression: int
    conv_kernel: int = 4
    chan_conv_kernel: int = 1
    rope_base: float = 10000.0
    qk_mean: bool = True
    value_shift: bool = True
    qk_norm: bool = True
    rope: bool = True
    norm_eps: float = 1e-6

    def __post_init__(self):
        assert self.d_model % self.n_heads == 0
        assert self.n_heads % self.n_kv_heads == 0
        assert (self.d_model // self.n_heads) % self.compression == 0
        assert self.conv_kernel >= 1 and self.chan_conv_kernel >= 1

    @property
    def head_dim(self) -> int:
        return self.d_model // self.n_heads

    @property
    def dl(self) -> int:
        """Latent head width d~ = (E/H)/C."""
        return self.head_dim // self.compression

    @property
    def group(self) -> int:
        return self.n_heads // self.n_kv_heads

    @property
    def n_q(self) -> int:
        return self.n_heads * self.dl

    @property
    def n_kv(self) -> int:
        return self.n_kv_heads * self.dl

    def with_(self, **kw) -> "OracleConfig":
        return replace(self, **kw)


@dataclass
class OracleWeights:
    """Float64 copies of the layer's parameters.

    w_q [n_q, E], w_k [n_kv, E], w_v [n_kv, E], w_o [E, n_q] (Linear layout [out, in]);
    conv_seq [n_q + n_kv, k] (one causal filter per latent q / k channel, tap k-1 on the
    current token); conv_chan [n_heads + n_kv_heads, d~, d~, k_c] (out, in, tap).
    """

    w_q: np.ndarray
    w_k: np.ndarray
    w_v: np.ndarray
    w_o: np.ndarray
    conv_seq: np.ndarray
    conv_chan: np.ndarray

    @staticmethod
    def from_arrays(cfg: OracleConfig, w_qkv, w_o, conv_seq, conv_chan) -> "OracleWeights":
        w_qkv = np.asarray(w_qkv, dtype=np.float64)
        nq, nkv = cfg.n_q, cfg.n_kv
        assert w_qkv.shape == (nq + 2 * nkv, cfg.d_model)
        return OracleWeights(
            w_q=w_qkv[:nq], w_k=w_qkv[nq:nq + nkv], w_v=w_qkv[nq + nkv:],
            w_o=np.asarray(w_o, dtype=np.float64),
            conv_seq=np.asarray(conv_seq, dtype=np.float64).reshape(nq + nkv, cfg.conv_kernel),
            conv_chan=np.asarray(conv_chan, dtype=np.float64).reshape(
                cfg.n_heads + cfg.n_kv_heads, cfg.dl, cfg.dl, cfg.chan_conv_kernel))


# ---------------------------------------------------------------------------------------
# Step 1: down-projection.  [gist] §2 Core Mechanism, "Down-Projection"; [abs]: the method
# "down-projects queries, keys, and values".
# ---------------------------------------------------------------------------------------
def down_project(x, w: OracleWeights):
    """x [S, E] -> (pq [S, n_q], pk [S, n_kv], pv [S, n_kv]) with p = x W^T."""
    x = np.asarray(x, dtype=np.float64)
    return x @ w.w_q.T, x @ w.w_k.T, x @ w.w_v.T


# ---------------------------------------------------------------------------------------
# Step 2: causal depthwise convolution along the sequence.  [gist] §2 "Convolutional
# Mixing": 1-D convolutions over the sequence dimension of latent q and k, like the causal
# convolutions of state-space models; [blog] "How CCA Works".
# ---------------------------------------------------------------------------------------
def seq_conv(p, conv_seq, history=None):
    """a[t, c] = sum_{j=0}^{k-1} conv_seq[c, j] * p[t - (k-1) + j, c].

    Rows before the first are taken from ``history`` (the k-1 rows that precede p, oldest
    first) or are zero.  Tap k-1 weights the current token.
    """
    p = np.asarray(p, dtype=np.float64)
    s, ch = p.shape
    k = conv_seq.shape[1]
    if history is None:
        history = np.zeros((k - 1, ch))
    padded = np.concatenate([np.asarray(history, dtype=np.float64).reshape(k - 1, ch), p], axis=0)
    out = np.zeros((s, ch))
    for j in range(k):
        # padded row (t + j) is sequence position t - (k-1) + j
        out += conv_seq[:, j][None, :] * padded[j:j + s, :]
    return out


# ---------------------------------------------------------------------------------------
# Step 3: per-head channel convolution.  [gist] §2 "Convolutional Mixing": convolutions
# "across both the sequence and channel dimensions"; read as a grouped convolution with
# one group per latent head that mixes the d~ channels of that head.
# ---------------------------------------------------------------------------------------
def channel_conv(a, conv_chan, n_groups, dl, history=None):
    """b[t, h, i] = sum_tau sum_j conv_chan[h, i, j, tau] * a[t - (k_c-1) + tau, h, j]."""
    a = np.asarray(a, dtype=np.float64)
    s = a.shape[0]
    kc = conv_chan.shape[3]
    a3 = a.reshape(s, n_groups, dl)
    if history is None:
        history = np.zeros((kc - 1, n_groups * dl))
    padded = np.concatenate(
        [np.asarray(history, dtype=np.float64).reshape(kc - 1, n_groups, dl), a3], axis=0)
    out = np.zeros((s, n_groups, dl))
    for tau in range(kc):
        window = padded[tau:tau + s]                       # [s, groups, j]
        out += np.einsum("gij,sgj->sgi", conv_chan[:, :, :, tau], window)
    return out.reshape(s, n_groups * dl)


# ---------------------------------------------------------------------------------------
# Step 4: q-k-mean.  [gist] §2 "Q-K-Mean": the mean of the pre- and post-convolution q and
# k is added back, a skip connection; [blog]: it shares information between queries and
# keys; [gistde] §2: it strengthens the diagonal of the attention matrix.
# ---------------------------------------------------------------------------------------
def qk_mean(bq, bk, pq, pk, cfg: OracleConfig):
    """q = bq + (pq + pk[group]) / 2;  k = bk + (mean of the group's pq + pk) / 2."""
    s = bq.shape[0]
    H, Hk, G, d = cfg.n_heads, cfg.n_kv_heads, cfg.group, cfg.dl
    pq3 = pq.reshape(s, H, d)
    pk3 = pk.reshape(s, Hk, d)
    pk_for_q = np.repeat(pk3, G, axis=1)                   # head h pairs with kv head h // G
    pq_group_mean = pq3.reshape(s, Hk, G, d).mean(axis=2)
    q = bq.reshape(s, H, d) + 0.5 * (pq3 + pk_for_q)
    k = bk.reshape(s, Hk, d) + 0.5 * (pq_group_mean + pk3)
    return q.reshape(s, H * d), k.reshape(s, Hk * d)


# ---------------------------------------------------------------------------------------
# Step 5: value-shift.  [gist] §2 "Value-Shift": values come from the current token and
# the previous token, so half of the heads do not see the present token (as in RWKV's
# token shift); [blog] "How CCA Works".
# ---------------------------------------------------------------------------------------
def value_shift(pv, prev_row=None):
    """v[t, c] = pv[t, c] for c < n_kv/2 and pv[t-1, c] for c >= n_kv/2.

    ``prev_row`` holds pv[-1, n_kv/2:] (the shifted half of the token before the first);
    zero when absent.
    """
    pv = np.asarray(pv, dtype=np.float64)
    s, nkv = pv.shape
    half = nkv // 2
    v = pv.copy()
    prev = np.zeros(nkv - half) if prev_row is None else np.asarray(prev_row, dtype=np.float64)
    shifted = np.concatenate([prev[None, :], pv[:-1, half:]], axis=0) if s > 0 else pv[:, half:]
    v[:, half:] = shifted
    return v


# ---------------------------------------------------------------------------------------
# Step 6: normalisation of q and k.  [gist] §2 "Q-K-Mean" names it only as "combined with
# normalization"; read as RMS normalisation of every latent head vector, no weight.
# ---------------------------------------------------------------------------------------
def rms_norm_heads(u, n_heads, dl, eps):
    s = u.shape[0]
    u3 = u.reshape(s, n_heads, dl)
    rms = np.sqrt(np.mean(u3 * u3, axis=2, keepdims=True) + eps)
    return (u3 / rms).reshape(s, n_heads * dl)


# ---------------------------------------------------------------------------------------
# Step 7: rotary position embedding on the latent q and k.  [gist] §2 "RoPE Integration":
# RoPE is applied directly to the compressed queries and keys, with no extra RoPE heads.
# Pairing is rotate-half: channel i rotates with channel i + d~/2 by angle t * base^(-2i/d~).
# ---------------------------------------------------------------------------------------
def rope_heads(u, positions, n_heads, dl, base):
    s = u.shape[0]
    half = dl // 2
    u3 = u.reshape(s, n_heads, dl)
    i = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * i / dl)                         # [half]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = u3[:, :, :half], u3[:, :, half:]
    out = np.concatenate([x1 * cos - x2 * sin, x1 * sin + x2 * cos], axis=2)
    return out.reshape(s, n_heads * dl)


# ---------------------------------------------------------------------------------------
# Step 8: causal softmax attention on latent-width heads.  [gistde] §2: Softmax(Q K^T) V is
# computed entirely in the compressed space; [gist] "Extension: CCGQA": query heads share
# key/value heads in contiguous groups.
# ---------------------------------------------------------------------------------------
def causal_attention(q, k, v, cfg: OracleConfig, q_positions=None, rows_per_block=256):
    """O[t, h] = sum_{s <= pos(t)} softmax_s(q[t,h] . k[s,g] / sqrt(d~)) v[s,g], g = h // G.

    ``q`` holds the rows whose absolute positions are ``q_positions`` (default 0..Sq-1);
    ``k`` and ``v`` hold positions 0..Sk-1.  Each score row is formed in full, reduced by
    its maximum, exponentiated and normalised.  Rows are processed ``rows_per_block`` at a
    time only to bound memory; no row's arithmetic depends on the blocking.
    """
    sq = q.shape[0]
    sk = k.shape[0]
    H, Hk, G, d = cfg.n_heads, cfg.n_kv_heads, cfg.group, cfg.dl
    if q_positions is None:
        q_positions = np.arange(sq)
    q_positions = np.asarray(q_positions)
    q3 = q.reshape(sq, H, d)
    k3 = k.reshape(sk, Hk, d)
    v3 = v.reshape(sk, Hk, d)
    scale = 1.0 / math.sqrt(d)
    out = np.zeros((sq, H, d))
    key_pos = np.arange(sk)
    for h in range(H):
        g = h // G
        for r0 in range(0, sq, rows_per_block):
            r1 = min(sq, r0 + rows_per_block)
            pos = q_positions[r0:r1]
            kmax = int(pos.max()) + 1
            scores = (q3[r0:r1, h, :] @ k3[:kmax, g, :].T) * scale    # [rows, kmax]
            visible = key_pos[None, :kmax] <= pos[:, None]
            scores = np.where(visible, scores, -np.inf)
            scores = scores - scores.max(axis=1, keepdims=True)
            e = np.exp(scores)
            probs = e / e.sum(axis=1, keepdims=True)
            out[r0:r1, h, :] = probs @ v3[:kmax, g, :]
    return out.reshape(sq, H * d)


# ---------------------------------------------------------------------------------------
# Step 9: up-projection back to the residual width.  [gist] §2 Core Mechanism: attention
# runs in the latent space and nothing is up-projected before it; the result returns to
# width E afterwards through one output matrix.
# ---------------------------------------------------------------------------------------
def up_project(o, w: OracleWeights):
    return np.asarray(o, dtype=np.float64) @ w.w_o.T


# ---------------------------------------------------------------------------------------
# Steps 2-7 for rows of one sequence.
# ---------------------------------------------------------------------------------------
def latent_qkv(cfg: OracleConfig, w: OracleWeights, pq, pk, pv, positions,
               conv_history=None, chan_history=None, vshift_prev=None):
    """From the projections of consecutive tokens to the q, k, v the attention consumes.

    ``conv_history``: the k-1 [pq|pk] rows before the first row (oldest first) or None
    (zeros).  ``chan_history``: the k_c-1 sequence-conv outputs before the first row.
    ``vshift_prev``: pv[-1, n_kv/2:] of the token before the first row.
    Returns (q, k, v, a) where ``a`` is the sequence-conv output (for the channel-conv state).
    """
    H, Hk, d = cfg.n_heads, cfg.n_kv_heads, cfg.dl
    pqk = np.concatenate([pq, pk], axis=1)
    a = seq_conv(pqk, w.conv_seq, conv_history)
    b = channel_conv(a, w.conv_chan, H + Hk, d, chan_history)
    bq, bk = b[:, :cfg.n_q], b[:, cfg.n_q:]
    if cfg.qk_mean:
        q, k = qk_mean(bq, bk, pq, pk, cfg)
    else:
        q, k = bq, bk
    v = value_shift(pv, vshift_prev) if cfg.value_shift else np.array(pv, dtype=np.float64)
    if cfg.qk_norm:
        q = rms_norm_heads(q, H, d, cfg.norm_eps)
        k = rms_norm_heads(k, Hk, d, cfg.norm_eps)
    if cfg.rope:
        q = rope_heads(q, positions, H, d, cfg.rope_base)
        k = rope_heads(k, positions, Hk, d, cfg.rope_base)
    return q, k, v, a


@dataclass
class OracleState:
    """Decode state of one sequence after L tokens.

    k_cache / v_cache [L, n_kv]: final keys (after conv, q-k-mean, norm, RoPE) and values
    (after value-shift); conv_state [k-1, n_q + n_kv]: the last k-1 pre-conv [pq|pk] rows
    (oldest first, zero before position 0); chan_state [k_c-1, n_q + n_kv]: the last k_c-1
    sequence-conv outputs; vshift_state [n_kv - n_kv/2]: pv[L-1, n_kv/2:].
    """

    k_cache: np.ndarray
    v_cache: np.ndarray
    conv_state: np.ndarray
    chan_state: np.ndarray
    vshift_state: np.ndarray

    @property
    def length(self) -> int:
        return self.k_cache.shape[0]


def _tail_rows(rows, n, width):
    """The last n rows of ``rows``, zero-padded at the front when fewer exist."""
    out = np.zeros((n, width))
    if n == 0:
        return out
    take = min(n, rows.shape[0])
    if take:
        out[n - take:] = rows[rows.shape[0] - take:]
    return out


def prefill_sequence(cfg: OracleConfig, w: OracleWeights, x, return_stages=False):
    """Full layer forward of one sequence x [S, E] from position 0.

    Returns y [S, E] and the decode state after the last token (and, on request, a dict of
    the intermediate stages).
    """
    x = np.asarray(x, dtype=np.float64)
    s = x.shape[0]
    pq, pk, pv = down_project(x, w)
    q, k, v, a = latent_qkv(cfg, w, pq, pk, pv, np.arange(s))
    o = causal_attention(q, k, v, cfg)
    y = up_project(o, w)
    width = cfg.n_q + cfg.n_kv
    half = cfg.n_kv // 2
    state = OracleState(
        k_cache=k, v_cache=v,
        conv_state=_tail_rows(np.concatenate([pq, pk], axis=1), cfg.conv_kernel - 1, width),
        chan_state=_tail_rows(a, cfg.chan_conv_kernel - 1, width),
        vshift_state=(pv[-1, half:].copy() if s > 0 else np.zeros(cfg.n_kv - half)))
    if return_stages:
        stages = dict(pq=pq, pk=pk, pv=pv, a=a, q=q, k=k, v=v, o=o)
        return y, state, stages
    return y, state


def prefill(cfg: OracleConfig, w: OracleWeights, x):
    """Batched forward x [B, S, E] -> y [B, S, E] (sequences are independent)."""
    x = np.asarray(x, dtype=np.float64)
    return np.stack([prefill_sequence(cfg, w, x[b])[0] for b in range(x.shape[0])])


def prefill_rows(cfg: OracleConfig, w: OracleWeights, x, rows):
    """Outputs y[rows] of one sequence x [S, E] without forming every query row.

    Keys and values need every token (they are causal functions of the whole prefix);
    queries, attention and the up-projection are evaluated only at ``rows``.
    """
    x = np.asarray(x, dtype=np.float64)
    s = x.shape[0]
    rows = np.asarray(rows)
    pq, pk, pv = down_project(x, w)
    q_all, k, v, _ = latent_qkv(cfg, w, pq, pk, pv, np.arange(s))
    o = causal_attention(q_all[rows], k, v, cfg, q_positions=rows)
    return up_project(o, w)


def decode_step(cfg: OracleConfig, w: OracleWeights, x_new, state: OracleState):
    """One new token x_new [E] at position L = state.length; returns (y [E], new state).

    The new token's projections are convolved with the stored pre-conv rows, its key and
    value are appended to the cache, and its query attends to positions 0..L.
    """
    x_new = np.asarray(x_new, dtype=np.float64).reshape(1, -1)
    L = state.length
    pq, pk, pv = down_project(x_new, w)
    q, k, v, a = latent_qkv(cfg, w, pq, pk, pv, np.array([L]),
                            conv_history=state.conv_state, chan_history=state.chan_state,
                            vshift_prev=state.vshift_state)
    k_cache = np.concatenate([state.k_cache, k], axis=0)
    v_cache = np.concatenate([state.v_cache, v], axis=0)
    o = causal_attention(q, k_cache, v_cache, cfg, q_positions=np.array([L]))
    y = up_project(o, w)[0]
    width = cfg.n_q + cfg.n_kv
    half = cfg.n_kv // 2
    new_conv = np.concatenate([state.conv_state, np.concatenate([pq, pk], axis=1)], axis=0)
    new_chan = np.concatenate([state.chan_state, a], axis=0)
    new_state = OracleState(
        k_cache=k_cache, v_cache=v_cache,
        conv_state=new_conv[new_conv.shape[0] - (cfg.conv_kernel - 1):] if cfg.conv_kernel > 1
        else np.zeros((0, width)),
        chan_state=new_chan[new_chan.shape[0] - (cfg.chan_conv_kernel - 1):]
        if cfg.chan_conv_kernel > 1 else np.zeros((0, width)),
        vshift_state=pv[0, half:].copy())
    return y, new_state


def decode_batch(cfg: OracleConfig, w: OracleWeights, x_new, k_cache, v_cache, lengths,
                 conv_state, vshift_state):
    """Batched decode step over caches laid out [B, n_kv_heads, max_seq, d~].

    x_new [B, E]; conv_state [B, k-1, n_q+n_kv]; vshift_state [B, n_kv - n_kv/2];
    lengths [B].  Returns (y [B, E], k_new [B, n_kv], v_new [B, n_kv], conv_state',
    vshift_state') where k_new / v_new are the rows appended at position lengths[b].
    Requires chan_conv_kernel == 1 (no channel-conv state in this layout).
    """
    assert cfg.chan_conv_kernel == 1
    B = x_new.shape[0]
    Hk, d = cfg.n_kv_heads, cfg.dl
    ys, ks, vs, cs, vss = [], [], [], [], []
    for b in range(B):
        L = int(lengths[b])
        kc = np.asarray(k_cache[b, :, :L, :], dtype=np.float64).transpose(1, 0, 2).reshape(L, Hk * d)
        vc = np.asarray(v_cache[b, :, :L, :], dtype=np.float64).transpose(1, 0, 2).reshape(L, Hk * d)
        st = OracleState(k_cache=kc, v_cache=vc,
                         conv_state=np.asarray(conv_state[b], dtype=np.float64),
                         chan_state=np.zeros((0, cfg.n_q + cfg.n_kv)),
                         vshift_state=np.asarray(vshift_state[b], dtype=np.float64))
        y, ns = decode_step(cfg, w, x_new[b], st)
        ys.append(y)
        ks.append(ns.k_cache[L])
        vs.append(ns.v_cache[L])
        cs.append(ns.conv_state)
        vss.append(ns.vshift_state)
    return np.stack(ys), np.stack(ks), np.stack(vs), np.stack(cs), np.stack(vss)


# ---------------------------------------------------------------------------------------
# Analytic counts the pages state in words.
# ---------------------------------------------------------------------------------------
def parameter_count(cfg: OracleConfig) -> int:
    """Projection parameters: W_q, W_k, W_v (down) and W_o (up); conv filters excluded."""
    return cfg.d_model * (cfg.n_q + 2 * cfg.n_kv) + cfg.n_q * cfg.d_model


def kv_cache_elements_per_token(cfg: OracleConfig) -> int:
    """Cached elements per token: one latent key and one latent value per kv head."""
    return 2 * cfg.n_kv
