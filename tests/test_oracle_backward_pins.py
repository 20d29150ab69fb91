"""Pins of the backward oracle (oracle/cca_oracle_backward.py) to things other than itself.

1. Central finite differences of the forward oracle (already pinned by test_oracle_pins) for
   every input and parameter tensor, Richardson-extrapolated over two step sizes: along random
   directions (sum(grad * V) against the difference quotient of L = sum(y * dy) in direction V)
   and on single entries, for several switch settings, group sizes and conv widths.
2. The MHA reduction (C = 1, identity convs, only RoPE on) against torch autograd of
   scaled_dot_product_attention with the projections and RoPE as torch ops (a library
   routine's own backward).
3. Planted mistakes (the RoPE gradient rotated the wrong way, the key heads' norm gradient
   halved, the value-shift left out of the forward the backward recomputes, the sequence-conv
   taps reversed) each fail the finite-difference pin.
"""
import math

import numpy as np
import pytest
import torch

import oracle.cca_oracle as O
import oracle.cca_oracle_backward as OB
from oracle.cca_oracle import OracleConfig, OracleWeights


def _setup(cfg: OracleConfig, B=2, S=9, seed=0, conv_std=0.4):
    rng = np.random.default_rng(seed)
    E, nq, nkv, d = cfg.d_model, cfg.n_q, cfg.n_kv, cfg.dl
    w = OracleWeights(
        w_q=rng.normal(0, 0.3, (nq, E)), w_k=rng.normal(0, 0.3, (nkv, E)),
        w_v=rng.normal(0, 0.3, (nkv, E)), w_o=rng.normal(0, 0.3, (E, nq)),
        conv_seq=rng.normal(0, conv_std, (nq + nkv, cfg.conv_kernel)),
        conv_chan=rng.normal(0, conv_std, (cfg.n_heads + cfg.n_kv_heads, d, d, 1)))
    x = rng.normal(0, 1, (B, S, E))
    dy = rng.normal(0, 1, (B, S, E))
    return w, x, dy


def _loss(cfg, w, x, dy):
    return float(np.sum(O.prefill(cfg, w, x) * dy))


def _perturbed(w: OracleWeights, name, delta):
    kw = dict(w_q=w.w_q, w_k=w.w_k, w_v=w.w_v, w_o=w.w_o, conv_seq=w.conv_seq,
              conv_chan=w.conv_chan)
    if name == "w_qkv":
        nq, nkv = w.w_q.shape[0], w.w_k.shape[0]
        kw["w_q"] = w.w_q + delta[:nq]
        kw["w_k"] = w.w_k + delta[nq:nq + nkv]
        kw["w_v"] = w.w_v + delta[nq + nkv:]
    else:
        kw[name] = kw[name] + delta
    return OracleWeights(**kw)


def _grad_of(g: OB.OracleGrads, name):
    return dict(x=g.dx, w_qkv=g.dw_qkv, w_o=g.dw_o, conv_seq=g.dconv_seq,
                conv_chan=g.dconv_chan)[name]


def _shape_of(cfg, w, x, name):
    if name == "x":
        return x.shape
    if name == "w_qkv":
        return (cfg.n_q + 2 * cfg.n_kv, cfg.d_model)
    return getattr(w, name).shape


def _central(cfg, w, x, dy, name, V, eps):
    if name == "x":
        lp, lm = _loss(cfg, w, x + eps * V, dy), _loss(cfg, w, x - eps * V, dy)
    else:
        lp = _loss(cfg, _perturbed(w, name, eps * V), x, dy)
        lm = _loss(cfg, _perturbed(w, name, -eps * V), x, dy)
    return (lp - lm) / (2 * eps)


def _directional_check(cfg, w, x, dy, g, name, rng, eps=1e-4):
    """Richardson-extrapolated central difference (the eps^2 error term cancels; what is left
    is O(eps^4) plus rounding) against the analytic directional derivative."""
    V = rng.normal(0, 1, _shape_of(cfg, w, x, name))
    f1 = _central(cfg, w, x, dy, name, V, eps)
    f2 = _central(cfg, w, x, dy, name, V, eps / 2)
    fd = (4.0 * f2 - f1) / 3.0
    an = float(np.sum(_grad_of(g, name) * V))
    return fd, an


NAMES = ["x", "w_qkv", "w_o", "conv_seq", "conv_chan"]

CASES = [
    dict(d_model=16, n_heads=2, n_kv_heads=2, compression=2),                  # CCA, d~=4
    dict(d_model=32, n_heads=4, n_kv_heads=2, compression=2),                  # CCGQA G=2
    dict(d_model=32, n_heads=4, n_kv_heads=1, compression=2, conv_kernel=3),   # G=4, k=3
    dict(d_model=24, n_heads=2, n_kv_heads=1, compression=3, conv_kernel=1),   # d~=4, k=1
]


@pytest.mark.parametrize("flags", [15, 0, 14, 13, 11, 7])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_backward_matches_finite_differences(case, flags):
    kw = dict(CASES[case])
    cfg = OracleConfig(**kw, qk_mean=bool(flags & 1), value_shift=bool(flags & 2),
                       qk_norm=bool(flags & 4), rope=bool(flags & 8))
    w, x, dy = _setup(cfg, seed=case * 7 + flags)
    g = OB.backward(cfg, w, x, dy)
    rng = np.random.default_rng(100 + case)
    for name in NAMES:
        for _ in range(2):
            fd, an = _directional_check(cfg, w, x, dy, g, name, rng)
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, fd, an)


def test_backward_single_entries():
    """A handful of individual gradient entries by central differences (no direction mixing)."""
    cfg = OracleConfig(d_model=16, n_heads=2, n_kv_heads=1, compression=2, conv_kernel=3)
    w, x, dy = _setup(cfg, B=1, S=6, seed=3)
    g = OB.backward(cfg, w, x, dy)
    eps = 1e-4
    picks = [("x", (0, 4, 3)), ("x", (0, 0, 7)), ("w_qkv", (2, 5)), ("w_qkv", (9, 1)),
             ("w_qkv", (13, 0)), ("w_o", (3, 6)), ("conv_seq", (4, 0)), ("conv_seq", (10, 2)),
             ("conv_chan", (1, 2, 3, 0)), ("conv_chan", (2, 0, 1, 0))]
    for name, idx in picks:
        V = np.zeros(_shape_of(cfg, w, x, name))
        V[idx] = 1.0
        fd = (4.0 * _central(cfg, w, x, dy, name, V, eps / 2) - _central(cfg, w, x, dy, name, V, eps)) / 3.0
        an = _grad_of(g, name)[idx]
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, idx, fd, an)


def test_mha_reduction_matches_torch_autograd():
    """C = 1, identity convolutions, only RoPE: the gradients equal those torch autograd gives
    for textbook causal MHA (linear layers, rotate-half RoPE, scaled_dot_product_attention)."""
    E, H, S, B = 16, 2, 8, 2
    d = E // H
    cfg = OracleConfig(d_model=E, n_heads=H, n_kv_heads=H, compression=1, conv_kernel=2,
                       qk_mean=False, value_shift=False, qk_norm=False, rope=True)
    rng = np.random.default_rng(5)
    wq, wk, wv, wo = (rng.normal(0, 0.3, (E, E)) for _ in range(4))
    conv_seq = np.zeros((2 * E, 2))
    conv_seq[:, -1] = 1.0
    conv_chan = np.zeros((2 * H, d, d, 1))
    conv_chan[:, np.arange(d), np.arange(d), 0] = 1.0
    w = OracleWeights(w_q=wq, w_k=wk, w_v=wv, w_o=wo, conv_seq=conv_seq, conv_chan=conv_chan)
    x = rng.normal(0, 1, (B, S, E))
    dy = rng.normal(0, 1, (B, S, E))
    g = OB.backward(cfg, w, x, dy)

    T = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    xt, wqt, wkt, wvt, wot = T(x), T(wq), T(wk), T(wv), T(wo)
    half = d // 2
    theta = 10000.0 ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
    ang = torch.arange(S, dtype=torch.float64)[:, None] * theta[None, :]
    cos, sin = torch.cos(ang), torch.sin(ang)

    def rope(u):                                  # u [B, H, S, d]
        u1, u2 = u[..., :half], u[..., half:]
        return torch.cat([u1 * cos - u2 * sin, u1 * sin + u2 * cos], dim=-1)

    def heads(t):
        return t.reshape(B, S, H, d).transpose(1, 2)

    q = rope(heads(xt @ wqt.T))
    k = rope(heads(xt @ wkt.T))
    v = heads(xt @ wvt.T)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    y = o.transpose(1, 2).reshape(B, S, E) @ wot.T
    (y * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(g.dx, xt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(g.dw_qkv, torch.cat([wqt.grad, wkt.grad, wvt.grad]).numpy(),
                               rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(g.dw_o, wot.grad.numpy(), rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("mistake", ["rope_forward", "halved_key_norm_grad", "no_value_shift",
                                     "reversed_taps"])
def test_planted_mistakes_fail_the_pin(monkeypatch, mistake):
    cfg = OracleConfig(d_model=32, n_heads=4, n_kv_heads=2, compression=2, conv_kernel=3)
    w, x, dy = _setup(cfg, seed=11)
    if mistake == "rope_forward":                 # rotate the gradient the wrong way
        real = OB.rope_heads
        monkeypatch.setattr(OB, "rope_heads", lambda u, pos, *a: real(u, np.abs(pos), *a))
    elif mistake == "halved_key_norm_grad":       # the key heads' norm gradient halved
        real_norm = OB._norm_backward

        def patched(u, n, dn, n_heads, dl, eps):
            out = real_norm(u, n, dn, n_heads, dl, eps)
            return out if n_heads == cfg.n_heads else out * 0.5
        monkeypatch.setattr(OB, "_norm_backward", patched)
    elif mistake == "no_value_shift":             # the recomputed forward skips the shift
        monkeypatch.setattr(OB, "value_shift", lambda pv, prev=None: np.array(pv))
    elif mistake == "reversed_taps":
        w = OracleWeights(w_q=w.w_q, w_k=w.w_k, w_v=w.w_v, w_o=w.w_o,
                          conv_seq=w.conv_seq, conv_chan=w.conv_chan)
        real_bwd = OB.backward_sequence

        def patched_bwd(cfg_, w_, x_, dy_):
            wr = OracleWeights(w_q=w_.w_q, w_k=w_.w_k, w_v=w_.w_v, w_o=w_.w_o,
                               conv_seq=w_.conv_seq[:, ::-1].copy(), conv_chan=w_.conv_chan)
            return real_bwd(cfg_, wr, x_, dy_)
        monkeypatch.setattr(OB, "backward_sequence", patched_bwd)
    g = OB.backward(cfg, w, x, dy)
    rng = np.random.default_rng(1)
    worst = 0.0
    for name in NAMES:
        fd, an = _directional_check(cfg, w, x, dy, g, name, rng)
        worst = max(worst, abs(fd - an) / max(1.0, abs(fd)))
    assert worst > 1e-4, (mistake, worst)
