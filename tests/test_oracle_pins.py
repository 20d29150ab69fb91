"""Pins of the CPU oracle to things other than itself.

Every step of the oracle is checked against a library routine (torch conv1d, torch
scaled-dot-product attention, torch rms_norm), a closed form (hand-derived fixtures in
tests/golden/hand_examples.json, complex-number RoPE), brute force, or an invariant the
method fixes (reduction to causal MHA, CCGQA as CCA with repeated key/value heads,
causality, decode == prefill).  A final group plants plausible mistakes in a copy of the
oracle and checks that some pin catches each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.cca_oracle as O
from oracle.cca_oracle import OracleConfig, OracleWeights

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def rand_weights(cfg: OracleConfig, rng, conv_std=0.3, proj_std=0.2):
    nq, nkv, E = cfg.n_q, cfg.n_kv, cfg.d_model
    return OracleWeights(
        w_q=rng.normal(0, proj_std, (nq, E)), w_k=rng.normal(0, proj_std, (nkv, E)),
        w_v=rng.normal(0, proj_std, (nkv, E)), w_o=rng.normal(0, proj_std, (E, nq)),
        conv_seq=rng.normal(0, conv_std, (nq + nkv, cfg.conv_kernel)),
        conv_chan=rng.normal(0, conv_std, (cfg.n_heads + cfg.n_kv_heads, cfg.dl, cfg.dl,
                                           cfg.chan_conv_kernel)))


def identity_convs(cfg: OracleConfig, w: OracleWeights):
    w.conv_seq = np.zeros_like(w.conv_seq)
    w.conv_seq[:, -1] = 1.0
    w.conv_chan = np.zeros_like(w.conv_chan)
    for g in range(w.conv_chan.shape[0]):
        w.conv_chan[g, :, :, -1] = np.eye(cfg.dl)
    return w


CFG_SMALL = OracleConfig(d_model=64, n_heads=4, n_kv_heads=2, compression=2)    # d~ = 8


# ------------------------------------------------------------------ hand-derived fixtures
def test_golden_seq_conv_taps():
    ex = GOLDEN["seq_conv_taps"]
    p = np.array(ex["p"], dtype=np.float64)[:, None]
    w = np.array(ex["weights"], dtype=np.float64)[None, :]
    got = O.seq_conv(p, w)[:, 0]
    np.testing.assert_allclose(got, ex["expected"], rtol=0, atol=1e-12)


def test_golden_qk_mean_group():
    ex = GOLDEN["qk_mean_group"]
    cfg = OracleConfig(d_model=ex["n_heads"], n_heads=ex["n_heads"], n_kv_heads=ex["n_kv_heads"],
                       compression=1)
    q, k = O.qk_mean(np.array(ex["bq"], float), np.array(ex["bk"], float),
                     np.array(ex["pq"], float), np.array(ex["pk"], float), cfg)
    np.testing.assert_allclose(q, ex["expected_q"], atol=1e-12)
    np.testing.assert_allclose(k, ex["expected_k"], atol=1e-12)


def test_golden_value_shift():
    ex = GOLDEN["value_shift_rows"]
    np.testing.assert_allclose(O.value_shift(np.array(ex["pv"], float)), ex["expected"], atol=0)


def test_golden_rms_norm():
    ex = GOLDEN["rms_norm_3_4"]
    got = O.rms_norm_heads(np.array([ex["u"]], float), 1, 2, ex["eps"])[0]
    np.testing.assert_allclose(got, ex["expected"], rtol=1e-14)


def test_golden_rope():
    ex = GOLDEN["rope_d4"]
    u = np.tile(np.array(ex["u"], float), (len(ex["positions"]), 1))
    got = O.rope_heads(u, np.array(ex["positions"]), 1, ex["dl"], ex["base"])
    np.testing.assert_allclose(got, ex["expected"], rtol=0, atol=1e-14)


def test_golden_attention():
    ex = GOLDEN["attention_quarter_three_quarters"]
    cfg = OracleConfig(d_model=2, n_heads=1, n_kv_heads=1, compression=1)
    got = O.causal_attention(np.array(ex["q"]), np.array(ex["k"]), np.array(ex["v"]), cfg)
    np.testing.assert_allclose(got, ex["expected"], atol=1e-12)


# ------------------------------------------------------------------ library routines
@pytest.mark.parametrize("k", [1, 2, 4])
def test_seq_conv_matches_torch_conv1d(k):
    rng = np.random.default_rng(1)
    s, ch = 37, 12
    p = rng.normal(size=(s, ch))
    w = rng.normal(size=(ch, k))
    ref = torch.nn.functional.conv1d(torch.tensor(p.T[None]), torch.tensor(w[:, None, :]),
                                     padding=k - 1, groups=ch)[0, :, :s].numpy().T
    np.testing.assert_allclose(O.seq_conv(p, w), ref, rtol=1e-12, atol=1e-12)


def test_seq_conv_history_continues_sequence():
    rng = np.random.default_rng(2)
    p = rng.normal(size=(20, 6))
    w = rng.normal(size=(6, 4))
    full = O.seq_conv(p, w)
    tail = O.seq_conv(p[12:], w, history=p[9:12])
    np.testing.assert_allclose(tail, full[12:], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("kc", [1, 3])
def test_channel_conv_matches_grouped_conv1d(kc):
    rng = np.random.default_rng(3)
    s, groups, d = 29, 5, 8
    a = rng.normal(size=(s, groups * d))
    w = rng.normal(size=(groups, d, d, kc))
    ref = torch.nn.functional.conv1d(torch.tensor(a.T[None]),
                                     torch.tensor(w.reshape(groups * d, d, kc)),
                                     padding=kc - 1, groups=groups)[0, :, :s].numpy().T
    np.testing.assert_allclose(O.channel_conv(a, w, groups, d), ref, rtol=1e-12, atol=1e-12)


def test_channel_conv_identity():
    rng = np.random.default_rng(4)
    a = rng.normal(size=(9, 3 * 4))
    w = np.zeros((3, 4, 4, 1))
    w[:, :, :, 0] = np.eye(4)
    np.testing.assert_allclose(O.channel_conv(a, w, 3, 4), a, atol=0)


def test_rms_norm_matches_torch():
    rng = np.random.default_rng(5)
    u = rng.normal(size=(11, 3 * 16)) * 3.0
    ref = torch.nn.functional.rms_norm(torch.tensor(u.reshape(11, 3, 16)), (16,), eps=1e-6)
    np.testing.assert_allclose(O.rms_norm_heads(u, 3, 16, 1e-6), ref.reshape(11, 48).numpy(),
                               rtol=1e-12, atol=1e-12)


def rope_complex(u, positions, n_heads, dl, base):
    """RoPE written as multiplication of complex pairs z_i = u_i + j u_{i+d/2} by
    exp(j t base^(-2i/d)) -- an independent formulation of the rotation."""
    s = u.shape[0]
    half = dl // 2
    u3 = u.reshape(s, n_heads, dl)
    z = u3[:, :, :half] + 1j * u3[:, :, half:]
    freqs = np.array([base ** (-2.0 * i / dl) for i in range(half)])
    rot = np.exp(1j * np.outer(positions, freqs))[:, None, :]
    zr = z * rot
    return np.concatenate([zr.real, zr.imag], axis=2).reshape(s, n_heads * dl)


def test_rope_matches_complex_rotation_and_properties():
    rng = np.random.default_rng(6)
    s, H, d = 23, 3, 16
    u = rng.normal(size=(s, H * d))
    pos = np.arange(100, 100 + s)
    got = O.rope_heads(u, pos, H, d, 10000.0)
    np.testing.assert_allclose(got, rope_complex(u, pos, H, d, 10000.0), rtol=1e-12, atol=1e-12)
    # position 0 is the identity; norms are preserved
    np.testing.assert_allclose(O.rope_heads(u, np.zeros(s), H, d, 10000.0), u, atol=0)
    np.testing.assert_allclose(np.linalg.norm(got.reshape(s, H, d), axis=2),
                               np.linalg.norm(u.reshape(s, H, d), axis=2), rtol=1e-12)
    # relative property: shifting every position by p0 leaves every q.k unchanged
    q = rng.normal(size=(s, d))
    k = rng.normal(size=(s, d))
    t = np.arange(s)
    sc0 = O.rope_heads(q, t, 1, d, 1e4) @ O.rope_heads(k, t, 1, d, 1e4).T
    sc1 = O.rope_heads(q, t + 777, 1, d, 1e4) @ O.rope_heads(k, t + 777, 1, d, 1e4).T
    np.testing.assert_allclose(sc0, sc1, rtol=1e-9, atol=1e-9)


def test_rms_norm_commutes_with_rope():
    rng = np.random.default_rng(7)
    u = rng.normal(size=(10, 2 * 8)) * 5
    pos = np.arange(10) * 3
    a = O.rope_heads(O.rms_norm_heads(u, 2, 8, 1e-6), pos, 2, 8, 1e4)
    b = O.rms_norm_heads(O.rope_heads(u, pos, 2, 8, 1e4), 2, 8, 1e-6)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("H,Hk", [(4, 4), (4, 2), (6, 1)])
def test_attention_matches_torch_sdpa(H, Hk):
    rng = np.random.default_rng(8)
    cfg = OracleConfig(d_model=H * 8, n_heads=H, n_kv_heads=Hk, compression=1)
    s, d = 45, cfg.dl
    q = rng.normal(size=(s, H * d)) * 2
    k = rng.normal(size=(s, Hk * d)) * 2
    v = rng.normal(size=(s, Hk * d))
    G = H // Hk
    qt = torch.tensor(q.reshape(s, H, d)).transpose(0, 1)
    kt = torch.tensor(k.reshape(s, Hk, d)).transpose(0, 1).repeat_interleave(G, dim=0)
    vt = torch.tensor(v.reshape(s, Hk, d)).transpose(0, 1).repeat_interleave(G, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    ref = ref.transpose(0, 1).reshape(s, H * d).numpy()
    got = O.causal_attention(q, k, v, cfg, rows_per_block=7)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_attention_brute_force_and_closed_forms():
    rng = np.random.default_rng(9)
    cfg = OracleConfig(d_model=8, n_heads=1, n_kv_heads=1, compression=1)
    s, d = 17, 8
    q = rng.normal(size=(s, d))
    k = rng.normal(size=(s, d))
    v = rng.normal(size=(s, d))
    # explicit full score matrix, mask, softmax written with python loops
    ref = np.zeros((s, d))
    for t in range(s):
        w = [math.exp(float(q[t] @ k[j]) / math.sqrt(d)) for j in range(t + 1)]
        z = sum(w)
        ref[t] = sum(wj / z * v[j] for j, wj in enumerate(w))
    np.testing.assert_allclose(O.causal_attention(q, k, v, cfg), ref, rtol=1e-12, atol=1e-12)
    # row 0 sees only itself
    np.testing.assert_allclose(O.causal_attention(q, k, v, cfg)[0], v[0], atol=1e-15)
    # equal keys: every visible key has the same weight -> running mean of the values
    keq = np.tile(k[:1], (s, 1))
    run_mean = np.cumsum(v, axis=0) / np.arange(1, s + 1)[:, None]
    np.testing.assert_allclose(O.causal_attention(q, keq, v, cfg), run_mean, rtol=1e-12)


def test_attention_row_subset_matches_full():
    rng = np.random.default_rng(10)
    cfg = CFG_SMALL
    s = 40
    q = rng.normal(size=(s, cfg.n_q))
    k = rng.normal(size=(s, cfg.n_kv))
    v = rng.normal(size=(s, cfg.n_kv))
    full = O.causal_attention(q, k, v, cfg)
    rows = np.array([0, 5, 17, 39])
    np.testing.assert_allclose(O.causal_attention(q[rows], k, v, cfg, q_positions=rows),
                               full[rows], rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------ whole-operator pins
def textbook_mha(x, wq, wk, wv, wo, H, rope_base, qk_rmsnorm=False):
    """Causal multi-head attention with RoPE, written independently of the oracle:
    complex-number RoPE and torch's scaled-dot-product attention."""
    s, E = x.shape
    hd = E // H
    q = (x @ wq.T)
    k = (x @ wk.T)
    v = (x @ wv.T)
    if qk_rmsnorm:
        q = torch.nn.functional.rms_norm(torch.tensor(q.reshape(s, H, hd)), (hd,), eps=1e-6).reshape(s, E).numpy()
        k = torch.nn.functional.rms_norm(torch.tensor(k.reshape(s, H, hd)), (hd,), eps=1e-6).reshape(s, E).numpy()
    q = rope_complex(q, np.arange(s), H, hd, rope_base)
    k = rope_complex(k, np.arange(s), H, hd, rope_base)
    qt = torch.tensor(q.reshape(s, H, hd)).transpose(0, 1)
    kt = torch.tensor(k.reshape(s, H, hd)).transpose(0, 1)
    vt = torch.tensor(v.reshape(s, H, hd)).transpose(0, 1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o.transpose(0, 1).reshape(s, E).numpy() @ wo.T


@pytest.mark.parametrize("norm", [False, True])
def test_reduces_to_causal_mha(norm):
    """C = 1, identity convs, q-k-mean and value-shift off: the layer is causal MHA with
    RoPE (and with QK RMS-norm when normalisation is on).  [gist] §2: CCA is attention
    moved into the latent space; at C = 1 the latent space is the full space."""
    rng = np.random.default_rng(11)
    cfg = OracleConfig(d_model=64, n_heads=4, n_kv_heads=4, compression=1,
                       qk_mean=False, value_shift=False, qk_norm=norm)
    w = identity_convs(cfg, rand_weights(cfg, rng))
    x = rng.normal(size=(33, 64))
    y, _ = O.prefill_sequence(cfg, w, x)
    ref = textbook_mha(x, w.w_q, w.w_k, w.w_v, w.w_o, 4, 10000.0, qk_rmsnorm=norm)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


def test_ccgqa_equals_cca_with_repeated_kv_heads():
    """[gist] Extension: CCGQA shares each latent key/value head among a contiguous group
    of query heads.  With q-k-mean off, CCGQA(H, Hkv) equals CCA(H, H) whose key/value
    projection rows and key conv filters are repeated per group."""
    rng = np.random.default_rng(12)
    H, Hk, C, E = 8, 2, 2, 128
    G = H // Hk
    g_cfg = OracleConfig(d_model=E, n_heads=H, n_kv_heads=Hk, compression=C, qk_mean=False)
    a_cfg = g_cfg.with_(n_kv_heads=H)
    d = g_cfg.dl
    wg = rand_weights(g_cfg, rng)
    rep_rows = lambda m: np.repeat(m.reshape(Hk, d, -1), G, axis=0).reshape(H * d, -1)
    wa = OracleWeights(
        w_q=wg.w_q, w_k=rep_rows(wg.w_k), w_v=rep_rows(wg.w_v), w_o=wg.w_o,
        conv_seq=np.concatenate([wg.conv_seq[:g_cfg.n_q], rep_rows(wg.conv_seq[g_cfg.n_q:])]),
        conv_chan=np.concatenate([wg.conv_chan[:H], np.repeat(wg.conv_chan[H:], G, axis=0)]))
    x = rng.normal(size=(30, E))
    yg, _ = O.prefill_sequence(g_cfg, wg, x)
    ya, _ = O.prefill_sequence(a_cfg, wa, x)
    np.testing.assert_allclose(yg, ya, rtol=1e-11, atol=1e-12)


def test_ccgqa_qk_mean_at_group_one_is_symmetric():
    """At G = 1 the same vector (pq + pk)/2 is added to q and to k."""
    rng = np.random.default_rng(13)
    cfg = OracleConfig(d_model=32, n_heads=4, n_kv_heads=4, compression=2)
    pq, pk, bq, bk = (rng.normal(size=(5, 16)) for _ in range(4))
    q, k = O.qk_mean(bq, bk, pq, pk, cfg)
    np.testing.assert_allclose(q - bq, k - bk, atol=1e-15)


@pytest.mark.parametrize("kc", [1, 2])
def test_causality(kc):
    rng = np.random.default_rng(14)
    cfg = CFG_SMALL.with_(chan_conv_kernel=kc)
    w = rand_weights(cfg, rng)
    x = rng.normal(size=(25, cfg.d_model))
    y0, _ = O.prefill_sequence(cfg, w, x)
    for t in (0, 1, 7, 23):
        x2 = x.copy()
        x2[t + 1:] += rng.normal(size=x2[t + 1:].shape)
        y1, _ = O.prefill_sequence(cfg, w, x2)
        np.testing.assert_allclose(y1[:t + 1], y0[:t + 1], rtol=1e-13, atol=1e-13)
        assert not np.allclose(y1[t + 1:], y0[t + 1:])


@pytest.mark.parametrize("kc,s0", [(1, 0), (1, 1), (1, 9), (2, 9), (1, 2)])
def test_decode_equals_prefill(kc, s0):
    """Prefill of s0 tokens then n single-token steps over the cache and conv state gives
    the same outputs and state as one prefill of s0 + n tokens."""
    rng = np.random.default_rng(15)
    cfg = CFG_SMALL.with_(chan_conv_kernel=kc)
    w = rand_weights(cfg, rng)
    n = 6
    x = rng.normal(size=(s0 + n, cfg.d_model))
    y_full, st_full = O.prefill_sequence(cfg, w, x)
    _, st = O.prefill_sequence(cfg, w, x[:s0])
    for i in range(n):
        y, st = O.decode_step(cfg, w, x[s0 + i], st)
        np.testing.assert_allclose(y, y_full[s0 + i], rtol=1e-11, atol=1e-12)
    for name in ("k_cache", "v_cache", "conv_state", "chan_state", "vshift_state"):
        np.testing.assert_allclose(getattr(st, name), getattr(st_full, name), rtol=1e-11, atol=1e-12)


def test_decode_batch_layout_matches_sequences():
    rng = np.random.default_rng(16)
    cfg = CFG_SMALL
    w = rand_weights(cfg, rng)
    B, max_seq = 3, 16
    lens = [4, 0, 11]
    Hk, d = cfg.n_kv_heads, cfg.dl
    kc = np.zeros((B, Hk, max_seq, d))
    vc = np.zeros((B, Hk, max_seq, d))
    conv = np.zeros((B, cfg.conv_kernel - 1, cfg.n_q + cfg.n_kv))
    vsh = np.zeros((B, cfg.n_kv - cfg.n_kv // 2))
    xs, full = [], []
    for b, L in enumerate(lens):
        x = rng.normal(size=(L + 1, cfg.d_model))
        yf, _ = O.prefill_sequence(cfg, w, x)
        _, st = O.prefill_sequence(cfg, w, x[:L])
        kc[b, :, :L] = st.k_cache.reshape(L, Hk, d).transpose(1, 0, 2)
        vc[b, :, :L] = st.v_cache.reshape(L, Hk, d).transpose(1, 0, 2)
        conv[b] = st.conv_state
        vsh[b] = st.vshift_state
        xs.append(x[L])
        full.append(yf[L])
    y, *_ = O.decode_batch(cfg, w, np.stack(xs), kc, vc, lens, conv, vsh)
    np.testing.assert_allclose(y, np.stack(full), rtol=1e-11, atol=1e-12)


def test_prefill_rows_matches_full():
    rng = np.random.default_rng(17)
    cfg = CFG_SMALL
    w = rand_weights(cfg, rng)
    x = rng.normal(size=(50, cfg.d_model))
    y, _ = O.prefill_sequence(cfg, w, x)
    rows = np.array([0, 3, 31, 32, 49])
    np.testing.assert_allclose(O.prefill_rows(cfg, w, x, rows), y[rows], rtol=1e-12, atol=1e-12)


def test_value_shift_state_and_switch():
    rng = np.random.default_rng(18)
    pv = rng.normal(size=(6, 8))
    prev = rng.normal(size=4)
    v = O.value_shift(pv, prev)
    np.testing.assert_allclose(v[0, 4:], prev)
    np.testing.assert_allclose(v[1:, 4:], pv[:-1, 4:])
    np.testing.assert_allclose(v[:, :4], pv[:, :4])
    cfg = CFG_SMALL.with_(value_shift=False, qk_mean=False, qk_norm=False, rope=False)
    w = rand_weights(cfg, rng)
    x = rng.normal(size=(5, cfg.d_model))
    _, _, st = O.prefill_sequence(cfg, w, x, return_stages=True)
    np.testing.assert_allclose(st["v"], st["pv"])


# ------------------------------------------------------------------ analytic counts
def test_parameters_and_cache_shrink_by_compression():
    """[abs]: parameters, KV cache and FLOPs all shrink by the compression factor C; with
    head sharing (CCGQA) the cache shrinks by a further H/Hkv (e.g. 8x at C=4, G=2)."""
    E, H = 2048, 16
    mha = OracleConfig(d_model=E, n_heads=H, n_kv_heads=H, compression=1)
    for C in (2, 4, 8):
        cca = mha.with_(compression=C)
        assert O.parameter_count(cca) == 4 * E * E // C
        assert O.parameter_count(mha) == C * O.parameter_count(cca)
        assert O.kv_cache_elements_per_token(mha) == C * O.kv_cache_elements_per_token(cca)
    ccgqa = mha.with_(compression=4, n_kv_heads=H // 2)
    assert O.kv_cache_elements_per_token(mha) == 8 * O.kv_cache_elements_per_token(ccgqa)


# ------------------------------------------------------------------ planted mistakes
def test_planted_mistakes_are_caught(monkeypatch):
    """Plausible mistakes planted in the oracle (CPU only) must each fail a pin."""
    orig_rope = O.rope_heads
    orig_shift = O.value_shift
    orig_conv = O.seq_conv
    orig_qkm = O.qk_mean

    def rope_wrong_sign(u, positions, n_heads, dl, base):
        return orig_rope(u, -np.asarray(positions, dtype=np.float64), n_heads, dl, base)

    def shift_by_two(pv, prev_row=None):
        v = orig_shift(pv, prev_row)
        half = pv.shape[1] // 2
        v[2:, half:] = pv[:-2, half:]
        return v

    def conv_reversed(p, w, history=None):
        return orig_conv(p, w[:, ::-1], history)

    def qkm_wrong_group(bq, bk, pq, pk, cfg):
        s = bq.shape[0]
        H, Hk, d = cfg.n_heads, cfg.n_kv_heads, cfg.dl
        pk_for_q = np.tile(pk.reshape(s, Hk, d), (1, H // Hk, 1))   # h % Hk instead of h // G
        q = bq.reshape(s, H, d) + 0.5 * (pq.reshape(s, H, d) + pk_for_q)
        _, k = orig_qkm(bq, bk, pq, pk, cfg)
        return q.reshape(s, H * d), k

    planted = [("rope_heads", rope_wrong_sign, [test_golden_rope, test_rope_matches_complex_rotation_and_properties]),
               ("value_shift", shift_by_two, [test_golden_value_shift]),
               ("seq_conv", conv_reversed, [test_golden_seq_conv_taps, lambda: test_seq_conv_matches_torch_conv1d(4)]),
               ("qk_mean", qkm_wrong_group, [test_golden_qk_mean_group])]
    for name, fn, pins in planted:
        with monkeypatch.context() as m:
            m.setattr(O, name, fn)
            for pin in pins:
                with pytest.raises(AssertionError):
                    pin()
