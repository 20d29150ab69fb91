"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bounds: float32 |y - y_oracle| <= 1e-4 + 1e-4 |y_oracle| elementwise; bf16
max |y - y_oracle| / rms(y_oracle) <= 2e-2.  The oracle computes in float64 from the exact
(rounded) values handed to the GPU.  Full-size workloads are checked on sampled rows
(first/last 16, tile boundaries +-1, 512 seeded rows per sequence) in the launch
configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle.cca_oracle as O
import workloads as W
from gpu_helpers import (BF16_TOL, assert_fp32_close, bf16_err, f64, oracle_config,
                         oracle_weights, sample_rows)

pytestmark = pytest.mark.gpu


def small(name, **kw):
    base = dict(batch=2, seq=200, d_model=256, n_heads=4, n_kv_heads=2, compression=2,
                description=name)
    base.update(kw)
    return W.Workload(name, **base)


# ------------------------------------------------------------------ single kernels
@pytest.mark.parametrize("a_trans,b_trans", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 264, 77), (1536, 2048, 1000),
                                   (2048, 1024, 4099), (64, 520, 8)])
def test_gemm_transposed_operands(cuda_lib, M, N, K, a_trans, b_trans):
    """cca_gemm_t: either operand read as stored transposed ([K, M] / [K, N], the MN-major
    tiles of the backward's gradient products), ragged M, N and K, against a float64 product."""
    cls = cuda_lib
    if (not a_trans or not b_trans) and K % 8:      # a K-major operand needs K % 8 == 0
        K += 8 - K % 8
    g = torch.Generator("cpu").manual_seed(M * 7 + N * 3 + K + a_trans * 2 + b_trans)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    ref = A.double() @ B.double().T
    As = (A.t() if a_trans else A).contiguous().cuda()
    Bs = (B.t() if b_trans else B).contiguous().cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    C32 = torch.empty(M, N, dtype=torch.float32, device="cuda")
    cls.cca_gemm_t(cls.CCA_F32, As, Bs, C32, M, N, K, a_trans, b_trans, status)
    C16 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    cls.cca_gemm_t(cls.CCA_BF16, As, Bs, C16, M, N, K, a_trans, b_trans, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    err = (C32.double().cpu() - ref).abs()
    assert (err <= 2e-5 * ref.abs() + 1e-4 * ref.pow(2).mean().sqrt()).all(), float(err.max())
    err16 = (C16.double().cpu() - ref).abs()
    assert (err16 <= 8e-3 * ref.abs() + 2e-3 * ref.pow(2).mean().sqrt()).all(), float(err16.max())


def test_gemm_transposed_rejects_ragged_rows(cuda_lib):
    cls = cuda_lib
    A = torch.zeros(12, 16, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(16, 16, dtype=torch.float32, device="cuda")
    with pytest.raises(cls.CCAError) as e:       # A stored [K=12, M=16]: fine; B [K, N=12]: not
        cls.cca_gemm_t(cls.CCA_F32, A, A, C, 16, 12, 12, 1, 1)
    assert e.value.code == cls.CCA_ERR_UNSUPPORTED


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 520, 200), (1000, 1536, 2048),
                                   (257, 768, 512), (64, 2048, 512), (4096, 2048, 1024)])
def test_gemm_bf16_tcgen05(cuda_lib, M, N, K):
    cls = cuda_lib
    g = torch.Generator("cpu").manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    ref = A.double() @ B.double().T
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cls.cca_gemm(cls.CCA_BF16, cls.CCA_BF16, A.cuda(), B.cuda(), C, M, N, K, status)
    C32 = torch.empty(M, N, dtype=torch.float32, device="cuda")
    cls.cca_gemm(cls.CCA_BF16, cls.CCA_F32, A.cuda(), B.cuda(), C32, M, N, K, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    err = (C.double().cpu() - ref).abs()
    assert (err <= 8e-3 * ref.abs() + 2e-3 * ref.pow(2).mean().sqrt()).all(), float(err.max())
    # float16 operands (the up-projection of 16-bit layers)
    Ch = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    Ah, Bh = A.half(), B.half()
    cls.cca_gemm(cls.CCA_F16, cls.CCA_BF16, Ah.cuda(), Bh.cuda(), Ch, M, N, K, status)
    refh = Ah.double() @ Bh.double().T
    errh = (Ch.double().cpu() - refh).abs()
    assert (errh <= 8e-3 * refh.abs() + 2e-3 * refh.pow(2).mean().sqrt()).all(), float(errh.max())
    # float32 result: only the fp32 accumulation order differs from the float64 product
    err32 = (C32.double().cpu() - ref).abs()
    assert (err32 <= 1e-5 * ref.abs() + 1e-5 * ref.pow(2).mean().sqrt()).all(), float(err32.max())


@pytest.mark.parametrize("M,N,K", [(128, 192, 256), (77, 130, 48)])
def test_gemm_f32_simt(cuda_lib, M, N, K):
    cls = cuda_lib
    g = torch.Generator("cpu").manual_seed(7)
    A = torch.randn(M, K, generator=g)
    B = torch.randn(N, K, generator=g) * 0.05
    C = torch.empty(M, N, device="cuda")
    cls.cca_gemm(cls.CCA_F32, cls.CCA_F32, A.cuda(), B.cuda(), C, M, N, K)
    torch.cuda.synchronize()
    assert_fp32_close(f64(C), (A.double() @ B.double().T).numpy())


# Shapes cover d~ = 16 / 32 / 64, G = 1..8, token counts off the 32-token unit, sequence-conv
# widths other than 4 (the generic-tap code paths; width 1 has no halo of its own), and G = 8 at
# d~ = 64, whose filters and P tiles do not fit the persistent kernel (the per-tile fallback).
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("H,Hkv,C,E,S,KC", [(4, 4, 4, 256, 130, 4), (8, 2, 2, 512, 77, 4),
                                            (6, 3, 1, 96, 65, 4), (4, 1, 2, 512, 33, 4),
                                            (8, 2, 2, 512, 70, 2), (4, 2, 4, 256, 45, 6),
                                            (4, 4, 4, 256, 40, 1), (8, 1, 1, 512, 70, 4)])
def test_stencil_matches_oracle(cuda_lib, dtype, H, Hkv, C, E, S, KC):
    cls = cuda_lib
    w = W.Workload("t", 2, S, E, H, Hkv, C, dtype=dtype, conv_kernel=KC)
    ocfg = oracle_config(w)
    inp = W.make_inputs(w, seed=3, conv_std=0.3, identity_conv=True)
    dt = w.torch_dtype
    g = torch.Generator("cpu").manual_seed(11)
    P = torch.randn(2 * S, w.n_q + 2 * w.n_kv, generator=g)            # projections: float32
    q = torch.empty(2, H, S, w.dl, dtype=w.latent_dtype, device="cuda")
    k = torch.empty(2, Hkv, S + 5, w.dl, dtype=w.latent_dtype, device="cuda")
    v = torch.empty(2, Hkv, S + 5, w.dl, dtype=w.latent_dtype, device="cuda")
    cfg = cls.make_config(E, H, Hkv, C, conv_kernel=KC,
                          dtype=cls.CCA_BF16 if dtype == "bf16" else cls.CCA_F32)
    ws = torch.empty(cls.cca_stage_stencil_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    cls.cca_stage_stencil(cfg, P.cuda(), 2, S, inp.conv_seq.cuda(), inp.conv_chan.cuda(), q, k, v,
                          S + 5, ws)
    cls.cca_workspace_status(ws)
    ow = oracle_weights(ocfg, inp)
    for b in range(2):
        p = f64(P[b * S:(b + 1) * S])
        pq, pk, pv = p[:, :w.n_q], p[:, w.n_q:w.n_q + w.n_kv], p[:, w.n_q + w.n_kv:]
        rq, rk, rv, _ = O.latent_qkv(ocfg, ow, pq, pk, pv, np.arange(S))
        gq = f64(q[b]).transpose(1, 0, 2).reshape(S, -1)
        gk = f64(k[b, :, :S]).transpose(1, 0, 2).reshape(S, -1)
        gv = f64(v[b, :, :S]).transpose(1, 0, 2).reshape(S, -1)
        for got, ref in ((gq, rq), (gk, rk), (gv, rv)):
            if dtype == "f32":
                assert_fp32_close(got, ref)
            else:
                assert bf16_err(got, ref) <= BF16_TOL


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
# S = 385, 769 and 1000 give CTAs with all their query tiles in use and several tile groups
# per head, including rows whose whole diagonal key tile is masked.
@pytest.mark.parametrize("H,Hkv,DL,S", [(4, 4, 16, 130), (4, 2, 32, 200), (8, 2, 64, 129),
                                        (3, 1, 32, 64), (2, 2, 64, 1), (4, 1, 64, 385),
                                        (4, 2, 64, 769), (2, 1, 64, 1000), (8, 2, 32, 385),
                                        (4, 4, 32, 1000), (8, 1, 32, 769), (8, 8, 16, 1000),
                                        (4, 4, 128, 385), (4, 2, 128, 200), (2, 1, 128, 1000),
                                        (8, 1, 128, 130)])
def test_attention_matches_oracle(cuda_lib, dtype, H, Hkv, DL, S):
    cls = cuda_lib
    if DL == 128 and dtype == "f32":
        pytest.skip("latent width 128 is a 16-bit path")
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    qkt = torch.float32 if dtype == "f32" else torch.float16
    g = torch.Generator("cpu").manual_seed(5)
    B = 2
    q = torch.randn(B, H, S, DL, generator=g).to(qkt)
    k = torch.randn(B, Hkv, S, DL, generator=g).to(qkt)
    v = torch.randn(B, Hkv, S, DL, generator=g).to(qkt)
    o = torch.empty(B * S, H * DL, dtype=qkt, device="cuda")
    E = H * DL * 2
    cfg = cls.make_config(E, H, Hkv, 2, dtype=cls.CCA_BF16 if dtype == "bf16" else cls.CCA_F32)
    cls.cca_stage_attention(cfg, q.cuda(), k.cuda(), v.cuda(), B, S, S, o)
    torch.cuda.synchronize()
    ocfg = O.OracleConfig(d_model=E, n_heads=H, n_kv_heads=Hkv, compression=2)
    for b in range(B):
        ref = O.causal_attention(f64(q[b]).transpose(1, 0, 2).reshape(S, -1),
                                 f64(k[b]).transpose(1, 0, 2).reshape(S, -1),
                                 f64(v[b]).transpose(1, 0, 2).reshape(S, -1), ocfg)
        got = f64(o[b * S:(b + 1) * S])
        if dtype == "f32":
            assert_fp32_close(got, ref)
        else:
            assert bf16_err(got, ref) <= BF16_TOL


# ------------------------------------------------------------------ whole layer
def run_prefill(cls, w, inp, flags=None):
    layer = cls.CCALayer.from_workload(w, inp, flags=flags)
    y = layer.prefill(inp.x.cuda())
    torch.cuda.synchronize()
    return layer, y


@pytest.mark.parametrize("conv_std", [0.02, 0.5])
def test_prefill_tiny_fp32(cuda_lib, conv_std):
    """CCA tiny fp32: B=1 S=128 E=256 H=4 Hkv=4 C=4 (d~=16)."""
    w = W.WORKLOADS["cca_tiny_fp32"]
    inp = W.make_inputs(w, seed=0, conv_std=conv_std)
    _, y = run_prefill(cuda_lib, w, inp)
    ocfg = oracle_config(w)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))
    assert_fp32_close(f64(y), ref)


@pytest.mark.parametrize("flags", [15, 14, 13, 11, 7, 0])
@pytest.mark.parametrize("shape", [
    dict(n_heads=4, n_kv_heads=4, compression=4, seq=129),              # CCA, d~=16
    dict(n_heads=4, n_kv_heads=2, compression=2, seq=200),              # CCGQA, d~=32
    dict(n_heads=8, n_kv_heads=2, compression=1, d_model=512, seq=77),  # d~=64, G=4
])
def test_prefill_bf16_flags(cuda_lib, shape, flags):
    w = small("bf16", **shape)
    inp = W.make_inputs(w, seed=1, conv_std=0.4, identity_conv=True)
    _, y = run_prefill(cuda_lib, w, inp, flags)
    ocfg = oracle_config(w, flags)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))
    assert bf16_err(f64(y), ref) <= BF16_TOL


@pytest.mark.parametrize("seq", [1, 2, 3, 4, 63, 64, 65, 127, 128, 129, 300])
def test_prefill_ragged_lengths(cuda_lib, seq):
    w = small("ragged", seq=seq, n_heads=6, n_kv_heads=3, d_model=192, compression=1)   # d~=32
    inp = W.make_inputs(w, seed=seq, conv_std=0.4)
    _, y = run_prefill(cuda_lib, w, inp)
    ocfg = oracle_config(w)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))
    assert bf16_err(f64(y), ref) <= BF16_TOL


def test_prefill_causality_gpu(cuda_lib):
    w = small("causal", seq=257)
    inp = W.make_inputs(w, seed=2, conv_std=0.4)
    layer, y0 = run_prefill(cuda_lib, w, inp)
    x2 = inp.x.clone()
    x2[:, 130:] = torch.randn(x2[:, 130:].shape, generator=torch.Generator().manual_seed(9)).to(x2.dtype)
    y1 = layer.prefill(x2.cuda())
    torch.cuda.synchronize()
    assert torch.equal(y0[:, :130], y1[:, :130])
    assert not torch.equal(y0[:, 130:], y1[:, 130:])


def test_ccgqa_kv_eq_heads_equals_cca(cuda_lib):
    """The GPU path with Hkv = H is CCA: equal to the oracle's CCA."""
    w = small("cca", n_heads=4, n_kv_heads=4, compression=2, seq=150)
    inp = W.make_inputs(w, seed=4, conv_std=0.3)
    _, y = run_prefill(cuda_lib, w, inp)
    ocfg = oracle_config(w)
    assert bf16_err(f64(y), O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))) <= BF16_TOL


@pytest.mark.parametrize("name", ["cca_prefill_4k", "ccgqa_prefill_16k", "ccgqa_prefill_32k"])
def test_full_size_prefill_sampled(cuda_lib, name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0)
    _, y = run_prefill(cuda_lib, w, inp)
    ocfg = oracle_config(w)
    ow = oracle_weights(ocfg, inp)
    rng = np.random.default_rng(0)
    for b in range(w.batch):
        rows = sample_rows(w.seq, rng)
        ref = O.prefill_rows(ocfg, ow, f64(inp.x[b]), rows)
        got = f64(y[b, torch.as_tensor(rows)])
        assert np.isfinite(got).all()
        assert bf16_err(got, ref) <= BF16_TOL, (b, bf16_err(got, ref))


def test_prefill_fills_cache_and_state(cuda_lib):
    cls = cuda_lib
    w = small("cache", seq=70)
    inp = W.make_inputs(w, seed=6, conv_std=0.4)
    layer = cls.CCALayer.from_workload(w, inp)
    cache = layer.new_cache(w.batch, 96)
    layer.prefill(inp.x.cuda(), cache=cache)
    torch.cuda.synchronize()
    ocfg = oracle_config(w)
    ow = oracle_weights(ocfg, inp)
    assert cache.lengths.tolist() == [70, 70]
    for b in range(w.batch):
        _, st = O.prefill_sequence(ocfg, ow, f64(inp.x[b]))
        gk = f64(cache.k[b, :, :70]).transpose(1, 0, 2).reshape(70, -1)
        gv = f64(cache.v[b, :, :70]).transpose(1, 0, 2).reshape(70, -1)
        assert bf16_err(gk, st.k_cache) <= BF16_TOL
        assert bf16_err(gv, st.v_cache) <= BF16_TOL
        assert bf16_err(f64(cache.conv_state[b]), st.conv_state) <= BF16_TOL
        assert bf16_err(f64(cache.vshift_state[b]), st.vshift_state) <= BF16_TOL


# ------------------------------------------------------------------ decode
def load_cache(cache, inp, ctx):
    cache.k[:, :, :ctx] = inp.k_cache.cuda()
    cache.v[:, :, :ctx] = inp.v_cache.cuda()
    cache.conv_state.copy_(inp.conv_state.cuda())
    cache.vshift_state.copy_(inp.vshift_state.cuda())
    cache.lengths.copy_(inp.lengths.cuda())


def decode_vs_oracle(cls, w, inp, max_seq):
    layer = cls.CCALayer.from_workload(w, inp)
    cache = layer.new_cache(w.batch, max_seq)
    load_cache(cache, inp, w.seq)
    y = layer.decode(inp.x.cuda(), cache)
    cls.cca_cache_check(cache.struct)
    ocfg = oracle_config(w)
    ow = oracle_weights(ocfg, inp)
    ref_y, ref_k, ref_v, ref_conv, ref_vs = O.decode_batch(
        ocfg, ow, f64(inp.x), f64(inp.k_cache), f64(inp.v_cache), inp.lengths.numpy(),
        f64(inp.conv_state), f64(inp.vshift_state))
    return layer, cache, y, (ref_y, ref_k, ref_v, ref_conv, ref_vs)


def test_decode_step_full_size(cuda_lib):
    """CCGQA bf16 decode: B=64, 8192 cached tokens, one new token each."""
    w = W.WORKLOADS["ccgqa_decode_8k"]
    inp = W.make_inputs(w, seed=0)
    layer, cache, y, (ry, rk, rv, rc, rvs) = decode_vs_oracle(cuda_lib, w, inp, w.seq + 64)
    assert bf16_err(f64(y), ry) <= BF16_TOL
    L = w.seq
    gk = f64(cache.k[:, :, L]).reshape(w.batch, -1)
    gv = f64(cache.v[:, :, L]).reshape(w.batch, -1)
    assert bf16_err(gk, rk) <= BF16_TOL and bf16_err(gv, rv) <= BF16_TOL
    assert bf16_err(f64(cache.conv_state), rc) <= BF16_TOL
    assert bf16_err(f64(cache.vshift_state), rvs) <= BF16_TOL
    assert (cache.lengths.cpu() == L + 1).all()


def test_decode_kernel_count(cuda_lib):
    """The step launches projection, stencil, attention and output kernels, plus the merge of
    the attention's key splits when the (sequence, group) pairs are fewer than the SMs; with
    unsplit keys and d~ <= 32 the stencil runs inside the attention kernel."""
    cls = cuda_lib
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cfg = cls.make_config(2048, 16, 4, 4)
    assert cls.cca_decode_kernel_count(cfg, 64, 8300) == (3 if 64 * 4 >= sms else 5)
    cfg64 = cls.make_config(2048, 16, 4, 2)                  # d~ = 64: stencil kernel of its own
    assert cls.cca_decode_kernel_count(cfg64, 64, 8300) == (4 if 64 * 4 >= sms else 5)
    assert cls.cca_decode_kernel_count(cfg, 2, 8300) == 5
    assert cls.cca_decode_kernel_count(cls.make_config(256, 4, 4, 4, dtype=cls.CCA_F32), 64, 300) == 5
    assert cls.cca_decode_kernel_count(cfg, 0, 8300) < 0


@pytest.mark.parametrize("C,max_seq,lengths", [
    (2, 320, [0, 1, 255, 256, 300]),      # d~=32, keys split over CTAs (merge kernel)
    (2, 256, [0, 1, 129, 255, 200]),      # d~=32, unsplit: stencil inside the attention kernel
    (4, 256, [3, 0, 255, 64, 77]),        # d~=16, unsplit, fused
])
def test_decode_ragged_lengths(cuda_lib, C, max_seq, lengths):
    w = W.Workload("dec", 5, max(lengths), 256, 4, 2, C, decode=True)
    inp = W.make_inputs(w, seed=2, conv_std=0.4, lengths=lengths)
    _, cache, y, (ry, *_rest) = decode_vs_oracle(cuda_lib, w, inp, max_seq)
    assert bf16_err(f64(y), ry) <= BF16_TOL
    assert cache.lengths.cpu().tolist() == [l + 1 for l in lengths]


@pytest.mark.parametrize("C,max_seq", [(2, 2048), (4, 3072)])
def test_decode_ragged_long_unsplit(cuda_lib, C, max_seq):
    """Unsplit keys (160 (sequence, group) pairs) over many 256-key sub-chunks: lengths on and
    around the sub-chunk boundaries, the end of the sub-chunks the fused kernel parks in tensor
    memory (4 at d~=32, 5 at d~=16) and the end of those it leaves in the copy ring."""
    edges = [0, 1, 255, 256, 257, 511, 512, 767, 768, 1023, 1024, 1025, 1279, 1280, 1281,
             1535, 1536, 1537, 1791, 1792, 2047]
    rng = np.random.default_rng(5)
    lengths = [min(e, max_seq - 1) for e in edges] + \
        [int(v) for v in rng.integers(0, max_seq, 40 - len(edges))]
    w = W.Workload("dec_long", 40, max(lengths), 512, 8, 4, C, decode=True)
    inp = W.make_inputs(w, seed=4, conv_std=0.4, lengths=lengths)
    assert cuda_lib.cca_decode_kernel_count(cuda_lib.make_config(512, 8, 4, C), 40, max_seq) == 3
    _, cache, y, (ry, rk, rv, *_rest) = decode_vs_oracle(cuda_lib, w, inp, max_seq)
    assert bf16_err(f64(y), ry) <= BF16_TOL
    assert cache.lengths.cpu().tolist() == [l + 1 for l in lengths]
    idx = torch.tensor(lengths)
    ar = torch.arange(w.batch)
    gk = f64(cache.k[ar, :, idx]).reshape(w.batch, -1)
    gv = f64(cache.v[ar, :, idx]).reshape(w.batch, -1)
    assert bf16_err(gk, rk) <= BF16_TOL and bf16_err(gv, rv) <= BF16_TOL


@pytest.mark.parametrize("KC", [4, 2, 6])
def test_decode_equals_prefill_gpu(cuda_lib, KC):
    """Prefill S0 tokens into the cache, then n decode steps == prefill of S0 + n tokens (the
    conv state carries KC - 1 pre-conv rows from the prefill into the decode)."""
    cls = cuda_lib
    w = small("dp", seq=40, batch=3, conv_kernel=KC)
    inp = W.make_inputs(w, seed=8, conv_std=0.4)
    layer = cls.CCALayer.from_workload(w, inp)
    s0, n = 33, 7
    x = inp.x.cuda()
    y_full = layer.prefill(x)
    cache = layer.new_cache(w.batch, 64)
    layer.prefill(x[:, :s0].contiguous(), cache=cache)
    for i in range(n):
        yi = layer.decode(x[:, s0 + i].contiguous(), cache)
        torch.cuda.synchronize()
        assert bf16_err(f64(yi), f64(y_full[:, s0 + i])) <= BF16_TOL
    ocfg = oracle_config(w)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))
    assert bf16_err(f64(yi), ref[:, s0 + n - 1]) <= BF16_TOL
    assert cache.lengths.tolist() == [s0 + n] * w.batch


def test_decode_f32_equals_prefill(cuda_lib):
    cls = cuda_lib
    w = W.WORKLOADS["cca_tiny_fp32"].with_(batch=2, seq=20)
    inp = W.make_inputs(w, seed=3, conv_std=0.4)
    layer = cls.CCALayer.from_workload(w, inp)
    cache = layer.new_cache(2, 32)
    x = inp.x.cuda()
    layer.prefill(x[:, :15].contiguous(), cache=cache)
    ocfg = oracle_config(w)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))
    for i in range(15, 20):
        yi = layer.decode(x[:, i].contiguous(), cache)
        torch.cuda.synchronize()
        assert_fp32_close(f64(yi), ref[:, i])


def test_decode_cache_full(cuda_lib):
    cls = cuda_lib
    w = W.Workload("full", 2, 16, 256, 4, 2, 2, decode=True)
    inp = W.make_inputs(w, seed=1, lengths=[16, 10])
    layer = cls.CCALayer.from_workload(w, inp)
    cache = layer.new_cache(2, 16)
    load_cache(cache, inp, 16)
    k_before = cache.k.clone()
    y = layer.decode(inp.x.cuda(), cache)
    with pytest.raises(cls.CCAError) as e:
        cls.cca_cache_check(cache.struct)
    assert e.value.code == cls.CCA_ERR_CACHE_FULL
    cls.cca_cache_check(cache.struct)          # the status word was cleared
    assert torch.equal(y[0].float().cpu(), torch.zeros(w.d_model))
    assert torch.equal(cache.k[0], k_before[0])
    assert cache.lengths.tolist() == [16, 11]


def test_prefill_workspace_status_clean(cuda_lib):
    cls = cuda_lib
    w = small("st", seq=300)
    inp = W.make_inputs(w, seed=0)
    layer, _ = run_prefill(cls, w, inp)
    cls.cca_workspace_status(layer._ws)


def test_latent_range_is_reported(cuda_lib):
    """A value latent beyond the float16 range is reported, not silently stored."""
    cls = cuda_lib
    w = small("range", seq=40)
    inp = W.make_inputs(w, seed=0)
    layer = cls.CCALayer.from_workload(w, inp)
    layer.prefill((inp.x.float() * 3e5).to(inp.x.dtype).cuda())
    with pytest.raises(cls.CCAError) as e:
        cls.cca_workspace_status(layer._ws)
    assert e.value.code == cls.CCA_ERR_RANGE
    layer.prefill(inp.x.cuda())
    cls.cca_workspace_status(layer._ws)        # the status word is reset by every call


# ------------------------------------------------------------------ identity convolutions
@pytest.mark.parametrize("flags", [8 | 16, 15 | 16, 16])
@pytest.mark.parametrize("shape", [
    dict(d_model=512, n_heads=4, n_kv_heads=4, compression=1, seq=300),   # MHA, hd=128
    dict(d_model=512, n_heads=4, n_kv_heads=2, compression=1, seq=257),   # GQA, hd=128
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=2, seq=130),   # d~=32
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=1, seq=333),   # d~=64
    dict(d_model=256, n_heads=4, n_kv_heads=4, compression=4, seq=99),    # d~=16
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=2, seq=77, dtype="f32"),
])
def test_prefill_no_conv(cuda_lib, shape, flags):
    """CCA_NO_CONV: both convolutions are the identity.  With C = 1 and RoPE alone this is
    textbook causal MHA / GQA with rotary embeddings (the oracle's MHA reduction)."""
    w = small("noconv", **shape)
    inp = W.make_inputs(w, seed=7)
    _, y = run_prefill(cuda_lib, w, inp, flags)
    ocfg = oracle_config(w, flags)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp, no_conv=True), f64(inp.x))
    if w.dtype == "f32":
        assert_fp32_close(f64(y), ref)
    else:
        assert bf16_err(f64(y), ref) <= BF16_TOL


@pytest.mark.parametrize("name", ["mha_prefill_16k", "gqa8_prefill_16k"])
def test_baseline_prefill_sampled(cuda_lib, name):
    """The MHA and GQA-8 baselines the benchmark times, at full size, on sampled rows."""
    w = W.BASELINES[name]
    inp = W.make_inputs(w, seed=0)
    _, y = run_prefill(cuda_lib, w, inp)
    ocfg = oracle_config(w, w.flags)
    ow = oracle_weights(ocfg, inp, no_conv=True)
    rng = np.random.default_rng(1)
    b = 1
    rows = sample_rows(w.seq, rng, n_random=128)
    ref = O.prefill_rows(ocfg, ow, f64(inp.x[b]), rows)
    got = f64(y[b, torch.as_tensor(rows)])
    assert np.isfinite(got).all()
    assert bf16_err(got, ref) <= BF16_TOL


def test_no_conv_rejects_decode(cuda_lib):
    cls = cuda_lib
    cfg = cls.make_config(512, 4, 4, 1, flags=8 | 16)
    with pytest.raises(cls.CCAError) as e:
        cls.cca_cache_alloc(cfg, 2, 64)
    assert e.value.code == cls.CCA_ERR_UNSUPPORTED


# ------------------------------------------------------------------ fused projection + stencil
@pytest.mark.parametrize("shape", [
    dict(d_model=512, n_heads=8, n_kv_heads=2, compression=1, seq=300),     # d~=64, G=4, NG=1
    dict(d_model=512, n_heads=8, n_kv_heads=4, compression=2, seq=250),     # d~=32, G=2
    dict(d_model=256, n_heads=4, n_kv_heads=4, compression=4, seq=131),     # d~=16, G=1, NG=4
    dict(d_model=512, n_heads=16, n_kv_heads=4, compression=1, seq=129, conv_kernel=6),
    dict(d_model=512, n_heads=16, n_kv_heads=8, compression=1, seq=64, conv_kernel=1),
])
def test_prefill_fused_and_unfused_paths(cuda_lib, shape, monkeypatch):
    """The fused down-projection + stencil kernel and the separate GEMM + stencil kernels both
    match the oracle (and each other) on the same inputs, with a cache (decode state) too."""
    w = small("fused", **shape)
    inp = W.make_inputs(w, seed=12, conv_std=0.4, identity_conv=True)
    ocfg = oracle_config(w)
    ow = oracle_weights(ocfg, inp)
    ref = O.prefill(ocfg, ow, f64(inp.x))
    outs = []
    for unfused in ("fused", "unfused"):
        monkeypatch.setenv("CCA_PREFILL_PATH", unfused)
        layer = cuda_lib.CCALayer.from_workload(w, inp)
        cache = layer.new_cache(w.batch, w.seq + 8)
        y = layer.prefill(inp.x.cuda(), cache=cache)
        torch.cuda.synchronize()
        cuda_lib.cca_workspace_status(layer._ws)
        assert bf16_err(f64(y), ref) <= BF16_TOL, unfused
        for b in range(w.batch):
            _, st = O.prefill_sequence(ocfg, ow, f64(inp.x[b]))
            S = w.seq
            assert bf16_err(f64(cache.k[b, :, :S]).transpose(1, 0, 2).reshape(S, -1), st.k_cache) <= BF16_TOL
            assert bf16_err(f64(cache.v[b, :, :S]).transpose(1, 0, 2).reshape(S, -1), st.v_cache) <= BF16_TOL
            if w.conv_kernel > 1:
                assert bf16_err(f64(cache.conv_state[b]), st.conv_state) <= BF16_TOL
            assert bf16_err(f64(cache.vshift_state[b]), st.vshift_state) <= BF16_TOL
        assert cache.lengths.tolist() == [w.seq] * w.batch
        outs.append(f64(y))
    assert bf16_err(outs[0], outs[1]) <= BF16_TOL


# ------------------------------------------------------------------ FMA-pipe exponential
def test_exp2_poly_stage(cuda_lib):
    """The cubic exp2 the latent attention evaluates part of its probabilities with, on the
    device: relative error below 1e-4 against float64 exp2 on [-125, 126]; arguments below
    -125 give about 2^-125 (zero once rounded to float16); odd lengths are refused."""
    cls = cuda_lib
    g = torch.Generator("cpu").manual_seed(5)
    x = torch.cat([torch.rand(1 << 20, generator=g, dtype=torch.float64) * 251 - 125,
                   torch.arange(-125, 126.5, 0.5, dtype=torch.float64),
                   torch.tensor([0.0, 1e-7, -1e-7, 0.4999999, -0.4999999])]).float()
    x = x[: x.numel() // 2 * 2].contiguous()
    xd = x.cuda()
    yd = torch.empty_like(xd)
    cls.cca_stage_exp2_poly(xd, yd)
    torch.cuda.synchronize()
    y = yd.cpu().double()
    ref = torch.exp2(x.double())
    assert float((y / ref - 1).abs().max()) < 1e-4
    low = torch.tensor([-126.0, -500.0, float("-inf"), -125.0], device="cuda")
    ylow = torch.empty_like(low)
    cls.cca_stage_exp2_poly(low, ylow)
    torch.cuda.synchronize()
    assert bool((ylow > 0).all()) and float(ylow.max()) <= 2.0 ** -124.9
    with pytest.raises(cls.CCAError):
        cls.cca_stage_exp2_poly(low[:3], ylow[:3])
