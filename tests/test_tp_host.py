"""Tensor parallelism by key/value group, host side (no GPU): the weight slices of the ranks
partition the layer's parameters, the ranks' value-shift splits together are the layer's,
the C ABI accepts and checks the rank fields, and on world-size-2 gloo ranks the sum of the
ranks' up-projection shares (one all-reduce) is the oracle's layer output."""
import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _shapes():
    return [W.Workload("tp", 1, 40, 512, 8, 4, 2, dtype="f32"),     # CCGQA, d~=32, G=2
            W.Workload("tp", 1, 40, 256, 4, 4, 4, dtype="f32"),     # CCA, d~=16
            W.Workload("tp", 1, 40, 512, 8, 2, 1, dtype="f32")]     # d~=64, G=4


@pytest.mark.parametrize("wi", range(3))
@pytest.mark.parametrize("tp", [1, 2, 4])
def test_shards_partition_the_weights(wi, tp):
    from compressed_latent_space_b200.tp import shard_weights
    w = _shapes()[wi]
    if w.n_kv_heads % tp:
        pytest.skip("kv heads not divisible")
    inp = W.make_inputs(w, seed=0)
    parts = [shard_weights(inp.w_qkv, inp.w_o, inp.conv_seq, inp.conv_chan, w.n_heads,
                           w.n_kv_heads, w.dl, tp, r) for r in range(tp)]
    nq_l, nkv_l = w.n_q // tp, w.n_kv // tp
    # W_q, W_k, W_v rows, conv rows and channel-conv heads, W_o columns: each exactly once
    wq = torch.cat([p[0][:nq_l] for p in parts])
    wk = torch.cat([p[0][nq_l:nq_l + nkv_l] for p in parts])
    wv = torch.cat([p[0][nq_l + nkv_l:] for p in parts])
    assert torch.equal(torch.cat([wq, wk, wv]), inp.w_qkv)
    assert torch.equal(torch.cat([p[1] for p in parts], dim=1), inp.w_o)
    cq = torch.cat([p[2][:nq_l] for p in parts])
    ck = torch.cat([p[2][nq_l:] for p in parts])
    assert torch.equal(torch.cat([cq, ck]), inp.conv_seq)
    hq, hk = w.n_heads // tp, w.n_kv_heads // tp
    fq = torch.cat([p[3][:hq] for p in parts])
    fk = torch.cat([p[3][hq:] for p in parts])
    assert torch.equal(torch.cat([fq, fk]), inp.conv_chan)
    for p in parts:
        assert p[0].shape == (nq_l + 2 * nkv_l, w.d_model) and p[0].is_contiguous()
        assert p[1].shape == (w.d_model, nq_l) and p[1].is_contiguous()


@pytest.mark.parametrize("wi", range(3))
@pytest.mark.parametrize("tp", [1, 2, 4])
def test_value_shift_split_follows_the_layer(wi, tp):
    """Global value channel c is shifted iff c >= n_kv/2 (the layer's reading); rank r's local
    channel j is global channel r * n_kv/R + j."""
    from compressed_latent_space_b200.layer import CCALayer
    from compressed_latent_space_b200.tp import shard_weights
    w = _shapes()[wi]
    if w.n_kv_heads % tp:
        pytest.skip("kv heads not divisible")
    inp = W.make_inputs(w, seed=0)
    shifted = set()
    for r in range(tp):
        lw = shard_weights(inp.w_qkv, inp.w_o, inp.conv_seq, inp.conv_chan, w.n_heads,
                           w.n_kv_heads, w.dl, tp, r)
        layer = CCALayer(w.d_model, w.n_heads, w.n_kv_heads, w.compression, *lw, dtype="f32",
                         device="cpu", tp_size=tp, tp_rank=r)
        shifted |= {r * layer.n_kv + j for j in range(layer.vshift_begin, layer.n_kv)}
    assert shifted == set(range(w.n_kv // 2, w.n_kv))


def test_abi_checks_the_rank_fields():
    from compressed_latent_space_b200 import build
    build.build()
    import compressed_latent_space_b200 as cls
    lib = cls.load()
    n = ctypes.c_size_t(0)

    def cache_bytes(**kw):
        c = cls.make_config(512, 8, 4, 2, dtype=cls.CCA_BF16, **kw)
        rc = lib.cca_cache_alloc(ctypes.byref(c), 2, 64, None, ctypes.byref(n), None, None)
        return rc, n.value

    assert cache_bytes(tp_size=2, tp_rank=2)[0] == cls.CCA_ERR_INVALID_ARG
    assert cache_bytes(tp_size=2, tp_rank=-1)[0] == cls.CCA_ERR_INVALID_ARG
    assert cache_bytes(tp_size=8, tp_rank=0)[0] == cls.CCA_ERR_INVALID_ARG    # 4 kv heads
    rc0, b0 = cache_bytes(tp_size=2, tp_rank=0)
    rc1, b1 = cache_bytes(tp_size=2, tp_rank=1)
    rcf, bf = cache_bytes()
    assert rc0 == rc1 == rcf == 0
    # rank 0 holds only unshifted value channels, rank 1 only shifted ones: the value-shift
    # state (64 sequences' worth of 64 floats, 256-byte aligned) lives on rank 1 alone
    assert b1 - b0 == 256 * ((2 * 64 * 4 + 255) // 256)
    assert b0 < bf and b1 < bf


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, ROOT)
    import oracle.cca_oracle as O
    from compressed_latent_space_b200.tp import kv_group_slice, shard_weights, tp_all_reduce
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.Workload("tp", 1, 48, 512, 8, 4, 2, dtype="f32")
        inp = W.make_inputs(w, seed=4, conv_std=0.3)
        cfg = O.OracleConfig(d_model=w.d_model, n_heads=w.n_heads, n_kv_heads=w.n_kv_heads,
                             compression=w.compression)
        f64 = lambda t: t.to(torch.float64).numpy()
        ow = O.OracleWeights.from_arrays(cfg, f64(inp.w_qkv), f64(inp.w_o), f64(inp.conv_seq),
                                         f64(inp.conv_chan))
        y, _, st = O.prefill_sequence(cfg, ow, f64(inp.x[0]), return_stages=True)
        # this rank's heads of the attention output and its columns of W_o
        sl = kv_group_slice(w.n_heads, w.n_kv_heads, w.dl, world, rank)
        _, wo_local, _, _ = shard_weights(inp.w_qkv, inp.w_o, inp.conv_seq, inp.conv_chan,
                                          w.n_heads, w.n_kv_heads, w.dl, world, rank)
        share = torch.from_numpy(st["o"][:, sl.q_rows.start:sl.q_rows.stop] @ f64(wo_local).T)
        total = tp_all_reduce(share.clone(), world)
        out[rank] = torch.tensor([float(np.max(np.abs(total.numpy() - y))),
                                  float(np.max(np.abs(share.numpy() - y)))], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_two_rank_shares_sum_to_the_layer():
    world = 2
    out = torch.zeros(world, 2, dtype=torch.float64).share_memory_()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert (out[:, 0] < 1e-12).all(), out            # the all-reduced shares are the layer
    assert (out[:, 1] > 1e-3).all(), out             # one share alone is not
