"""Tensor parallelism by key/value group on the GPU kernels, with the ranks emulated on one
device: each rank's share (tp_size / tp_rank in the config, the rank's weight slices) runs
through the C ABI in turn, nothing waits on another rank, and the shares are summed on the
host in float64 (the all-reduce).  The sum must match the oracle's whole layer, for prefill
and for decode steps over each rank's own cache."""
import numpy as np
import pytest
import torch

import oracle.cca_oracle as O
import workloads as W
from gpu_helpers import BF16_TOL, bf16_err, f64, oracle_config, oracle_weights

pytestmark = pytest.mark.gpu


def _rank_layers(cls, w, inp, tp):
    from compressed_latent_space_b200.tp import TPLayer
    return [TPLayer.from_workload(w, inp, tp, r) for r in range(tp)]


@pytest.mark.parametrize("tp", [2, 4])
@pytest.mark.parametrize("shape", [dict(d_model=512, n_heads=8, n_kv_heads=4, compression=2),
                                   dict(d_model=256, n_heads=4, n_kv_heads=4, compression=4)])
def test_tp_prefill_shares_sum_to_the_layer(cuda_lib, tp, shape):
    w = W.Workload("tp", 2, 150, **shape)
    inp = W.make_inputs(w, seed=9, conv_std=0.4)
    x = inp.x.cuda()
    total = None
    for layer in _rank_layers(cuda_lib, w, inp, tp):
        share = f64(layer.prefill_share(x))
        total = share if total is None else total + share
    torch.cuda.synchronize()
    ocfg = oracle_config(w)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))
    assert bf16_err(total, ref) <= BF16_TOL


@pytest.mark.parametrize("tp", [2, 4])
def test_tp_decode_over_rank_caches(cuda_lib, tp):
    """Prefill 30 tokens into each rank's cache, decode 6 more; every step's summed shares
    equal the oracle's output at that position."""
    w = W.Workload("tpd", 2, 36, 512, 8, 4, 2)
    inp = W.make_inputs(w, seed=2, conv_std=0.4)
    x = inp.x.cuda()
    layers = _rank_layers(cuda_lib, w, inp, tp)
    caches = [l.new_cache(w.batch, 48) for l in layers]
    for l, c in zip(layers, caches):
        l.prefill_share(x[:, :30].contiguous(), cache=c)
    ocfg = oracle_config(w)
    ref = O.prefill(ocfg, oracle_weights(ocfg, inp), f64(inp.x))
    for i in range(30, 36):
        total = None
        for l, c in zip(layers, caches):
            s = f64(l.decode_share(x[:, i].contiguous(), c))
            total = s if total is None else total + s
        torch.cuda.synchronize()
        assert bf16_err(total, ref[:, i]) <= BF16_TOL, i
    for c in caches:
        cuda_lib.cca_cache_check(c.struct)
        assert c.lengths.tolist() == [36] * w.batch
