"""Backward pass on the GPU (cca_backward through the C ABI) against the float64 backward
oracle on the same bf16 inputs: dx, dW_qkv, dW_o and both conv filters' gradients.

Bound: the bf16 parity measure (max-abs error over the row's RMS, per row of each gradient
tensor, <= 2e-2), as for the forward."""
import numpy as np
import pytest
import torch

import oracle.cca_oracle_backward as OB
import workloads as W
from gpu_helpers import BF16_TOL, bf16_err, f64, oracle_config, oracle_weights

pytestmark = pytest.mark.gpu


def run_backward(cls, w, inp, dy, flags=None):
    layer = cls.CCALayer.from_workload(w, inp, flags=flags)
    grads = layer.backward(inp.x.cuda(), dy.cuda())
    torch.cuda.synchronize()
    cls.cca_workspace_status(layer._ws)
    return grads


def check(grads, ref, dl):
    dx, dwqkv, dwo, dcs, dcc = (f64(g) for g in grads)
    assert np.isfinite(dx).all() and np.isfinite(dwqkv).all()
    errs = dict(dx=bf16_err(dx, ref.dx), dw_qkv=bf16_err(dwqkv, ref.dw_qkv),
                dw_o=bf16_err(dwo, ref.dw_o), dconv_seq=bf16_err(dcs.reshape(1, -1), ref.dconv_seq.reshape(1, -1)),
                dconv_chan=bf16_err(dcc.reshape(-1, dl), ref.dconv_chan.reshape(-1, dl)))
    for k, e in errs.items():
        assert e <= BF16_TOL, (k, errs)


@pytest.mark.parametrize("flags", [15, 0, 14, 7])
@pytest.mark.parametrize("shape", [
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=2, seq=200),    # d~=32, G=2
    dict(d_model=512, n_heads=8, n_kv_heads=2, compression=1, seq=300),    # d~=64, G=4
    dict(d_model=256, n_heads=4, n_kv_heads=4, compression=4, seq=129),    # d~=16, CCA
])
def test_backward_matches_oracle(cuda_lib, shape, flags):
    shape = dict(shape)
    S = shape.pop("seq")
    w = W.Workload("bwd", 2, S, **shape)
    inp = W.make_inputs(w, seed=21, conv_std=0.4, identity_conv=True)
    g = torch.Generator("cpu").manual_seed(22)
    dy = torch.randn(w.batch, S, w.d_model, generator=g).to(torch.bfloat16)
    grads = run_backward(cuda_lib, w, inp, dy, flags)
    ocfg = oracle_config(w, flags)
    ref = OB.backward(ocfg, oracle_weights(ocfg, inp), f64(inp.x), f64(dy))
    check(grads, ref, w.dl)


@pytest.mark.parametrize("shape", [
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=2, seq=77, conv_kernel=1),
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=2, seq=150, conv_kernel=2),
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=2, seq=33, conv_kernel=6),
    dict(d_model=256, n_heads=4, n_kv_heads=2, compression=2, seq=260, conv_kernel=8),
    dict(d_model=512, n_heads=8, n_kv_heads=1, compression=2, seq=140),    # d~=32, G=8
    dict(d_model=256, n_heads=2, n_kv_heads=1, compression=2, seq=5),      # d~=64, G=2, S < tile
])
def test_backward_conv_widths_and_groups(cuda_lib, shape):
    """Conv widths 1..8 (the halo of the sequence conv's transpose across tiles and sequence
    starts), a group of 8 query heads, a sequence shorter than one tile."""
    shape = dict(shape)
    S = shape.pop("seq")
    w = W.Workload("bwd_kc", 2, S, **shape)
    inp = W.make_inputs(w, seed=31, conv_std=0.4, identity_conv=True)
    g = torch.Generator("cpu").manual_seed(32)
    dy = torch.randn(w.batch, S, w.d_model, generator=g).to(torch.bfloat16)
    grads = run_backward(cuda_lib, w, inp, dy)
    ocfg = oracle_config(w)
    ref = OB.backward(ocfg, oracle_weights(ocfg, inp), f64(inp.x), f64(dy))
    check(grads, ref, w.dl)


def test_backward_long_sequence(cuda_lib):
    """The 16k workload's heads (E=2048, 16 query / 4 kv heads, d~=64) over 1024 tokens: many
    key and query tiles per head, the conv widths' halo across tiles."""
    w = W.Workload("bwd_long", 1, 1024, 2048, 16, 4, 2)
    inp = W.make_inputs(w, seed=23, conv_std=0.3, identity_conv=True)
    g = torch.Generator("cpu").manual_seed(24)
    dy = torch.randn(1, 1024, 2048, generator=g).to(torch.bfloat16)
    grads = run_backward(cuda_lib, w, inp, dy)
    ocfg = oracle_config(w)
    ref = OB.backward(ocfg, oracle_weights(ocfg, inp), f64(inp.x), f64(dy))
    check(grads, ref, w.dl)


def test_backward_rejects_unsupported(cuda_lib):
    cls = cuda_lib
    assert cls.cca_backward_workspace_size(cls.make_config(256, 4, 4, 4, dtype=cls.CCA_F32), 1, 8) == 0
    assert cls.cca_backward_workspace_size(cls.make_config(512, 4, 4, 1, flags=8 | 16), 1, 8) == 0
    assert cls.cca_backward_workspace_size(cls.make_config(512, 8, 2, 1), 1, 8) > 0
