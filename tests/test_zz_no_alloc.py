"""cca_decode_step_static: the decode step for callers that cannot allocate device memory
on their decode path (a serving loop with memory fixed at start-up, code running under an
allocator it does not control).  Its scratch is the library's built-in device array instead
of a caller workspace, so it must give the same result as cca_decode_step, call after call
(the array keeps the previous call's contents).

This file is collected last on purpose, and also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

import workloads as W
from gpu_helpers import BF16_TOL, bf16_err, f64

pytestmark = pytest.mark.gpu


def _load_cache(cache, inp, ctx):
    cache.k[:, :, :ctx] = inp.k_cache.cuda()
    cache.v[:, :, :ctx] = inp.v_cache.cuda()
    cache.conv_state.copy_(inp.conv_state.cuda())
    cache.vshift_state.copy_(inp.vshift_state.cuda())
    cache.lengths.copy_(inp.lengths.cuda())


def test_static_scratch_decode_matches_workspace_decode(cuda_lib):
    cls = cuda_lib
    w = W.WORKLOADS["ccgqa_decode_8k"]            # B=64, 8192 cached tokens, d~=32
    inp = W.make_inputs(w, seed=3)
    layer = cls.CCALayer.from_workload(w, inp)
    max_seq = w.seq + 16
    assert cls.cca_decode_workspace_size(layer.cfg, w.batch, max_seq) <= 8 << 20
    ref_cache = layer.new_cache(w.batch, max_seq)
    st_cache = layer.new_cache(w.batch, max_seq)
    _load_cache(ref_cache, inp, w.seq)
    _load_cache(st_cache, inp, w.seq)
    g = torch.Generator("cpu").manual_seed(11)
    for step in range(2):                           # two calls in a row
        x = torch.randn(w.batch, w.d_model, generator=g).to(torch.bfloat16).cuda()
        y_ref = layer.decode(x, ref_cache)
        y_st = torch.empty_like(x)
        cls.cca_decode_step_static(layer.cfg, layer.weights, x, y_st, st_cache.struct)
        torch.cuda.synchronize()
        cls.cca_cache_check(st_cache.struct)
        assert bf16_err(f64(y_st), f64(y_ref)) <= BF16_TOL, step
        L = w.seq + step
        assert bf16_err(f64(st_cache.k[:, :, L]).reshape(w.batch, -1),
                        f64(ref_cache.k[:, :, L]).reshape(w.batch, -1)) <= BF16_TOL
        assert st_cache.lengths.tolist() == ref_cache.lengths.tolist() == [L + 1] * w.batch


def test_static_scratch_rejects_oversized_steps(cuda_lib):
    cls = cuda_lib
    w = W.WORKLOADS["ccgqa_decode_8k"]
    inp = W.make_inputs(w.with_(seq=16), seed=0)
    layer = cls.CCALayer.from_workload(w.with_(seq=16), inp)
    B, max_seq = w.batch, w.seq + 16
    while cls.cca_decode_workspace_size(layer.cfg, B, max_seq) <= 8 << 20:
        B *= 2                                       # a step that needs more than 8 MiB
    fake = cls.cca_cache_t(16, 32, 48, 64, 80, 96, B, max_seq)     # rejected before any use
    x = torch.zeros(B, w.d_model, dtype=torch.bfloat16, device="cuda")
    y = torch.empty_like(x)
    rc = cls.load().cca_decode_step_static(ctypes.byref(layer.cfg), ctypes.byref(layer.weights),
                                           ctypes.c_void_p(x.data_ptr()),
                                           ctypes.c_void_p(y.data_ptr()), ctypes.byref(fake), None)
    assert rc == cls.CCA_ERR_WORKSPACE
    assert "scratch" in cls.cca_last_error_string()
