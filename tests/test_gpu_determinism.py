"""Repeatability of the CUDA path: the same inputs give bitwise the same outputs, call after
call.  Every reduction in the kernels has a fixed order, so a difference between two runs
points at a race (a read before the write it depends on is visible), which a tolerance test
can pass by luck.  Decode runs several steps, so the kernels overlap their launches
(programmatic dependent launch) the way a serving loop drives them.
"""
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


def _fresh_cache(layer, inp, w, max_seq):
    cache = layer.new_cache(w.batch, max_seq)
    cache.k[:, :, :w.seq] = inp.k_cache.cuda()
    cache.v[:, :, :w.seq] = inp.v_cache.cuda()
    cache.conv_state.copy_(inp.conv_state.cuda())
    cache.vshift_state.copy_(inp.vshift_state.cuda())
    cache.lengths.copy_(inp.lengths.cuda())
    return cache


def test_prefill_bitwise_repeatable(cuda_lib):
    w = W.WORKLOADS["ccgqa_prefill_16k"].with_(batch=1, seq=2048 + 77)
    inp = W.make_inputs(w, seed=4)
    layer = cuda_lib.CCALayer.from_workload(w, inp)
    x = inp.x.cuda()
    ys = [layer.prefill(x).clone() for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


def test_decode_bitwise_repeatable(cuda_lib):
    w = W.WORKLOADS["ccgqa_decode_8k"].with_(seq=3000)
    inp = W.make_inputs(w, seed=6)
    layer = cuda_lib.CCALayer.from_workload(w, inp)
    g = torch.Generator("cpu").manual_seed(1)
    xs = [torch.randn(w.batch, w.d_model, generator=g).to(torch.bfloat16).cuda() for _ in range(4)]
    runs = []
    for _ in range(3):
        cache = _fresh_cache(layer, inp, w, w.seq + 16)
        ys = [layer.decode(x, cache).clone() for x in xs]     # four steps back to back
        torch.cuda.synchronize()
        cuda_lib.cca_cache_check(cache.struct)
        runs.append((ys, cache.k[:, :, w.seq:w.seq + 4].clone(), cache.conv_state.clone(),
                     cache.vshift_state.clone(), cache.lengths.clone()))
    for ys, k, cs, vs, ln in runs[1:]:
        for a, b in zip(ys, runs[0][0]):
            assert torch.equal(a, b)
        assert torch.equal(k, runs[0][1])
        assert torch.equal(cs, runs[0][2]) and torch.equal(vs, runs[0][3])
        assert torch.equal(ln, runs[0][4])
