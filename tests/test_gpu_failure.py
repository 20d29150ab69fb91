"""Failure detection and state handling on the GPU, without faulting it.

- A bounded mbarrier wait that can never complete gives up after its limit, reports the
  timeout through its status word, and the context stays usable.
- A bf16 output-projection weight beyond the float16 range (the up-projection of 16-bit
  layers runs on float16 operands) is reported, not silently changed.
- The decode state lives in one caller buffer: a copy taken mid-decode continues exactly
  like the original (checkpoint / resume).
"""
import time

import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ms", [2, 20])
def test_bounded_wait_runs_out(cuda_lib, limit_ms):
    cls = cuda_lib
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    cls.cca_stage_wait_probe(limit_ms * 1_000_000, False, status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(status.item()) == 1                   # DEV_WAIT_TIMEOUT
    assert dt >= limit_ms * 1e-3 * 0.9, dt           # it did wait ...
    assert dt < 1.0, dt                              # ... and gave up at its own limit
    # the context is still usable: a small GEMM runs and is right
    A = torch.randn(128, 64, device="cuda").to(torch.bfloat16)
    B = torch.randn(256, 64, device="cuda").to(torch.bfloat16)
    C = torch.empty(128, 256, dtype=torch.float32, device="cuda")
    cls.cca_gemm(cls.CCA_BF16, cls.CCA_F32, A, B, C, 128, 256, 64)
    torch.cuda.synchronize()
    ref = A.double() @ B.double().T
    assert (C.double() - ref).abs().max().item() < 1e-3


def test_bounded_wait_completes_when_armed(cuda_lib):
    cls = cuda_lib
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cls.cca_stage_wait_probe(500_000_000, True, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_wait_probe_rejects_bad_limit(cuda_lib):
    cls = cuda_lib
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(cls.CCAError) as e:
        cls.cca_stage_wait_probe(10, False, status)
    assert e.value.code == cls.CCA_ERR_INVALID_ARG


def test_out_projection_weight_beyond_f16_is_reported(cuda_lib):
    """W_o of a bf16 layer is converted to float16 per call; an entry beyond 65504 sets
    CCA_ERR_RANGE in the workspace status instead of passing as infinity."""
    cls = cuda_lib
    w = W.Workload("wo", 1, 64, 256, 4, 2, 2)
    inp = W.make_inputs(w, seed=0)
    inp.w_o[3, 5] = 1.0e5                            # representable in bf16, not in f16
    layer = cls.CCALayer.from_workload(w, inp)
    layer.prefill(inp.x.cuda())
    with pytest.raises(cls.CCAError) as e:
        cls.cca_workspace_status(layer._ws)
    assert e.value.code == cls.CCA_ERR_RANGE
    inp2 = W.make_inputs(w, seed=0)                  # in range: clean status
    layer2 = cls.CCALayer.from_workload(w, inp2)
    layer2.prefill(inp2.x.cuda())
    cls.cca_workspace_status(layer2._ws)


def test_cache_copy_continues_identically(cuda_lib):
    """Save / restore of the decode state is a copy of the caller's cache buffer: after the
    copy, the original and the copy decode the same tokens to bitwise equal outputs."""
    cls = cuda_lib
    w = W.Workload("ckpt", 3, 40, 256, 4, 2, 2)
    inp = W.make_inputs(w, seed=5, conv_std=0.4)
    layer = cls.CCALayer.from_workload(w, inp)
    x = inp.x.cuda()
    cache = layer.new_cache(w.batch, 64)
    layer.prefill(x[:, :30].contiguous(), cache=cache)
    for i in range(30, 33):
        layer.decode(x[:, i].contiguous(), cache)
    copy = layer.new_cache(w.batch, 64)              # same layout (cca_cache_alloc), zeroed
    copy.buf.copy_(cache.buf)                        # the checkpoint
    for i in range(33, 40):
        ya = layer.decode(x[:, i].contiguous(), cache)
        yb = layer.decode(x[:, i].contiguous(), copy)
        torch.cuda.synchronize()
        assert torch.equal(ya, yb), i
    assert torch.equal(cache.buf, copy.buf)
    cls.cca_cache_check(cache.struct)
    cls.cca_cache_check(copy.struct)
