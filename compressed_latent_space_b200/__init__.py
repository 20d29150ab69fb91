"""Python binding of libcca, the sm_100a implementation of CCA / CCGQA.

Every function here has the name of the C entry point it wraps (include/cca.h,
include/cca_stages.h) and only marshals arguments: torch tensors become device pointers,
the current CUDA stream is passed along, and a nonzero status raises CCAError with the
library's message.  All arithmetic happens in the CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_size_t, c_uint, c_void_p

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcca.so")

CCA_F32, CCA_BF16, CCA_F16 = 0, 1, 2
CCA_OK = 0
CCA_ERR_INVALID_ARG = -1
CCA_ERR_UNSUPPORTED = -2
CCA_ERR_WORKSPACE = -3
CCA_ERR_CACHE_FULL = -4
CCA_ERR_ALIGNMENT = -5
CCA_ERR_CUDA = -6
CCA_ERR_DEVICE = -7
CCA_ERR_RANGE = -8
CCA_QK_MEAN, CCA_VALUE_SHIFT, CCA_QK_NORM, CCA_ROPE = 1, 2, 4, 8
CCA_DEFAULT_FLAGS = 15
CCA_NO_CONV = 16


class CCAError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"CCA error {code}: {message}")
        self.code = code


class cca_config_t(ctypes.Structure):
    _fields_ = [("d_model", c_int), ("n_heads", c_int), ("n_kv_heads", c_int),
                ("compression", c_int), ("conv_kernel", c_int), ("chan_conv_kernel", c_int),
                ("rope_base", c_float), ("norm_eps", c_float), ("flags", c_uint), ("dtype", c_int),
                ("tp_size", c_int), ("tp_rank", c_int)]


class cca_weights_t(ctypes.Structure):
    _fields_ = [("w_qkv", c_void_p), ("w_o", c_void_p), ("conv_seq", c_void_p),
                ("conv_chan", c_void_p)]


class cca_cache_t(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("conv_state", c_void_p),
                ("vshift_state", c_void_p), ("lengths", c_void_p), ("status", c_void_p),
                ("batch", c_int), ("max_seq", c_int)]


_lib = None

_SIGS = {
    "cca_last_error_string": (ctypes.c_char_p, []),
    "cca_cache_alloc": (c_int, [POINTER(cca_config_t), c_int, c_int, c_void_p, POINTER(c_size_t),
                                POINTER(cca_cache_t), c_void_p]),
    "cca_prefill_workspace_size": (c_size_t, [POINTER(cca_config_t), c_int, c_int]),
    "cca_decode_workspace_size": (c_size_t, [POINTER(cca_config_t), c_int, c_int]),
    "cca_decode_kernel_count": (c_int, [POINTER(cca_config_t), c_int, c_int]),
    "cca_prefill_forward": (c_int, [POINTER(cca_config_t), POINTER(cca_weights_t), c_void_p, c_int,
                                    c_int, c_void_p, POINTER(cca_cache_t), c_void_p, c_size_t,
                                    c_void_p]),
    "cca_decode_step": (c_int, [POINTER(cca_config_t), POINTER(cca_weights_t), c_void_p, c_void_p,
                                POINTER(cca_cache_t), c_void_p, c_size_t, c_void_p]),
    "cca_cache_check": (c_int, [POINTER(cca_cache_t), c_void_p]),
    "cca_gemm_t": (c_int, [c_int, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                           c_void_p, c_void_p]),
    "cca_gemm": (c_int, [c_int, c_int, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int,
                         c_void_p, c_void_p]),
    "cca_stage_stencil": (c_int, [POINTER(cca_config_t), c_void_p, c_int, c_int, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                  c_size_t, c_void_p]),
    "cca_stage_stencil_workspace_size": (c_size_t, [POINTER(cca_config_t)]),
    "cca_stage_attention": (c_int, [POINTER(cca_config_t), c_void_p, c_void_p, c_void_p, c_int,
                                    c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "cca_workspace_status": (c_int, [c_void_p, c_void_p]),
    "cca_decode_step_static": (c_int, [POINTER(cca_config_t), POINTER(cca_weights_t), c_void_p,
                                       c_void_p, POINTER(cca_cache_t), c_void_p]),
    "cca_stage_wait_probe": (c_int, [ctypes.c_longlong, c_int, c_void_p, c_void_p]),
    "cca_stage_exp2_poly": (c_int, [c_void_p, c_void_p, c_int, c_void_p]),
    "cca_backward_workspace_size": (c_size_t, [POINTER(cca_config_t), c_int, c_int]),
    "cca_backward": (c_int, [POINTER(cca_config_t), POINTER(cca_weights_t), c_void_p, c_void_p,
                             c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                             c_void_p, c_size_t, c_void_p]),
    "cca_stage_timing": (c_int, [c_int]),
    "cca_stage_times": (c_int, [POINTER(ctypes.c_double), c_int, POINTER(c_int)]),
}


def load(path: str = LIB_PATH):
    """Loads libcca.so (built by ``python -m compressed_latent_space_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m compressed_latent_space_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(rc: int):
    if rc != CCA_OK:
        raise CCAError(rc, _lib.cca_last_error_string().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return c_void_p(stream)
    return c_void_p(stream.cuda_stream)


def make_config(d_model, n_heads, n_kv_heads, compression, conv_kernel=4, chan_conv_kernel=1,
                rope_base=10000.0, norm_eps=1e-6, flags=CCA_DEFAULT_FLAGS, dtype=CCA_BF16,
                tp_size=1, tp_rank=0):
    return cca_config_t(d_model, n_heads, n_kv_heads, compression, conv_kernel, chan_conv_kernel,
                        rope_base, norm_eps, flags, dtype, tp_size, tp_rank)


def make_weights(w_qkv, w_o, conv_seq, conv_chan) -> cca_weights_t:
    """Conv filters may be None for CCA_NO_CONV layers (passed as NULL)."""
    ptr = lambda t: None if t is None else t.data_ptr()
    return cca_weights_t(w_qkv.data_ptr(), w_o.data_ptr(), ptr(conv_seq), ptr(conv_chan))


def cca_last_error_string() -> str:
    return load().cca_last_error_string().decode()


def cca_prefill_workspace_size(cfg: cca_config_t, batch: int, seq: int) -> int:
    return load().cca_prefill_workspace_size(ctypes.byref(cfg), batch, seq)


def cca_decode_workspace_size(cfg: cca_config_t, batch: int, max_seq: int) -> int:
    return load().cca_decode_workspace_size(ctypes.byref(cfg), batch, max_seq)


def cca_decode_kernel_count(cfg: cca_config_t, batch: int, max_seq: int) -> int:
    return load().cca_decode_kernel_count(ctypes.byref(cfg), batch, max_seq)


def cca_cache_alloc(cfg: cca_config_t, batch: int, max_seq: int, buf=None, stream=None):
    """buf None: returns the byte count.  Else lays out the cache in ``buf`` (a uint8 CUDA
    tensor of at least that many bytes) and returns the cca_cache_t."""
    lib = load()
    nbytes = c_size_t(0 if buf is None else buf.numel() * buf.element_size())
    if buf is None:
        _check(lib.cca_cache_alloc(ctypes.byref(cfg), batch, max_seq, None, ctypes.byref(nbytes),
                                   None, None))
        return nbytes.value
    out = cca_cache_t()
    _check(lib.cca_cache_alloc(ctypes.byref(cfg), batch, max_seq, _ptr(buf), ctypes.byref(nbytes),
                               ctypes.byref(out), _stream(stream)))
    return out


def cca_prefill_forward(cfg, weights, x, batch, seq, y, cache=None, workspace=None, stream=None):
    lib = load()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.cca_prefill_forward(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), batch, seq,
                                   _ptr(y), ctypes.byref(cache) if cache is not None else None,
                                   _ptr(workspace), ws_bytes, _stream(stream)))


def cca_decode_step(cfg, weights, x, y, cache, workspace=None, stream=None):
    lib = load()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.cca_decode_step(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(y),
                               ctypes.byref(cache), _ptr(workspace), ws_bytes, _stream(stream)))


def cca_decode_step_static(cfg, weights, x, y, cache, stream=None):
    """Decode step whose scratch is the library's built-in device array (no workspace)."""
    _check(load().cca_decode_step_static(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(y),
                                         ctypes.byref(cache), _stream(stream)))


def cca_backward_workspace_size(cfg: cca_config_t, batch: int, seq: int) -> int:
    return load().cca_backward_workspace_size(ctypes.byref(cfg), batch, seq)


def cca_backward(cfg, weights, x, dy, batch, seq, dx, dw_qkv, dw_o, dconv_seq, dconv_chan,
                 workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().cca_backward(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(dy), batch,
                               seq, _ptr(dx), _ptr(dw_qkv), _ptr(dw_o), _ptr(dconv_seq),
                               _ptr(dconv_chan), _ptr(workspace), ws_bytes, _stream(stream)))


def cca_cache_check(cache, stream=None):
    _check(load().cca_cache_check(ctypes.byref(cache), _stream(stream)))


def cca_gemm_t(out_dtype, A, B, C, M, N, K, a_trans, b_trans, status=None, stream=None):
    _check(load().cca_gemm_t(out_dtype, _ptr(A), _ptr(B), _ptr(C), M, N, K, 1 if a_trans else 0,
                             1 if b_trans else 0, _ptr(status), _stream(stream)))


def cca_gemm(dtype, out_dtype, A, B, C, M, N, K, status=None, stream=None):
    _check(load().cca_gemm(dtype, out_dtype, _ptr(A), _ptr(B), _ptr(C), M, N, K, _ptr(status), _stream(stream)))


def cca_stage_stencil_workspace_size(cfg):
    return load().cca_stage_stencil_workspace_size(ctypes.byref(cfg))


def cca_stage_stencil(cfg, P, batch, seq, conv_seq, conv_chan, q, k, v, kv_stride, workspace,
                      stream=None):
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().cca_stage_stencil(ctypes.byref(cfg), _ptr(P), batch, seq, _ptr(conv_seq),
                                    _ptr(conv_chan), _ptr(q), _ptr(k), _ptr(v), kv_stride,
                                    _ptr(workspace), ws_bytes, _stream(stream)))


def cca_stage_attention(cfg, q, k, v, batch, seq, kv_stride, o, status=None, stream=None):
    _check(load().cca_stage_attention(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), batch, seq,
                                      kv_stride, _ptr(o), _ptr(status), _stream(stream)))


def cca_workspace_status(workspace, stream=None):
    _check(load().cca_workspace_status(_ptr(workspace), _stream(stream)))


def cca_stage_exp2_poly(x, y, stream=None):
    """y = 2^x (float32 device tensors of one even length) by the attention's FMA-pipe cubic."""
    _check(load().cca_stage_exp2_poly(_ptr(x), _ptr(y), int(x.numel()), _stream(stream)))


def cca_stage_wait_probe(limit_ns: int, arm: bool, status, stream=None):
    _check(load().cca_stage_wait_probe(int(limit_ns), 1 if arm else 0, _ptr(status),
                                       _stream(stream)))


def cca_stage_timing(enable: bool):
    _check(load().cca_stage_timing(1 if enable else 0))


def cca_stage_times(n: int = 16):
    """(per-kernel summed milliseconds, number of recorded calls)."""
    lib = load()
    ms = (ctypes.c_double * n)()
    calls = c_int(0)
    slots = lib.cca_stage_times(ms, n, ctypes.byref(calls))
    if slots < 0:
        _check(slots)
    return [ms[i] for i in range(min(slots, n))], calls.value


from .layer import CCALayer  # noqa: E402,F401
