"""Host-side checks of the C ABI that need no GPU: the library builds for sm_100a, loads,
exports every entry point the headers declare, and rejects bad arguments before any
launch (validation runs on the host)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from compressed_latent_space_b200 import build
    build.build()
    import compressed_latent_space_b200 as cls
    return cls.load()


def declared_symbols():
    names = []
    for h in ("cca.h", "cca_stages.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        names += re.findall(r"CCA_API\s+[\w\s\*]+?\b(cca_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 10, names
    so = os.path.join(ROOT, "compressed_latent_space_b200", "libcca.so")
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\b(cca_\w+)\b", out))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)
    # nothing but the declared entry points leaves the library
    assert exported == set(names), exported ^ set(names)


def cfg(**kw):
    import compressed_latent_space_b200 as cls
    base = dict(d_model=256, n_heads=4, n_kv_heads=4, compression=4, dtype=cls.CCA_F32)
    base.update(kw)
    return cls.make_config(**base)


def test_workspace_and_cache_sizes(lib):
    import compressed_latent_space_b200 as cls
    c = cfg(dtype=cls.CCA_BF16, d_model=2048, n_heads=16, n_kv_heads=4, compression=4)
    B, S = 2, 100
    M = B * S
    nq, nkv = 16 * 32, 4 * 32
    al = lambda x: (x + 255) // 256 * 256
    expect = 256 + al(2048 * nq * 2) + al((16 + 4) * 32 * 32 * 4) + al(M * (nq + 2 * nkv) * 4) + al(M * nq * 2) + 2 * al(M * nkv * 2) + al(M * nq * 2)
    assert cls.cca_prefill_workspace_size(c, B, S) == expect
    # cache: keys and values are n_kv wide per token: C * H/Hkv = 16x smaller than MHA's 2E
    nbytes = cls.cca_cache_alloc(c, 3, 1000)
    kv = 2 * al(3 * 4 * 1000 * 32 * 2)
    state = al(3 * 3 * (nq + nkv) * 4) + al(3 * (nkv // 2) * 4) + al(3 * 4) + 256
    assert nbytes == kv + state
    assert cls.cca_decode_workspace_size(c, 3, 1000) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(n_heads=3), -1),                      # d_model % n_heads
    (dict(n_kv_heads=3), -1),                   # n_heads % n_kv_heads
    (dict(compression=3), -1),                  # head width % C
    (dict(compression=8), -2),                  # d~ = 8 unsupported
    (dict(compression=1), -2),                  # d~ = 64? head width 64 / 1 = 64 -> ok below
    (dict(conv_kernel=0), -2),
    (dict(conv_kernel=9), -2),
    (dict(chan_conv_kernel=2), -2),
    (dict(dtype=7), -1),
    (dict(flags=32), -1),                       # unknown flag bit
    (dict(norm_eps=-1.0), -1),
])
def test_config_validation(lib, kw, code):
    import compressed_latent_space_b200 as cls
    c = cfg(**kw)
    if kw == dict(compression=1):
        assert cls.cca_prefill_workspace_size(c, 1, 8) > 0
        return
    assert cls.cca_prefill_workspace_size(c, 1, 8) == 0
    n = ctypes.c_size_t(0)
    rc = lib.cca_cache_alloc(ctypes.byref(c), 1, 8, None, ctypes.byref(n), None, None)
    assert rc == code
    assert cls.cca_last_error_string() != ""


def test_prefill_argument_errors_before_launch(lib):
    import compressed_latent_space_b200 as cls
    c = cfg()
    w = cls.cca_weights_t(16, 32, 48, 64)           # fake, aligned, never dereferenced
    ws = cls.cca_prefill_workspace_size(c, 1, 8)
    call = lambda **kw: lib.cca_prefill_forward(
        ctypes.byref(kw.get("cfg", c)), ctypes.byref(kw.get("w", w)), kw.get("x", 4096), 1,
        kw.get("seq", 8), kw.get("y", 8192), None, kw.get("ws", 1 << 20), kw.get("wsb", ws), None)
    assert call(w=cls.cca_weights_t(0, 32, 48, 64)) == cls.CCA_ERR_INVALID_ARG
    assert call(x=None) == cls.CCA_ERR_INVALID_ARG
    assert call(x=4100) == cls.CCA_ERR_ALIGNMENT
    assert call(wsb=ws - 1) == cls.CCA_ERR_WORKSPACE
    assert call(ws=None) == cls.CCA_ERR_WORKSPACE
    assert call(seq=-1) == cls.CCA_ERR_INVALID_ARG
    assert "workspace" in cls.cca_last_error_string() or "seq" in cls.cca_last_error_string()


def test_cache_full_rejected_on_host(lib):
    import compressed_latent_space_b200 as cls
    c = cfg()
    w = cls.cca_weights_t(16, 32, 48, 64)
    cache = cls.cca_cache_t(4096, 8192, 12288, 16384, 20480, 24576, 1, 4)
    ws = cls.cca_prefill_workspace_size(c, 1, 8)
    rc = lib.cca_prefill_forward(ctypes.byref(c), ctypes.byref(w), 4096, 1, 8, 8192,
                                 ctypes.byref(cache), 1 << 20, ws, None)
    assert rc == cls.CCA_ERR_CACHE_FULL


def test_injected_launch_failure(lib, monkeypatch):
    import compressed_latent_space_b200 as cls
    c = cfg()
    w = cls.cca_weights_t(16, 32, 48, 64)
    ws = cls.cca_prefill_workspace_size(c, 1, 8)
    monkeypatch.setenv("CCA_FAULT_INJECT", "launch")
    rc = lib.cca_prefill_forward(ctypes.byref(c), ctypes.byref(w), 4096, 1, 8, 8192, None,
                                 1 << 20, ws, None)
    assert rc == cls.CCA_ERR_CUDA
    assert "injected" in cls.cca_last_error_string()


def test_errors_are_thread_local(lib):
    import threading
    import compressed_latent_space_b200 as cls
    cls.cca_prefill_workspace_size(cfg(n_heads=3), 1, 8)      # sets an error on this thread
    mine = cls.cca_last_error_string()
    seen = []
    t = threading.Thread(target=lambda: seen.append(cls.cca_last_error_string()))
    t.start()
    t.join()
    assert mine != "" and seen == [""]


def test_latent_width_128_rules(lib):
    """d~ = 128 runs only in bfloat16 layers without the convolutions (CCA_NO_CONV), and
    prefill only: the cache and decode kernels take widths up to 64."""
    import compressed_latent_space_b200 as cls
    n = ctypes.c_size_t(0)
    f32 = cfg(d_model=512, n_heads=4, n_kv_heads=4, compression=1, flags=8 | 16)
    assert cls.cca_prefill_workspace_size(f32, 1, 8) == 0
    conv = cfg(d_model=512, n_heads=4, n_kv_heads=4, compression=1, dtype=cls.CCA_BF16)
    assert cls.cca_prefill_workspace_size(conv, 1, 8) == 0
    plain = cfg(d_model=512, n_heads=4, n_kv_heads=2, compression=1, dtype=cls.CCA_BF16,
                flags=8 | 16)
    assert cls.cca_prefill_workspace_size(plain, 1, 8) > 0
    assert lib.cca_cache_alloc(ctypes.byref(plain), 1, 8, None, ctypes.byref(n), None, None) == -2
    assert cls.cca_decode_workspace_size(plain, 1, 8) == 0
    # the same switch at d~ = 32 is prefill-only too
    small = cfg(flags=15 | 16, dtype=cls.CCA_BF16)
    assert cls.cca_prefill_workspace_size(small, 1, 8) > 0
    assert lib.cca_cache_alloc(ctypes.byref(small), 1, 8, None, ctypes.byref(n), None, None) == -2
