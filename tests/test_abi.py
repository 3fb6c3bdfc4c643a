"""The C-ABI library loads without a GPU, exports every symbol the header
declares, and its host-side validation rejects bad arguments before any
device work.  No compute call is made here."""
import ctypes as C
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "qlora_nf4.h")


@pytest.fixture(scope="module")
def L():
    from tests.conftest import ensure_built
    ensure_built()
    from bit_nf4_quantized_pack_b200 import _lib
    return _lib


def header_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    declared = header_functions()
    assert len(declared) >= 13
    assert sorted(L.SIGNATURES) == declared
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (qlora_\w+)", out))
    assert set(declared) <= exported
    for name in declared:
        assert getattr(L.lib, name) is not None


def test_library_needs_no_libcuda_to_load(L):
    out = subprocess.run(["ldd", L.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_status_strings_and_counts(L):
    lib = L.lib
    assert lib.qlora_abi_version() == L.ABI_VERSION
    for code in range(7):
        assert lib.qlora_status_str(code)
    assert lib.qlora_status_str(99) == b"unknown status"
    assert lib.qlora_last_cuda_error()          # a static string, never NULL
    assert lib.qlora_nf4_n1(1) == 1 and lib.qlora_nf4_n1(64) == 1 and lib.qlora_nf4_n1(65) == 2
    assert lib.qlora_nf4_n2(64 * 256) == 1 and lib.qlora_nf4_n2(64 * 256 + 1) == 2
    assert lib.qlora_nf4_n1(0) == 0 and lib.qlora_nf4_n2(0) == 0


def test_workspace_sizes(L):
    lib = L.lib
    assert lib.qlora_nf4_quantize_workspace_size(1000, 0) == 0
    assert lib.qlora_nf4_quantize_workspace_size(64 * 100, 1) >= 2048 + 4 * 100
    # neither forward path needs a workspace when r % 8 == 0: both add their K
    # splits inside a thread-block cluster
    assert lib.qlora_linear_fwd_workspace_size(4096, 4096, 4096, 16) == 0
    assert lib.qlora_linear_fwd_workspace_size(4, 4096, 4096, 16) == 0
    assert lib.qlora_linear_fwd_workspace_size(4, 4096, 4096, 12) >= 4096 * 16 * 2
    # backward: dZ (M x r bf16)
    assert lib.qlora_linear_bwd_workspace_size(4096, 4096, 4096, 16) >= 4096 * 16 * 2
    # unsupported shapes report 0
    assert lib.qlora_linear_fwd_workspace_size(16, 100, 64, 16) == 0
    assert lib.qlora_linear_fwd_workspace_size(16, 64, 64, 0) == 0
    assert lib.qlora_linear_fwd_workspace_size(16, 64, 64, 65) == 0
    # a rank that is not a multiple of 8: A (K x 16) and Zc (M x 16) padded copies
    assert lib.qlora_linear_fwd_workspace_size(4096, 4096, 4096, 12) >= (4096 + 4096) * 16 * 2
    assert lib.qlora_linear_bwd_workspace_size(4096, 4096, 4096, 3) >= (2 * 4096 + 4096) * 8 * 2


def _state(L, numel=128, dq=0, packed=4096):
    st = L.NF4StateC()
    st.numel, st.blocksize, st.double_quant, st.dq_blocksize, st.codebook = numel, 64, dq, 256, 0
    st.packed = packed
    st.absmax = 4096
    st.code8, st.s2, st.offset = 4096, 4096, 4096
    return st


def test_host_validation_rejects_before_device_work(L):
    lib, E = L.lib, L
    st = _state(L)
    fake = C.c_void_p(4096)
    # null W, misaligned W, bad dtype, empty tensor, bad blocksize
    assert lib.qlora_nf4_quantize(None, 0, C.byref(st), None, 0, None, None) == E.QLORA_ERR_INVALID_ARG
    assert lib.qlora_nf4_quantize(C.c_void_p(4097), 0, C.byref(st), None, 0, None, None) == E.QLORA_ERR_INVALID_ARG
    assert lib.qlora_nf4_quantize(fake, 7, C.byref(st), None, 0, None, None) == E.QLORA_ERR_INVALID_ARG
    bad = _state(L, numel=0)
    assert lib.qlora_nf4_quantize(fake, 0, C.byref(bad), None, 0, None, None) == E.QLORA_ERR_INVALID_ARG
    bad = _state(L)
    bad.blocksize = 128
    assert lib.qlora_nf4_quantize(fake, 0, C.byref(bad), None, 0, None, None) == E.QLORA_ERR_INVALID_ARG
    bad = _state(L, numel=1 << 39)
    assert lib.qlora_nf4_quantize(fake, 0, C.byref(bad), None, 0, None, None) == E.QLORA_ERR_UNSUPPORTED
    # double quant without workspace
    dq = _state(L, dq=1)
    assert lib.qlora_nf4_quantize(fake, 0, C.byref(dq), None, 0, None, None) == E.QLORA_ERR_INVALID_ARG
    assert lib.qlora_nf4_quantize(None, 0, None, None, 0, None, None) == E.QLORA_ERR_INVALID_ARG
    assert lib.qlora_nf4_dequantize(C.byref(st), None, None, None) == E.QLORA_ERR_INVALID_ARG
    # linear: unsupported shapes and rank
    w = _state(L, numel=64 * 64)
    args = [fake, C.byref(w), fake, fake, 1.0, fake, fake, fake, 1 << 20, None, None]
    assert lib.qlora_linear_fwd(8, 100, 64, 16, *args) == E.QLORA_ERR_UNSUPPORTED
    assert lib.qlora_linear_fwd(8, 64, 64, 0, *args) == E.QLORA_ERR_UNSUPPORTED
    assert lib.qlora_linear_fwd(8, 64, 64, 65, *args) == E.QLORA_ERR_UNSUPPORTED
    assert lib.qlora_linear_fwd(8, 64, 64, 72, *args) == E.QLORA_ERR_UNSUPPORTED
    assert lib.qlora_linear_fwd(0, 64, 64, 16, *args) == E.QLORA_ERR_INVALID_ARG
    assert lib.qlora_linear_fwd(8, 128, 64, 16, *args) == E.QLORA_ERR_INVALID_ARG   # numel != K*N
    args_nan = [fake, C.byref(w), fake, fake, float("nan"), fake, fake, fake, 1 << 20, None, None]
    assert lib.qlora_linear_fwd(8, 64, 64, 16, *args_nan) == E.QLORA_ERR_INVALID_ARG
    args_small_ws = [fake, C.byref(w), fake, fake, 1.0, fake, fake, fake, 16, None, None]
    # a rank that needs a padded copy of A in the workspace
    assert lib.qlora_linear_fwd(8, 64, 64, 12, *args_small_ws) == E.QLORA_ERR_INVALID_ARG
    bargs = [fake, fake, fake, C.byref(w), fake, fake, 1.0, fake, fake, None, None, 0, None, None]
    assert lib.qlora_linear_bwd(8, 64, 64, 16, *bargs) == E.QLORA_ERR_INVALID_ARG  # null dB
    assert lib.qlora_status_sync(None, None, None) == E.QLORA_ERR_INVALID_ARG
    assert lib.qlora_status_clear(None, None) == E.QLORA_ERR_INVALID_ARG


def test_product_path_has_no_fallback():
    """The binding loads the CUDA library or fails; it never imports the oracle."""
    pkg = os.path.join(ROOT, "bit_nf4_quantized_pack_b200")
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            src = open(os.path.join(pkg, f), encoding="utf-8").read()
            assert not re.search(r"^\s*(from|import)\s+oracle\b", src, flags=re.M), f
            assert "import_module(\"oracle" not in src and "__import__(\"oracle" not in src, f


def test_selftest_validation(L):
    """The bounded-wait self-test rejects bad limits and a null status word on
    the host, before any launch."""
    lib = L.lib
    fake = C.c_void_p(256)   # never dereferenced: validation fails first
    assert lib.qlora_selftest_bounded_wait(0, fake, None) == 1
    assert lib.qlora_selftest_bounded_wait(20_000_000_000, fake, None) == 1
    assert lib.qlora_selftest_bounded_wait(1000, None, None) == 1


def test_workspace_cache_is_per_stream_and_bounded(L, monkeypatch):
    """Host logic of the binding's workspace cache, on CPU tensors with a
    stand-in for the current stream: one buffer per (purpose, device, stream),
    grown when too small, and at most `limit` buffers kept."""
    import torch

    import bit_nf4_quantized_pack_b200 as q

    class FakeStream:
        def __init__(self, h):
            self.cuda_stream = h

    cur = {"h": 1, "cap": False}
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: FakeStream(cur["h"]))
    monkeypatch.setattr(torch.cuda, "is_current_stream_capturing", lambda: cur["cap"])
    cache = q._WorkspaceCache(limit=3)
    a = cache.get(("b", "cpu"), 1000, "cpu")
    assert a is cache.get(("b", "cpu"), 900, "cpu")          # reused on the same stream
    cur["h"] = 2
    b = cache.get(("b", "cpu"), 1000, "cpu")
    assert b is not a                                          # another stream, another buffer
    c = cache.get(("b", "cpu"), 5000, "cpu")
    assert c is not b and c.numel() >= 5000                     # grown
    assert cache.get(("b", "cpu"), 0, "cpu") is None
    for h in (3, 4, 5):
        cur["h"] = h
        cache.get(("f", "cpu"), 10, "cpu")
    assert len(cache._bufs) == 3                               # bounded, oldest dropped
    cur["h"] = 1
    assert cache.get(("b", "cpu"), 1000, "cpu") is not a       # stream 1's buffer was evicted
    # while the stream captures a CUDA graph: no allocation, no growth, and the
    # buffer handed out stays referenced after a later call replaces it
    cur["h"] = 7
    d = cache.get(("b", "cpu"), 1000, "cpu")
    cur["cap"] = True
    assert cache.get(("b", "cpu"), 800, "cpu") is d
    with pytest.raises(RuntimeError):
        cache.get(("b", "cpu"), 4000, "cpu")
    with pytest.raises(RuntimeError):
        cache.get(("q", "cpu"), 10, "cpu")
    cur["cap"] = False
    e = cache.get(("b", "cpu"), 4000, "cpu")
    assert e is not d and any(x is d for x in cache._captured)
