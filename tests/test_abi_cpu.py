"""The C-ABI library on a machine without a GPU: it loads, exports every
entry point the header declares, and rejects bad arguments on the host
before any CUDA call (so no device is needed)."""
import ctypes
import os
import re
import subprocess

import pytest

from paged_kv_cache_456_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "paged_attention.h")


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_456_b200 import build
    build.build()
    return ops.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_surface():
    assert declared_functions() == sorted(ops.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    nm = subprocess.run(["nm", "-D", "--defined-only", ops._LIB_PATH], capture_output=True,
                        text=True, check=True).stdout
    exported = set(re.findall(r" T (pa_\w+)", nm))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_header_compiles_as_c():
    src = '#include "paged_attention.h"\nint main(void){ return PA_OK + PA_BF16 + PA_ERRBIT_TIMEOUT - 17; }\n'
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                        "-x", "c", "-", "-o", os.devnull], input=src, text=True, capture_output=True)
    assert r.returncode == 0, r.stderr


def test_status_strings(lib):
    assert ops.status_str(ops.PA_OK) == "PA_OK"
    assert ops.status_str(ops.PA_ERR_WORKSPACE) == "PA_ERR_WORKSPACE"
    assert ops.status_str(99) == "PA_ERR_UNKNOWN"


P = ctypes.c_void_p


def decode_call(lib, **kw):
    args = dict(out=P(16), q=P(16), k=P(16), v=P(16), tab=P(16), lens=P(16), S=2, Hq=8, Hkv=2, D=128,
                bs=16, tmax=4, N=10, maxlen=64, scale=0.1, part=0, dt=ops.PA_BF16, ws=P(16),
                wsb=1 << 20, err=None, stream=None)
    args.update(kw)
    return lib.pa_decode(args["out"], args["q"], args["k"], args["v"], args["tab"], args["lens"],
                         args["S"], args["Hq"], args["Hkv"], args["D"], args["bs"], args["tmax"],
                         args["N"], args["maxlen"], args["scale"], args["part"], args["dt"],
                         args["ws"], args["wsb"], args["err"], args["stream"])


def test_decode_rejects_bad_arguments_on_the_host(lib):
    assert decode_call(lib, out=None) == ops.PA_ERR_INVALID_ARG
    assert decode_call(lib, lens=None) == ops.PA_ERR_INVALID_ARG
    assert decode_call(lib, Hq=7) == ops.PA_ERR_INVALID_ARG          # Hq % Hkv
    assert decode_call(lib, part=24) == ops.PA_ERR_INVALID_ARG       # not a multiple of 16
    assert decode_call(lib, S=-1) == ops.PA_ERR_INVALID_ARG
    assert decode_call(lib, maxlen=-5) == ops.PA_ERR_INVALID_ARG
    assert decode_call(lib, dt=7) == ops.PA_ERR_INVALID_ARG
    assert decode_call(lib, scale=float("nan")) == ops.PA_ERR_INVALID_ARG
    assert decode_call(lib, k=P(24)) == ops.PA_ERR_INVALID_ARG       # misaligned
    assert decode_call(lib, tmax=0) == ops.PA_ERR_INVALID_ARG
    assert decode_call(lib, D=96) == ops.PA_ERR_UNSUPPORTED
    assert decode_call(lib, Hq=6, Hkv=2) == ops.PA_ERR_UNSUPPORTED   # group 3
    assert decode_call(lib, bs=32) == ops.PA_ERR_UNSUPPORTED
    assert decode_call(lib, S=0) == ops.PA_OK                        # nothing to do


def test_fused_append_rejects_bad_arguments_on_the_host(lib):
    def call(key=P(16), value=P(16), S=2, Hq=8):
        return lib.pa_decode_append(P(16), P(16), key, value, P(16), P(16), P(16), P(16), S, Hq, 2,
                                    128, 16, 4, 10, 64, 0.1, 0, ops.PA_BF16, P(16), 1 << 20, None,
                                    None)
    assert call(key=None) == ops.PA_ERR_INVALID_ARG
    assert call(value=P(40)) == ops.PA_ERR_INVALID_ARG             # misaligned
    assert call(Hq=6) == ops.PA_ERR_UNSUPPORTED                    # group 3
    assert call(key=None, value=None, S=0) == ops.PA_OK            # nothing to do


def test_prefill_rejects_bad_arguments_on_the_host(lib):
    def call(qs=P(16), S=2, T=5, Hq=8):
        return lib.pa_prefill(P(16), P(16), P(16), P(16), P(16), P(16), qs, S, T, Hq, 2, 128, 16,
                              4, 10, 64, 0.1, 0, ops.PA_BF16, P(16), 1 << 20, None, None)
    assert call(qs=None) == ops.PA_ERR_INVALID_ARG
    assert call(S=0) == ops.PA_ERR_INVALID_ARG           # query rows but no sequence
    assert call(T=-1) == ops.PA_ERR_INVALID_ARG
    assert call(Hq=6) == ops.PA_ERR_UNSUPPORTED          # group 3
    assert call(qs=None, T=0) == ops.PA_OK               # nothing to do
    n = ctypes.c_size_t(0)
    assert lib.pa_prefill_workspace_size(2, 8, 8, 2, 128, 64, 0, ops.PA_BF16, None) == \
        ops.PA_ERR_INVALID_ARG
    assert lib.pa_prefill_workspace_size(2, -1, 8, 2, 128, 64, 0, ops.PA_BF16,
                                         ctypes.byref(n)) == ops.PA_ERR_INVALID_ARG


def test_workspace_queries_validate_first(lib):
    n = ctypes.c_size_t(0)
    assert lib.pa_decode_workspace_size(2, 8, 2, 96, 64, 0, ops.PA_BF16, ctypes.byref(n)) == \
        ops.PA_ERR_UNSUPPORTED
    assert lib.pa_decode_workspace_size(2, 8, 2, 128, 64, 0, ops.PA_BF16, None) == \
        ops.PA_ERR_INVALID_ARG
    assert lib.pa_decode_workspace_init(None, 16, None) == ops.PA_ERR_INVALID_ARG
    assert lib.pa_decode_workspace_init(None, 0, None) == ops.PA_OK


def test_cache_ops_reject_bad_arguments_on_the_host(lib):
    r = lib.pa_reshape_and_cache
    assert r(P(16), P(16), P(16), P(16), P(16), -1, 2, 64, 16, 10, ops.PA_BF16, None, None) == \
        ops.PA_ERR_INVALID_ARG
    assert r(P(16), P(16), P(16), P(16), P(16), 4, 2, 4, 16, 10, ops.PA_BF16, None, None) == \
        ops.PA_ERR_INVALID_ARG                                       # row of 8 bytes
    assert r(P(16), None, P(16), P(16), P(16), 4, 2, 64, 16, 10, ops.PA_BF16, None, None) == \
        ops.PA_ERR_INVALID_ARG
    assert r(P(16), P(16), P(16), P(16), None, 0, 2, 64, 16, 10, ops.PA_BF16, None, None) == ops.PA_OK
    c = lib.pa_copy_blocks
    assert c(P(16), P(16), P(16), -2, 2, 64, 16, 10, ops.PA_BF16, None, None) == ops.PA_ERR_INVALID_ARG
    assert c(P(16), P(8), P(16), 3, 2, 64, 16, 10, ops.PA_BF16, None, None) == ops.PA_ERR_INVALID_ARG
    assert c(P(16), P(16), None, 3, 2, 64, 16, 10, ops.PA_BF16, None, None) == ops.PA_ERR_INVALID_ARG
    assert c(None, None, None, 0, 2, 64, 16, 10, ops.PA_BF16, None, None) == ops.PA_OK


def test_binding_fails_loudly_without_the_library(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        ops.library(str(tmp_path / "nope.so"))
