"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/kmip.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

from graph_transformer_sparse_kmip_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(kmip_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from graph_transformer_sparse_kmip_b200 import build
    build.build()
    return binding.load()


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert "kmip_attn_fwd" in declared and "kmip_attn_bwd" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(binding.EXPORTED) <= set(declared)


def test_forward_path_query(lib):
    assert binding.kmip_fwd_path(32, 15, binding.KMIP_BF16) == 1
    assert binding.kmip_fwd_path(16, 15, binding.KMIP_BF16) == 1
    assert binding.kmip_fwd_path(32, 15, binding.KMIP_F32) == 0
    assert binding.kmip_fwd_path(48, 15, binding.KMIP_BF16) == -1
    # Shapes whose lists, record buffers, Q tiles and two K stages fit in
    # shared memory take the tensor-core kernel; the rest the FMA kernel.
    for d, k, path in [(16, 64, 1), (32, 45, 1), (32, 64, 1), (64, 32, 1), (64, 45, 1),
                       (64, 64, 0), (128, 16, 1), (128, 17, 0), (128, 64, 0)]:
        assert binding.kmip_fwd_path(d, k, binding.KMIP_BF16) == path, (d, k)
    assert binding.kmip_fwd_path(32, 0, binding.KMIP_BF16) == -1


def test_error_strings_and_version(lib):
    for code, name in binding.STATUS_NAMES.items():
        assert binding.kmip_error_string(code).startswith(name)
    assert binding.kmip_error_string(99).startswith("KMIP_ERR_UNKNOWN")
    assert binding.kmip_version() >= 100


def _fwd(lib, N=16, H=1, d=32, k=4, scale=0.5, ptr=1 << 20, dtype=0, offsets=None, G=1):
    p = ctypes.c_void_p(ptr) if ptr else None
    return lib.kmip_attn_fwd(p, p, p, offsets, N, H, d, k, scale, p, p, p, None, G, dtype)


def test_argument_checks_need_no_device(lib):
    INVALID, UNSUP = 1, 2
    assert _fwd(lib, k=0) == INVALID
    assert _fwd(lib, N=-1) == INVALID
    assert _fwd(lib, scale=0.0) == INVALID
    assert _fwd(lib, scale=float("nan")) == INVALID
    assert _fwd(lib, scale=float("inf")) == INVALID
    assert _fwd(lib, dtype=7) == INVALID
    assert _fwd(lib, d=48) == UNSUP
    assert _fwd(lib, k=65) == UNSUP
    assert _fwd(lib, H=65) == UNSUP
    assert _fwd(lib, ptr=0) == INVALID                 # null tensors with N > 0
    assert _fwd(lib, ptr=(1 << 20) + 8) == INVALID     # not 16-byte aligned
    assert _fwd(lib, offsets=ctypes.c_void_p(1 << 20), G=0) == INVALID
    assert _fwd(lib, N=0, ptr=0) == 0                  # nothing to do
    p = None
    assert lib.kmip_attn_bwd(p, p, p, p, p, p, p, p, p, p, 8, 1, 32, 4, 0.5, 0) == INVALID
    assert lib.kmip_attn_bwd(p, p, p, p, p, p, p, p, p, p, 8, 1, 32, 0, 0.5, 0) == INVALID
    assert lib.kmip_attn_bwd(p, p, p, p, p, p, p, p, p, p, 0, 1, 32, 4, 0.5, 0) == 0
