"""The C-ABI library loads and exports every symbol include/bd.h declares.

No GPU needed: only symbol lookup and host-side argument validation (which
returns before any CUDA call) are exercised.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "bd.h")).read()
    return sorted(set(re.findall(r"^BD_API\s+[\w\s\*]+?\b(bd_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from decoding_bd_block_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_checks_build_exports_the_same_symbols():
    from decoding_bd_block_b200 import build
    build.build()
    checks = ctypes.CDLL(build.LIB_CHECKS)
    for n in _declared():
        assert hasattr(checks, n), n


def test_binding_covers_header():
    from decoding_bd_block_b200 import bd
    assert sorted(bd.EXPORTED) == _declared()


def test_status_strings(lib):
    lib.bd_status_string.restype = ctypes.c_char_p
    assert lib.bd_status_string(0) == b"ok"
    assert lib.bd_status_string(-3) == b"KV cache capacity exceeded"


def test_host_validation_without_gpu():
    from decoding_bd_block_b200 import bd
    sz = ctypes.c_size_t(0)
    f = bd._lib.bd_confidence_select_workspace_size
    assert f(1, 0, 1536, 151936, ctypes.byref(sz)) == -1      # batch 0
    assert f(7, 1, 1536, 151936, ctypes.byref(sz)) == -2      # unknown dtype
    assert f(1, 16, 3584, 152064, ctypes.byref(sz)) == 0 and sz.value > 0
    # null pointers / bad sub_block are rejected before any launch
    st = bd._lib.bd_confidence_select(1, 1, 1536, 151936, None, None, None, None, 0.9, 8,
                                      None, None, None, None, None, 0, None)
    assert st == -1
    shape = bd.make_shape(12, 2, 128, "bf16")
    assert bd._lib.bd_block_mask_attn(ctypes.byref(shape), None, None, None, None, 1, 64, 32,
                                      None) == -1
    bad = bd.make_shape(12, 5, 128, "bf16")
    assert bd._lib.bd_block_mask_attn(ctypes.byref(bad), 1, 1, 1, 1, 1, 64, 32, None) == -1
    d96 = bd.make_shape(12, 2, 96, "bf16")
    assert bd._lib.bd_block_mask_attn(ctypes.byref(d96), 1, 1, 1, 1, 1, 64, 32, None) == -2
    assert bd._lib.bd_block_mask_attn(ctypes.byref(shape), 1, 1, 1, 1, 1, 48, 32, None) == -1


@pytest.mark.parametrize("hidden,vocab,fits,refused", [(3584, 152064, 24, 25), (1536, 151936, 48, 49)])
def test_noalloc_size_limit_boundaries(hidden, vocab, fits, refused):
    # bd_confidence_select_noalloc refuses a step whose scratch (the
    # bd_confidence_select workspace) exceeds its fixed array: in bf16 on a
    # 148-SM B200 the last accepted batch is 24 at hidden 3584 and 48 at
    # hidden 1536 (the limits the header states).
    from decoding_bd_block_b200 import bd
    assert bd.bd_confidence_select_workspace_size("bf16", fits, hidden, vocab) \
        <= bd.BD_NOALLOC_SCRATCH_BYTES
    assert bd.bd_confidence_select_workspace_size("bf16", refused, hidden, vocab) \
        > bd.BD_NOALLOC_SCRATCH_BYTES
