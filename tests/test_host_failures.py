"""Failures injected on the host, at every entry point of the C ABI: null
pointers, bad shapes, unsupported dtypes, cache capacity overflow, repeated
sequences, workspace missing, too small or misaligned.  Each must come back
as its status code before anything is launched, so these run without a GPU
(the pointers passed are never dereferenced: a launch would fail here).
"""
import ctypes

import numpy as np
import pytest

OK, INVALID, UNSUPPORTED, CAPACITY, WORKSPACE, CUDA = 0, -1, -2, -3, -4, -5
FAKE = 1 << 20  # a 256-byte-aligned stand-in for a device pointer


@pytest.fixture(scope="module")
def bd():
    from decoding_bd_block_b200 import bd as _bd
    return _bd


def host_cache(bd, batch=2, max_blocks=4, n_blocks=(1, 3)):
    """A bd_kv_cache whose host mirrors are real arrays (the library reads
    them) and whose device pointers are stand-ins (never touched on error)."""
    table = np.arange(batch * max_blocks, dtype=np.int32).reshape(batch, max_blocks)
    nb = np.array(n_blocks, dtype=np.int32)
    c = bd.bd_kv_cache(pages=FAKE, n_pages=batch * max_blocks, page_table=FAKE,
                       page_table_host=table.ctypes.data, n_blocks=FAKE,
                       n_blocks_host=nb.ctypes.data, batch=batch, max_blocks=max_blocks)
    c._keep = (table, nb)
    return c


def test_cache_commit_failures(bd):
    lib = bd._lib
    sh = bd.make_shape(4, 2, 64, "f32")
    c = host_cache(bd)
    ids = (ctypes.c_int32 * 2)(0, 1)
    # sequence 1 holds 3 of 4 blocks: two more overflow its page table
    assert lib.bd_cache_commit(ctypes.byref(sh), ctypes.byref(c), FAKE, FAKE, ids, 2, 2, None) == CAPACITY
    dup = (ctypes.c_int32 * 2)(0, 0)
    assert lib.bd_cache_commit(ctypes.byref(sh), ctypes.byref(c), FAKE, FAKE, dup, 2, 1, None) == INVALID
    out = (ctypes.c_int32 * 1)(5)
    assert lib.bd_cache_commit(ctypes.byref(sh), ctypes.byref(c), FAKE, FAKE, out, 1, 1, None) == INVALID
    assert lib.bd_cache_commit(ctypes.byref(sh), ctypes.byref(c), None, FAKE, ids, 2, 1, None) == INVALID
    assert lib.bd_cache_commit(ctypes.byref(sh), ctypes.byref(c), FAKE, FAKE, ids, 2, 0, None) == INVALID
    assert lib.bd_cache_commit(ctypes.byref(sh), None, FAKE, FAKE, ids, 2, 1, None) == INVALID
    # the host block counts are untouched by a refused call
    assert list(c._keep[1]) == [1, 3]


def test_cache_page_table_out_of_range(bd):
    sh = bd.make_shape(4, 2, 64, "f32")
    c = host_cache(bd)
    c._keep[0][0, 1] = 99  # the page sequence 0's next block would be written to
    ids = (ctypes.c_int32 * 1)(0)
    assert bd._lib.bd_cache_commit(ctypes.byref(sh), ctypes.byref(c), FAKE, FAKE, ids, 1, 1,
                                   None) == INVALID


def test_shape_failures(bd):
    lib = bd._lib
    c = host_cache(bd)
    sz = ctypes.c_size_t(0)
    for bad, want in [(bd.make_shape(4, 3, 64, "f32"), INVALID),    # Hq % Hkv != 0
                      (bd.make_shape(4, 2, 96, "f32"), UNSUPPORTED),  # head_dim
                      (bd.make_shape(4, 2, 64, "f32", 0.0), INVALID)]:  # rope theta
        assert lib.bd_block_attn_workspace_size(ctypes.byref(bad), ctypes.byref(c),
                                                ctypes.byref(sz)) == want
    sh = bd.make_shape(4, 2, 64, "f32")
    sh.dtype = 9
    assert lib.bd_block_attn_workspace_size(ctypes.byref(sh), ctypes.byref(c),
                                            ctypes.byref(sz)) == UNSUPPORTED


def test_block_attn_workspace_and_alignment(bd):
    lib = bd._lib
    sh = bd.make_shape(4, 2, 64, "f32")
    c = host_cache(bd)
    sz = ctypes.c_size_t(0)
    assert lib.bd_block_attn_workspace_size(ctypes.byref(sh), ctypes.byref(c), ctypes.byref(sz)) == OK
    need = sz.value
    assert need > 0
    args = (ctypes.byref(sh), ctypes.byref(c), FAKE, FAKE, FAKE, FAKE)
    assert lib.bd_block_attn(*args, None, ctypes.c_size_t(need), None) == WORKSPACE
    assert lib.bd_block_attn(*args, FAKE, ctypes.c_size_t(need - 1), None) == WORKSPACE
    assert lib.bd_block_attn(*args, FAKE + 16, ctypes.c_size_t(need), None) == WORKSPACE
    assert lib.bd_block_attn(ctypes.byref(sh), ctypes.byref(c), FAKE + 4, FAKE, FAKE, FAKE, FAKE,
                             ctypes.c_size_t(need), None) == INVALID   # q not 16-byte aligned
    assert lib.bd_block_attn(ctypes.byref(sh), ctypes.byref(c), None, FAKE, FAKE, FAKE, FAKE,
                             ctypes.c_size_t(need), None) == INVALID


@pytest.mark.parametrize("name", ["bd_confidence_select", "bd_confidence_select_active"])
def test_select_failures(bd, name):
    lib = bd._lib
    f = getattr(lib, name)
    sz = ctypes.c_size_t(0)
    assert lib.bd_confidence_select_workspace_size(1, 2, 1536, 151936, ctypes.byref(sz)) == OK
    need = sz.value
    P = [FAKE] * 6  # h, h_prev, w, masked_bits, tokens, unmask

    def call(dtype=1, batch=2, hidden=1536, vocab=151936, tau=0.9, S=8, ptrs=P, ws=FAKE,
             ws_bytes=need):
        return f(dtype, batch, hidden, vocab, *ptrs[:4], ctypes.c_float(tau), S, *ptrs[4:],
                 None, None, ws, ctypes.c_size_t(ws_bytes), None)
    assert call(dtype=5) == UNSUPPORTED
    assert call(hidden=1540) == UNSUPPORTED          # hidden % 8
    assert call(batch=0) == INVALID
    assert call(S=7) == INVALID                      # sub_block must divide 32
    assert call(S=64) == INVALID
    assert call(tau=-0.5) == INVALID
    assert call(tau=float("nan")) == INVALID
    assert call(ptrs=[FAKE, FAKE, None, FAKE, FAKE, FAKE]) == INVALID
    assert call(ptrs=[FAKE + 8] + P[1:]) == INVALID  # h not 16-byte aligned
    assert call(ws=None) == WORKSPACE
    assert call(ws_bytes=need - 1) == WORKSPACE
    assert call(ws=FAKE + 128) == WORKSPACE          # workspace not 256-byte aligned


def test_noalloc_scratch_limit(bd):
    lib = bd._lib
    P = [FAKE] * 6
    # bf16 at hidden 3584: a batch above 24 needs more than the fixed scratch
    st = lib.bd_confidence_select_noalloc(1, 64, 3584, 152064, *P[:4], ctypes.c_float(0.9), 8,
                                          *P[4:], None, None, None)
    assert st == WORKSPACE


def test_masked_ce_failures(bd):
    lib = bd._lib
    sz = ctypes.c_size_t(0)
    assert lib.bd_masked_ce_workspace_size(1, 4, 1024, 264, 20001, ctypes.byref(sz)) == OK
    need = sz.value
    assert lib.bd_masked_ce_workspace_size(1, 4, 1000, 264, 20001, ctypes.byref(sz)) == UNSUPPORTED
    assert lib.bd_masked_ce_workspace_size(1, 4, 1024, 260, 20001, ctypes.byref(sz)) == UNSUPPORTED
    assert lib.bd_masked_ce_workspace_size(3, 4, 1024, 264, 20001, ctypes.byref(sz)) == UNSUPPORTED
    assert lib.bd_masked_ce_workspace_size(1, 0, 1024, 264, 20001, ctypes.byref(sz)) == INVALID

    def call(ws=FAKE, ws_bytes=need, h=FAKE, loss_sum=FAKE):
        return lib.bd_masked_ce(1, 4, 1024, 264, 20001, h, FAKE, FAKE, FAKE, None, loss_sum, None,
                                ws, ctypes.c_size_t(ws_bytes), None)
    assert call(h=None) == INVALID
    assert call(loss_sum=None) == INVALID
    assert call(h=FAKE + 2) == INVALID
    assert call(ws=None) == WORKSPACE
    assert call(ws_bytes=need - 1) == WORKSPACE


def test_status_of_a_refused_call_launches_nothing(bd):
    before = bd.bd_kernel_launches()
    sh = bd.make_shape(12, 2, 128, "bf16")
    assert bd._lib.bd_block_mask_attn(ctypes.byref(sh), None, FAKE, FAKE, FAKE, 1, 64, 32,
                                      None) == INVALID
    assert bd.bd_kernel_launches() == before


def test_mask_attn_views_failures(bd):
    # bd_block_mask_attn_views: views must be positive and divide n_seqs; the
    # other checks are those of bd_block_mask_attn.  Nothing is launched.
    before = bd.bd_kernel_launches()
    sh = bd.make_shape(12, 2, 128, "bf16")

    def call(q=FAKE, n_seqs=4, views=2, L=256, block=32, shape=sh):
        return bd._lib.bd_block_mask_attn_views(ctypes.byref(shape), q, FAKE, FAKE, FAKE, n_seqs,
                                                views, L, block, None)
    assert call(views=0) == INVALID
    assert call(views=-2) == INVALID
    assert call(views=3) == INVALID           # 4 entries are not whole groups of 3
    assert call(n_seqs=5) == INVALID
    assert call(q=None) == INVALID
    assert call(block=48) == INVALID          # block must divide L
    assert call(L=48, block=16) == UNSUPPORTED  # L must be a multiple of 32
    assert call(shape=bd.make_shape(12, 2, 96, "bf16")) == UNSUPPORTED
    assert bd.bd_kernel_launches() == before
