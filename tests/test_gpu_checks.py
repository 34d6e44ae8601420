"""Device-side index checks (the library built with BD_DEVICE_CHECKS).

The host validates every page id against the host mirror of the page table
before a launch, but the kernels read the device copy.  Here the device copy
is made to disagree (an out-of-range page id) while the host mirror stays
valid: the checks build must skip the access (no fault, finite outputs),
record the bad id, and report it once through bd_device_check_status.  The
normal build has no checks and says so."""
import ctypes
import dataclasses

import numpy as np
import pytest

from decoding_bd_block_b200 import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_normal_build_has_no_checks():
    from decoding_bd_block_b200 import bd
    with pytest.raises(bd.BdError) as e:
        bd.device_check_status()
    assert e.value.status == -2  # BD_ERR_UNSUPPORTED


@pytest.mark.parametrize("cfg", [
    dataclasses.replace(W.TINY_F32, batch=2, prefix_tokens=(96, 64), seed=601),   # CUDA-core attention
    dataclasses.replace(W.QWEN15B_STEP, batch=2, prefix_tokens=(256, 96), seed=602),  # tcgen05 attention
], ids=lambda c: c.dtype)
def test_bad_device_page_id_is_recorded_and_skipped(cfg):
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import BlockCacheState, to_device
    lib = bd.checks_library()
    bd.device_check_status(lib, reset=True)            # start clean
    a = W.make_attn_inputs(cfg)
    st = BlockCacheState(cfg, a["prefix_len"], a["prefix_k"], a["prefix_v"])
    c = st.cache
    bad = c.n_pages + 7
    c.page_table[0, 1] = bad                            # device copy only; host mirror valid
    q, kb, vb = (to_device(a[x], cfg.dtype) for x in ("q", "k_blk", "v_blk"))
    out = torch.full_like(q, float("nan"))
    n = ctypes.c_size_t(0)
    assert lib.bd_block_attn_workspace_size(ctypes.byref(c.shape), ctypes.byref(c.struct),
                                            ctypes.byref(n)) == 0
    ws = torch.zeros(max(n.value, 256), dtype=torch.uint8, device="cuda")
    st_code = lib.bd_block_attn(ctypes.byref(c.shape), ctypes.byref(c.struct), q.data_ptr(),
                                kb.data_ptr(), vb.data_ptr(), out.data_ptr(), ws.data_ptr(),
                                n.value, None)
    assert st_code == 0
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all())
    assert bd.device_check_status(lib, reset=True) == (1, bad)   # kCheckPageId, the bad id
    assert bd.device_check_status(lib, reset=True) == (0, 0)     # cleared
    # a valid table again: nothing recorded
    c.page_table[0, 1] = int(c.page_table_host[0, 1])
    assert lib.bd_block_attn(ctypes.byref(c.shape), ctypes.byref(c.struct), q.data_ptr(),
                             kb.data_ptr(), vb.data_ptr(), out.data_ptr(), ws.data_ptr(),
                             n.value, None) == 0
    torch.cuda.synchronize()
    assert bd.device_check_status(lib, reset=True) == (0, 0)


def test_commit_to_bad_device_page_writes_nothing():
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import BlockCacheState, to_device
    cfg = dataclasses.replace(W.TINY_F32, batch=1, prefix_tokens=(32,), seed=603)
    lib = bd.checks_library()
    bd.device_check_status(lib, reset=True)
    st = BlockCacheState(cfg, np.array([32]), None, None, extra_blocks=1)
    c = st.cache
    c.pages.fill_(3.0)
    before = c.pages.clone()
    c.page_table[0, 0] = -5                             # device copy only
    k = to_device(np.ones((1, 32, cfg.n_heads_kv, cfg.head_dim), np.float32), "f32")
    ids = np.array([0], dtype=np.int32)
    assert lib.bd_cache_commit(ctypes.byref(c.shape), ctypes.byref(c.struct), k.data_ptr(),
                               k.data_ptr(), ids.ctypes.data, 1, 1, None) == 0
    torch.cuda.synchronize()
    assert torch.equal(c.pages, before)                 # no page written
    assert bd.device_check_status(lib, reset=True) == (1, -5)
