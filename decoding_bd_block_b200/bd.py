"""Python binding of libbd (ctypes): argument marshalling only.

Every function here forwards to the C entry point of the same name in
``include/bd.h``; all computation happens in the CUDA kernels of
``libbd.so``.  Tensors are torch tensors on the current CUDA device (torch
provides device memory and streams); their data pointers are passed through.
Importing this module fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbd.so")

BD_BLOCK = 32
BD_F32, BD_BF16 = 0, 1
STATUS = {0: "BD_OK", -1: "BD_ERR_INVALID_ARG", -2: "BD_ERR_UNSUPPORTED",
          -3: "BD_ERR_CAPACITY", -4: "BD_ERR_WORKSPACE", -5: "BD_ERR_CUDA"}
EXPORTED = ("bd_cache_commit", "bd_block_attn_workspace_size", "bd_block_attn",
            "bd_confidence_select_workspace_size", "bd_confidence_select",
            "bd_block_mask_attn", "bd_status_string", "bd_last_cuda_error_string",
            "bd_kernel_launches", "bd_confidence_select_noalloc", "bd_confidence_select_active",
            "bd_masked_ce_workspace_size", "bd_masked_ce", "bd_eval_exp2",
            "bd_device_check_status", "bd_block_mask_attn_views")
BD_NOALLOC_SCRATCH_BYTES = 8 << 20

if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libbd.so not built ({_LIB_PATH}); run "
                      "`python -m decoding_bd_block_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)


class BdError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = _lib.bd_status_string(status).decode()
        if status == -5:
            msg += ": " + _lib.bd_last_cuda_error_string().decode()
        super().__init__(f"{fn} -> {STATUS.get(status, status)} ({msg})")


class bd_attn_shape(ctypes.Structure):
    _fields_ = [("n_heads_q", ctypes.c_int32), ("n_heads_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("rope_theta", ctypes.c_double)]


class bd_kv_cache(ctypes.Structure):
    _fields_ = [("pages", ctypes.c_void_p), ("n_pages", ctypes.c_int64),
                ("page_table", ctypes.c_void_p), ("page_table_host", ctypes.c_void_p),
                ("n_blocks", ctypes.c_void_p), ("n_blocks_host", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_blocks", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_SZ = ctypes.POINTER(ctypes.c_size_t)
_SIGS = {
    "bd_cache_commit": [ctypes.POINTER(bd_attn_shape), ctypes.POINTER(bd_kv_cache), _P, _P,
                        _P, _I, _I, _P],
    "bd_block_attn_workspace_size": [ctypes.POINTER(bd_attn_shape),
                                     ctypes.POINTER(bd_kv_cache), _SZ],
    "bd_block_attn": [ctypes.POINTER(bd_attn_shape), ctypes.POINTER(bd_kv_cache), _P, _P, _P,
                      _P, _P, ctypes.c_size_t, _P],
    "bd_confidence_select_workspace_size": [_I, _I, _I, _I, _SZ],
    "bd_confidence_select": [_I, _I, _I, _I, _P, _P, _P, _P, ctypes.c_float, _I, _P, _P, _P, _P,
                             _P, ctypes.c_size_t, _P],
    "bd_block_mask_attn": [ctypes.POINTER(bd_attn_shape), _P, _P, _P, _P, _I, _I, _I, _P],
    "bd_block_mask_attn_views": [ctypes.POINTER(bd_attn_shape), _P, _P, _P, _P, _I, _I, _I, _I,
                                 _P],
    "bd_confidence_select_noalloc": [_I, _I, _I, _I, _P, _P, _P, _P, ctypes.c_float, _I, _P, _P,
                                     _P, _P, _P],
    "bd_confidence_select_active": [_I, _I, _I, _I, _P, _P, _P, _P, ctypes.c_float, _I, _P, _P,
                                    _P, _P, _P, ctypes.c_size_t, _P],
    "bd_masked_ce_workspace_size": [_I, _I, _I, _I, _I, _SZ],
    "bd_masked_ce": [_I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "bd_eval_exp2": [_P, _P, _P, _P, _I, _P],
    "bd_device_check_status": [ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), _I],
}
for _name, _args in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int
_lib.bd_status_string.argtypes = [ctypes.c_int]
_lib.bd_status_string.restype = ctypes.c_char_p
_lib.bd_last_cuda_error_string.argtypes = []
_lib.bd_last_cuda_error_string.restype = ctypes.c_char_p
_lib.bd_kernel_launches.argtypes = []
_lib.bd_kernel_launches.restype = ctypes.c_longlong


def _check(fn, st):
    if st != 0:
        raise BdError(fn, st)


def _ptr(t):
    """Device pointer of a tensor (or an int / None passed through)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def dtype_code(dtype) -> int:
    s = str(dtype)
    if s in ("torch.bfloat16", "bf16", "bfloat16"):
        return BD_BF16
    if s in ("torch.float32", "f32", "float32"):
        return BD_F32
    raise ValueError(f"unsupported dtype {dtype}")


def make_shape(n_heads_q, n_heads_kv, head_dim, dtype, rope_theta=1e6) -> bd_attn_shape:
    return bd_attn_shape(n_heads_q, n_heads_kv, head_dim, dtype_code(dtype), float(rope_theta))


class KVCache:
    """Caller-owned block-level KV cache: page pool, page table, block counts.

    ``pages`` ``[n_pages, 2, Hkv, 32, d]``; ``page_table`` ``[batch,
    max_blocks]`` (device + host mirror, by default sequence s owns pages
    ``s*max_blocks ... (s+1)*max_blocks-1``); ``n_blocks`` ``[batch]``
    (device + host mirror, updated by :func:`bd_cache_commit`).
    """

    def __init__(self, shape: bd_attn_shape, batch: int, max_blocks: int, device="cuda",
                 n_pages=None, page_table=None):
        import torch
        self.shape = shape
        self.batch, self.max_blocks = int(batch), int(max_blocks)
        tdt = torch.bfloat16 if shape.dtype == BD_BF16 else torch.float32
        if page_table is None:
            page_table = np.arange(batch * max_blocks, dtype=np.int32).reshape(batch, max_blocks)
        self.page_table_host = np.ascontiguousarray(page_table, dtype=np.int32)
        self.n_pages = int(n_pages if n_pages is not None else self.page_table_host.max() + 1)
        self.pages = torch.empty((self.n_pages, 2, shape.n_heads_kv, BD_BLOCK, shape.head_dim),
                                 dtype=tdt, device=device)
        self.page_table = torch.from_numpy(self.page_table_host).to(device)
        self.n_blocks_host = np.zeros(batch, dtype=np.int32)
        self.n_blocks = torch.zeros(batch, dtype=torch.int32, device=device)
        self.struct = bd_kv_cache(
            self.pages.data_ptr(), self.n_pages, self.page_table.data_ptr(),
            self.page_table_host.ctypes.data, self.n_blocks.data_ptr(),
            self.n_blocks_host.ctypes.data, self.batch, self.max_blocks)


def bd_cache_commit(cache: KVCache, k, v, seq_ids, n_new_blocks: int = 1, stream=None):
    ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
    _check("bd_cache_commit", _lib.bd_cache_commit(
        ctypes.byref(cache.shape), ctypes.byref(cache.struct), _ptr(k), _ptr(v),
        ids.ctypes.data, len(ids), int(n_new_blocks), _stream(stream)))


def bd_block_attn_workspace_size(cache: KVCache) -> int:
    n = ctypes.c_size_t(0)
    _check("bd_block_attn_workspace_size", _lib.bd_block_attn_workspace_size(
        ctypes.byref(cache.shape), ctypes.byref(cache.struct), ctypes.byref(n)))
    return n.value


def bd_block_attn(cache: KVCache, q, k_blk, v_blk, out, workspace, workspace_bytes=None,
                  stream=None):
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("bd_block_attn", _lib.bd_block_attn(
        ctypes.byref(cache.shape), ctypes.byref(cache.struct), _ptr(q), _ptr(k_blk), _ptr(v_blk),
        _ptr(out), _ptr(workspace), int(wsb), _stream(stream)))


def bd_confidence_select_workspace_size(dtype, batch, hidden, vocab) -> int:
    n = ctypes.c_size_t(0)
    _check("bd_confidence_select_workspace_size", _lib.bd_confidence_select_workspace_size(
        dtype_code(dtype), int(batch), int(hidden), int(vocab), ctypes.byref(n)))
    return n.value


def bd_confidence_select(dtype, batch, hidden, vocab, h, h_prev, w_lm, masked_bits, tau,
                         sub_block, tokens, unmask_bits, pmax_out, argmax_out, workspace,
                         workspace_bytes=None, stream=None):
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("bd_confidence_select", _lib.bd_confidence_select(
        dtype_code(dtype), int(batch), int(hidden), int(vocab), _ptr(h), _ptr(h_prev),
        _ptr(w_lm), _ptr(masked_bits), float(tau), int(sub_block), _ptr(tokens),
        _ptr(unmask_bits), _ptr(pmax_out), _ptr(argmax_out), _ptr(workspace), int(wsb),
        _stream(stream)))


def bd_confidence_select_active(dtype, batch, hidden, vocab, h, h_prev, w_lm, masked_bits, tau,
                                sub_block, tokens, unmask_bits, pmax_out, argmax_out, workspace,
                                workspace_bytes=None, stream=None):
    """bd_confidence_select scoring only the unmask rule's candidates (the
    masked positions of the lowest sub-block that has one; see include/bd.h)."""
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("bd_confidence_select_active", _lib.bd_confidence_select_active(
        dtype_code(dtype), int(batch), int(hidden), int(vocab), _ptr(h), _ptr(h_prev),
        _ptr(w_lm), _ptr(masked_bits), float(tau), int(sub_block), _ptr(tokens),
        _ptr(unmask_bits), _ptr(pmax_out), _ptr(argmax_out), _ptr(workspace), int(wsb),
        _stream(stream)))


def bd_masked_ce_workspace_size(dtype, n_seqs, seq_len, hidden, vocab) -> int:
    n = ctypes.c_size_t(0)
    _check("bd_masked_ce_workspace_size", _lib.bd_masked_ce_workspace_size(
        dtype_code(dtype), int(n_seqs), int(seq_len), int(hidden), int(vocab), ctypes.byref(n)))
    return int(n.value)


def bd_masked_ce(dtype, n_seqs, seq_len, hidden, vocab, h, w_lm, targets, masked_bits, loss_out,
                 loss_sum, n_scored, workspace, workspace_bytes=None, stream=None):
    wsb = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("bd_masked_ce", _lib.bd_masked_ce(
        dtype_code(dtype), int(n_seqs), int(seq_len), int(hidden), int(vocab), _ptr(h),
        _ptr(w_lm), _ptr(targets), _ptr(masked_bits), _ptr(loss_out), _ptr(loss_sum),
        _ptr(n_scored), _ptr(workspace), int(wsb), _stream(stream)))


def bd_confidence_select_noalloc(dtype, batch, hidden, vocab, h, h_prev, w_lm, masked_bits, tau,
                                 sub_block, tokens, unmask_bits, pmax_out, argmax_out,
                                 stream=None):
    """bd_confidence_select for callers that cannot allocate a workspace: the
    library's own fixed device scratch is used instead (see include/bd.h)."""
    _check("bd_confidence_select_noalloc", _lib.bd_confidence_select_noalloc(
        dtype_code(dtype), int(batch), int(hidden), int(vocab), _ptr(h), _ptr(h_prev),
        _ptr(w_lm), _ptr(masked_bits), float(tau), int(sub_block), _ptr(tokens),
        _ptr(unmask_bits), _ptr(pmax_out), _ptr(argmax_out), _stream(stream)))


def bd_block_mask_attn(shape: bd_attn_shape, q, k, v, out, n_seqs, L, block, stream=None):
    _check("bd_block_mask_attn", _lib.bd_block_mask_attn(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out), int(n_seqs), int(L),
        int(block), _stream(stream)))


def bd_block_mask_attn_views(shape: bd_attn_shape, q, k, v, out, n_seqs, views, L, block,
                             stream=None):
    """bd_block_mask_attn for entries in groups of `views` views of one sample
    whose clean halves are equal (see include/bd.h)."""
    _check("bd_block_mask_attn_views", _lib.bd_block_mask_attn_views(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out), int(n_seqs), int(views),
        int(L), int(block), _stream(stream)))


def bd_eval_exp2(x, y_poly, y_pair, y_mufu, stream=None):
    """Diagnostic: the library's exponential approximations on the float32
    tensor x (see include/bd.h)."""
    _check("bd_eval_exp2", _lib.bd_eval_exp2(_ptr(x), _ptr(y_poly), _ptr(y_pair), _ptr(y_mufu),
                                             int(x.numel()), _stream(stream)))


def bd_kernel_launches() -> int:
    return int(_lib.bd_kernel_launches())


def device_check_status(lib=None, reset: bool = True):
    """(code, detail) of the device-side index checks of ``lib`` (default:
    this library, which has none and raises BD_ERR_UNSUPPORTED); see
    include/bd.h."""
    lib = _lib if lib is None else lib
    code, detail = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("bd_device_check_status", lib.bd_device_check_status(
        ctypes.byref(code), ctypes.byref(detail), 1 if reset else 0))
    return int(code.value), int(detail.value)


_CHECKS_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbd_checks.so")


def checks_library():
    """The same library built with the device-side index checks
    (libbd_checks.so): a ctypes handle whose entry points take the same
    arguments as this module's (marshal them with the helpers here)."""
    lib = ctypes.CDLL(_CHECKS_PATH)
    for name, args in _SIGS.items():
        getattr(lib, name).argtypes = args
    return lib


def raw_call(name, *args):
    """Call a C entry point with already-marshalled arguments; returns the status."""
    return getattr(_lib, name)(*args)


def library_path() -> str:
    return _LIB_PATH
