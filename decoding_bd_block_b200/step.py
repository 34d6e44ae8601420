"""Device-side set-up of one decoding step, driven through the C ABI.

A thin host harness: it allocates the caller-owned buffers with torch (the
KV cache, inputs, outputs and workspaces), fills the block-level cache with
``bd_cache_commit`` and runs the step as ``bd_block_attn`` followed by
``bd_confidence_select``.  All arithmetic happens in libbd's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import bd
from .workloads import BLOCK, StepConfig


def to_device(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Upload fp32 data, or bf16 bit patterns (uint16) as a bfloat16 tensor."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


class BlockCacheState:
    """KV cache of a batch, filled with the pre-RoPE prefix K/V of a workload."""

    def __init__(self, cfg: StepConfig, prefix_len, prefix_k=None, prefix_v=None,
                 extra_blocks: int = 2, device="cuda", page_table=None, n_pages=None):
        self.cfg = cfg
        self.shape = bd.make_shape(cfg.n_heads_q, cfg.n_heads_kv, cfg.head_dim, cfg.dtype,
                                   cfg.rope_theta)
        P = np.asarray(prefix_len)
        self.max_blocks = int(P.max()) // BLOCK + extra_blocks
        self.cache = bd.KVCache(self.shape, cfg.batch, self.max_blocks, device,
                                n_pages=n_pages, page_table=page_table)
        if prefix_k is not None:
            for s in range(cfg.batch):
                nb = int(P[s]) // BLOCK
                if nb == 0:
                    continue
                k = to_device(prefix_k[s], cfg.dtype, device)
                v = to_device(prefix_v[s], cfg.dtype, device)
                bd.bd_cache_commit(self.cache, k, v, [s], nb)


def _host_array(a: np.ndarray, dtype: str) -> np.ndarray:
    """The bytes a tensor of `dtype` holds for array a (bf16 as bit patterns)."""
    if dtype == "bf16":
        return np.ascontiguousarray(a).view(np.uint16)
    return np.ascontiguousarray(a, dtype=np.float32)


class DecodeStep:
    """Buffers of one denoising step: block attention + confidence select.

    The step's per-step inputs (q, k_blk, v_blk, h, h_prev, the mask bits
    and the block's tokens) and its results (the tokens again and the
    unmask bits) are views of one device arena, laid out as
    [inputs ... | tokens | unmask], so that a serving loop moves a step's
    inputs with one host-to-device copy (``arena[:in_bytes]``) and reads the
    result back with one device-to-host copy (``arena[out_off:]``).
    """

    def __init__(self, cfg: StepConfig, attn_in: dict | None, sel_in: dict | None,
                 device="cuda", cache: BlockCacheState | None = None):
        self.cfg = cfg
        B, dt = cfg.batch, cfg.dtype
        self.attn = attn_in is not None
        self.sel = sel_in is not None
        self.active_only = False  # score only the unmask rule's candidates
        tdt = torch_dtype(dt)
        parts = []  # (name, host array, torch dtype, shape)
        if self.attn:
            for name in ("q", "k_blk", "v_blk"):
                parts.append((name, _host_array(attn_in[name], dt), tdt, attn_in[name].shape))
        if self.sel:
            self.masked_host = np.ascontiguousarray(sel_in["masked_bits"], dtype=np.uint32)
            parts.append(("h", _host_array(sel_in["h"], dt), tdt, sel_in["h"].shape))
            parts.append(("h_prev", _host_array(sel_in["h_prev"], dt), tdt, sel_in["h_prev"].shape))
            parts.append(("masked", self.masked_host.view(np.int32), torch.int32, (B,)))
            parts.append(("tokens", np.ascontiguousarray(sel_in["tokens"], np.int32), torch.int32,
                          (B, BLOCK)))
            parts.append(("unmask", np.zeros(B, np.int32), torch.int32, (B,)))
        offs, off = [], 0
        for _, arr, _, _ in parts:
            offs.append(off)
            off = (off + arr.nbytes + 255) // 256 * 256
        host = np.zeros(max(off, 256), dtype=np.uint8)
        for (_, arr, _, _), o in zip(parts, offs):
            host[o:o + arr.nbytes] = np.frombuffer(arr.tobytes(), dtype=np.uint8)
        self.arena = torch.from_numpy(host).to(device)
        for (name, arr, tdtype, shape), o in zip(parts, offs):
            setattr(self, name, self.arena[o:o + arr.nbytes].view(tdtype).view(*shape))
        names = [p[0] for p in parts]
        self.in_bytes = offs[names.index("unmask")] if self.sel else off
        self.out_off = offs[names.index("tokens")] if self.sel else off
        if self.attn:
            self.cstate = cache or BlockCacheState(cfg, attn_in["prefix_len"], attn_in["prefix_k"],
                                                   attn_in["prefix_v"], device=device)
            self.out = torch.empty_like(self.q)
            n = bd.bd_block_attn_workspace_size(self.cstate.cache)
            self.attn_ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
        if self.sel:
            self.W = to_device(sel_in["W"], dt, device)
            self.tokens_in = self.tokens.clone()
            self.pmax = torch.empty((B, BLOCK), dtype=torch.float32, device=device)
            self.argmax = torch.empty((B, BLOCK), dtype=torch.int32, device=device)
            n = bd.bd_confidence_select_workspace_size(dt, B, cfg.hidden, cfg.vocab)
            self.sel_ws = torch.zeros(n, dtype=torch.uint8, device=device)  # header must start zero
            self.n_scored = int(sum(bin(int(b)).count("1") for b in self.masked_host))

    def run_attn(self, stream=None):
        bd.bd_block_attn(self.cstate.cache, self.q, self.k_blk, self.v_blk, self.out,
                         self.attn_ws, stream=stream)

    def run_select(self, tau: float, sub_block: int, stream=None, outputs=True,
                   active_only=None):
        """active_only (default: the step's `active_only`) scores only the
        unmask rule's candidates (bd_confidence_select_active)."""
        cfg = self.cfg
        if active_only is None:
            active_only = self.active_only
        fn = bd.bd_confidence_select_active if active_only else bd.bd_confidence_select
        fn(cfg.dtype, cfg.batch, cfg.hidden, cfg.vocab, self.h, self.h_prev, self.W, self.masked,
           tau, sub_block, self.tokens, self.unmask, self.pmax if outputs else None,
           self.argmax if outputs else None, self.sel_ws, stream=stream)

    def run(self, tau: float, sub_block: int, stream=None, active_only=None):
        if self.attn:
            self.run_attn(stream)
        if self.sel:
            self.run_select(tau, sub_block, stream, active_only=active_only)

    def capture(self, tau: float, sub_block: int, parts=("attn", "select"), active_only=None):
        """Record the step's launches (the same C-ABI calls) into CUDA graphs.

        Returns {part: torch.cuda.CUDAGraph}; replaying a graph re-runs that
        call's kernels on the current buffers without host-side launch cost.
        Part "step" holds both calls in one graph, so the select call's first
        kernel is chained to the attention call's last one.  The cache must
        not grow while the graphs are in use (its block counts size the
        attention launch).
        """
        graphs = {}
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.run(tau, sub_block, active_only=active_only)  # warm the launch path outside capture
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        for part in parts:
            if (part == "attn" and not self.attn) or (part == "select" and not self.sel):
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                if part == "attn":
                    self.run_attn(side)
                elif part == "select":
                    self.run_select(tau, sub_block, side, active_only=active_only)
                else:
                    self.run(tau, sub_block, side, active_only=active_only)
            graphs[part] = g
        torch.cuda.synchronize()
        return graphs
