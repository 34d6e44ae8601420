"""Helpers shared by the GPU parity tests: oracle runs and comparisons."""
from __future__ import annotations

import numpy as np

import oracle as O

ATOL = {"f32": 1e-5, "bf16": 2e-2}     # attention max-abs bound per storage type
PMAX_ATOL = 1e-4                        # p_max agreement needed by the tau band


def oracle_block_attn(cfg, attn_in, seqs=None):
    """fp64 oracle of bd_block_attn for the listed sequences -> {s: [32, Hq, d]}."""
    seqs = range(cfg.batch) if seqs is None else seqs
    res = {}
    for s in seqs:
        c = O.OracleCache(1, cfg.n_heads_kv, cfg.head_dim, cfg.rope_theta)
        if attn_in["prefix_len"][s]:
            c.commit(0, O.widen(attn_in["prefix_k"][s], cfg.dtype),
                     O.widen(attn_in["prefix_v"][s], cfg.dtype))
        res[s] = O.block_attn_seq(c.k[0], c.v[0], O.widen(attn_in["q"][s], cfg.dtype),
                                  O.widen(attn_in["k_blk"][s], cfg.dtype),
                                  O.widen(attn_in["v_blk"][s], cfg.dtype), cfg.rope_theta)
    return res


def _bf16_round(x):
    """Round float64 values to bf16 (nearest even), as the kernel stores them."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_storage_block_attn(cfg, attn_in, seqs=None):
    """The oracle's block attention with the rotated q and keys rounded to bf16,
    i.e. the precision of the library's cache pages and rotated queries.  Used
    to separate storage rounding from the kernel's own arithmetic error."""
    seqs = range(cfg.batch) if seqs is None else seqs
    res = {}
    th = cfg.rope_theta
    for s in seqs:
        P = int(attn_in["prefix_len"][s])
        kc = O.rope(O.widen(attn_in["prefix_k"][s], cfg.dtype), np.arange(P), th)
        vc = O.widen(attn_in["prefix_v"][s], cfg.dtype)
        pos = np.arange(P, P + 32)
        q = _bf16_round(O.rope(O.widen(attn_in["q"][s], cfg.dtype), pos, th))
        kb = _bf16_round(O.rope(O.widen(attn_in["k_blk"][s], cfg.dtype), pos, th))
        keys = np.concatenate([_bf16_round(kc), kb])
        vals = np.concatenate([vc, O.widen(attn_in["v_blk"][s], cfg.dtype)])
        res[s] = O.attention(q, keys, vals)
    return res


def compare_select(ref, tokens, unmask, pmax, argmax, masked_bits):
    """Bit-exact decisions and tokens outside the ambiguity flags.

    Returns a dict of counts; raises AssertionError on a mismatch.
    """
    B = len(masked_bits)
    n_amb_dec = int(ref["decision_ambiguous"].sum())
    n_amb_tok = int(ref["token_ambiguous"].sum())
    checked = 0
    for s in range(B):
        bits = int(masked_bits[s])
        for i in range(32):
            if not (bits >> i) & 1:
                assert np.isnan(pmax[s, i]) and argmax[s, i] == -1, (s, i)
                continue
            assert abs(pmax[s, i] - ref["pmax"][s, i]) <= PMAX_ATOL, \
                (s, i, float(pmax[s, i]), float(ref["pmax"][s, i]))
            if not ref["token_ambiguous"][s, i]:
                assert argmax[s, i] == ref["argmax"][s, i], (s, i, argmax[s, i], ref["argmax"][s, i])
        if ref["decision_ambiguous"][s]:
            continue
        assert int(unmask[s]) == int(ref["unmask"][s]), (s, hex(int(unmask[s])), hex(int(ref["unmask"][s])))
        for i in range(32):
            if not ref["token_ambiguous"][s, i]:
                assert int(tokens[s, i]) == int(ref["tokens"][s, i]), (s, i)
        checked += 1
    return dict(sequences_checked=checked, decision_ambiguous=n_amb_dec,
                token_ambiguous=n_amb_tok)
