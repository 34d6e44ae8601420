"""Seeded synthetic workloads for the block-diffusion decoding step.

This module only draws random inputs: it holds none of the step's arithmetic
(no RoPE, attention, softmax or selection).  Both the fp64 oracle (tests) and
the CUDA path (tests, bench) consume exactly the arrays built here, so the two
sides see bit-identical inputs.

Shapes follow the Qwen2.5-1.5B / 7B block-decoding workloads that the
Fast-dLLM v2 notes (papernotes.org, "Fast-dLLM v2", experiment section) name;
the concrete head counts, hidden sizes, vocab sizes, prefix lengths and value
distributions are the workload definitions below.  No dataset, prompt or
trained weight is involved: every tensor is drawn from a seeded PCG64 stream.

Conventions
-----------
* bf16 tensors are returned as ``uint16`` bit patterns, rounded from float32
  to nearest-even once, here.  fp32 tensors are ``float32``.
* ``masked_bits[s]`` bit ``i`` set <=> position ``i`` of sequence ``s``'s
  current 32-token block is still [MASK].
* ``tokens[s, i]`` holds the id decoded so far, ``MASK_TOKEN`` where masked.
* prefix K/V are pre-RoPE projections, ``[P_s, Hkv, d]`` per sequence; the
  library applies RoPE when a block is committed to the cache.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

BLOCK = 32            # D: tokens per block (the training block size)
MASK_TOKEN = -1       # placeholder id held by still-masked positions

_CHUNK = 1 << 22


# ----------------------------------------------------------------------------
# low-level seeded draws (threaded, chunked: each chunk has its own child
# stream of one SeedSequence, so the values do not depend on thread count)
# ----------------------------------------------------------------------------
def _to_bf16_bits_inplace(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (round to nearest, ties to even)."""
    b = x.view(np.uint32)
    t = b >> 16
    t &= 1
    t += 0x7FFF
    b += t
    b >>= 16
    return b.astype(np.uint16)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).copy()
    return _to_bf16_bits_inplace(x.reshape(-1)).reshape(x.shape)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def normal(seed, shape, std: float = 1.0, dtype: str = "bf16",
           threads: int = 8) -> np.ndarray:
    """N(0, std^2) samples of ``shape``: bf16 bits (uint16) or float32."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    nch = max(1, (n + _CHUNK - 1) // _CHUNK)
    kids = np.random.SeedSequence(seed).spawn(nch)
    out = np.empty(n, np.uint16 if dtype == "bf16" else np.float32)

    def work(i):
        lo = i * _CHUNK
        hi = min(n, lo + _CHUNK)
        x = np.random.Generator(np.random.PCG64(kids[i])).standard_normal(
            hi - lo, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[lo:hi] = _to_bf16_bits_inplace(x) if dtype == "bf16" else x

    if nch == 1:
        work(0)
    else:
        with ThreadPoolExecutor(min(threads, nch)) as ex:
            list(ex.map(work, range(nch)))
    return out.reshape(shape)


def as_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    return f32_from_bf16_bits(a) if dtype == "bf16" else a


# ----------------------------------------------------------------------------
# workload definitions
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class StepConfig:
    """One decoding-step workload (attention over the block cache + unmask)."""
    name: str
    dtype: str                     # "f32" or "bf16": storage of q/k/v/cache/h/W
    batch: int
    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    rope_theta: float
    prefix_tokens: tuple = ()      # fixed P per sequence (multiple of 32) ...
    prefix_range: tuple = ()       # ... or (lo, hi): P ~ U{lo..hi} rounded to 32
    n_masked: int = 0              # fixed masked count per sequence ...
    masked_range: tuple = ()       # ... or (lo, hi): count ~ U{lo..hi}
    hidden: int = 0                # H (0: attention-only workload)
    vocab: int = 0                 # V
    w_std: float = 0.02            # LM-head weight std
    s_max: float = 30.0            # planted-peak strength s ~ U(0, s_max)
    taus: tuple = (0.9,)
    sub_block: int = 8
    seed: int = 0

    @property
    def group(self) -> int:
        return self.n_heads_q // self.n_heads_kv


@dataclasses.dataclass(frozen=True)
class MaskAttnConfig:
    """Training-forward complementary-mask attention workload."""
    name: str
    samples: int
    views: int
    L: int
    block: int
    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    seed: int = 0
    dtype: str = "bf16"

    @property
    def n_seqs(self) -> int:
        return self.samples * self.views


# Tiny single step in fp32.  The weight scale reads "N(0, 0.02)" as variance
# 0.02 (std sqrt(0.02)): only then do planted peaks give p_max across (0, 1)
# at H=256, V=2048.  TINY_F32_LITERAL keeps std 0.02 (every p_max small, so
# every sequence takes the single-most-confident fallback).
TINY_F32 = StepConfig(
    name="tiny_f32", dtype="f32", batch=1, n_heads_q=4, n_heads_kv=2,
    head_dim=64, rope_theta=1e4, prefix_tokens=(96,), n_masked=20,
    hidden=256, vocab=2048, w_std=float(np.sqrt(0.02)), s_max=12.0,
    taus=(0.9, 1.0), sub_block=8, seed=1001)

TINY_F32_LITERAL = dataclasses.replace(
    TINY_F32, name="tiny_f32_std0.02", w_std=0.02, seed=1011)

QWEN15B_STEP = StepConfig(
    name="qwen2.5-1.5b_step", dtype="bf16", batch=1, n_heads_q=12,
    n_heads_kv=2, head_dim=128, rope_theta=1e6, prefix_tokens=(512,),
    n_masked=24, hidden=1536, vocab=151936, w_std=0.02, s_max=30.0,
    taus=(0.9,), sub_block=8, seed=1002)

# RoPE base of the 7B workload is not given with it; Qwen2.5-7B uses 1e6.
QWEN7B_RAGGED = StepConfig(
    name="qwen2.5-7b_ragged16", dtype="bf16", batch=16, n_heads_q=28,
    n_heads_kv=4, head_dim=128, rope_theta=1e6, prefix_range=(256, 2048),
    masked_range=(1, 32), hidden=3584, vocab=152064, w_std=0.02, s_max=30.0,
    taus=(0.9,), sub_block=8, seed=1003)

LONGCTX_ATTN = StepConfig(
    name="longctx_attn_b8_p32768", dtype="bf16", batch=8, n_heads_q=28,
    n_heads_kv=4, head_dim=128, rope_theta=1e6, prefix_tokens=(32768,) * 8,
    seed=1004)

MASK_ATTN = MaskAttnConfig(
    name="mask_attn_n8x2_L2048", samples=8, views=2, L=2048, block=32,
    n_heads_q=12, n_heads_kv=2, head_dim=128, seed=1005)

@dataclasses.dataclass(frozen=True)
class CeConfig:
    """Training masked-token cross-entropy workload: samples x views
    sequences of L positions; view 0 masks m ~ Bernoulli(mask_p) per
    position, view 1 the complement."""
    name: str
    samples: int
    views: int
    L: int
    hidden: int
    vocab: int
    w_std: float = 0.02
    s_max: float = 30.0
    mask_p: float = 0.5
    seed: int = 0
    dtype: str = "bf16"

    @property
    def n_seqs(self) -> int:
        return self.samples * self.views


# The training batch of the mask-attention workload (8 samples x 2 views,
# L = 2048) with the LM head of the 1.5B-shaped decoding workload.
MASKED_CE = CeConfig(name="masked_ce_n8x2_L2048", samples=8, views=2, L=2048, hidden=1536,
                     vocab=151936, seed=1006)

STEP_CONFIGS = {c.name: c for c in
                (TINY_F32, TINY_F32_LITERAL, QWEN15B_STEP, QWEN7B_RAGGED,
                 LONGCTX_ATTN)}


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------
def _stream(cfg_seed: int, tag: int):
    return [cfg_seed, tag]


def prefix_lengths(cfg: StepConfig) -> np.ndarray:
    """P_s per sequence, each a multiple of 32."""
    if cfg.prefix_tokens:
        p = np.array(cfg.prefix_tokens if len(cfg.prefix_tokens) == cfg.batch
                     else cfg.prefix_tokens * cfg.batch, dtype=np.int64)
    else:
        rng = np.random.Generator(np.random.PCG64(_stream(cfg.seed, 1)))
        lo, hi = cfg.prefix_range
        u = rng.integers(lo, hi + 1, size=cfg.batch)
        p = (np.rint(u / BLOCK) * BLOCK).astype(np.int64)
        p = np.clip(p, lo, hi)
    assert np.all(p % BLOCK == 0)
    return p


def make_attn_inputs(cfg: StepConfig, prefix=None):
    """Pre-RoPE prefix K/V per sequence and the current block's q, k, v.

    Returns dict with ``prefix_k``/``prefix_v``: lists of ``[P_s, Hkv, d]``,
    ``q``: ``[B, 32, Hq, d]``, ``k_blk``/``v_blk``: ``[B, 32, Hkv, d]``.
    All ~ N(0, 1).
    """
    P = prefix_lengths(cfg) if prefix is None else np.asarray(prefix)
    B, Hq, Hkv, d = cfg.batch, cfg.n_heads_q, cfg.n_heads_kv, cfg.head_dim
    pk, pv = [], []
    for s in range(B):
        pk.append(normal(_stream(cfg.seed, 100 + 2 * s), (int(P[s]), Hkv, d), 1.0, cfg.dtype))
        pv.append(normal(_stream(cfg.seed, 101 + 2 * s), (int(P[s]), Hkv, d), 1.0, cfg.dtype))
    q = normal(_stream(cfg.seed, 10), (B, BLOCK, Hq, d), 1.0, cfg.dtype)
    k = normal(_stream(cfg.seed, 11), (B, BLOCK, Hkv, d), 1.0, cfg.dtype)
    v = normal(_stream(cfg.seed, 12), (B, BLOCK, Hkv, d), 1.0, cfg.dtype)
    return dict(prefix_len=P, prefix_k=pk, prefix_v=pv, q=q, k_blk=k, v_blk=v)


def make_masked_bits(cfg: StepConfig) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(_stream(cfg.seed, 2)))
    bits = np.zeros(cfg.batch, dtype=np.uint32)
    for s in range(cfg.batch):
        if cfg.masked_range:
            m = int(rng.integers(cfg.masked_range[0], cfg.masked_range[1] + 1))
        else:
            m = cfg.n_masked
        idx = rng.choice(BLOCK, size=m, replace=False)
        bits[s] = np.uint32(sum(1 << int(i) for i in idx))
    return bits


def make_lm_weight(cfg: StepConfig) -> np.ndarray:
    """LM head W: ``[V, H]`` row-major, ~ N(0, w_std^2)."""
    return normal(_stream(cfg.seed, 20), (cfg.vocab, cfg.hidden), cfg.w_std, cfg.dtype)


def make_hidden(cfg: StepConfig, W: np.ndarray):
    """Planted-peak hidden rows: h = s * W[t] / ||W[t]|| + N(0, I).

    Returns ``h`` ``[B, 32, H]`` (rows of the current block) and ``h_prev``
    ``[B, H]`` (last row of the previous block), each row with its own
    planted token t ~ U{0..V-1} and strength s ~ U(0, s_max).
    """
    B, H, V = cfg.batch, cfg.hidden, cfg.vocab
    rng = np.random.Generator(np.random.PCG64(_stream(cfg.seed, 3)))
    t = rng.integers(0, V, size=(B, BLOCK + 1))
    s = rng.uniform(0.0, cfg.s_max, size=(B, BLOCK + 1)).astype(np.float32)
    noise = normal(_stream(cfg.seed, 21), (B, BLOCK + 1, H), 1.0, "f32")
    Wt = as_f32(W[t.reshape(-1)], cfg.dtype).reshape(B, BLOCK + 1, H)
    nrm = np.sqrt((Wt.astype(np.float64) ** 2).sum(-1, keepdims=True)).astype(np.float32)
    rows = (s[..., None] * Wt / nrm + noise).astype(np.float32)
    if cfg.dtype == "bf16":
        rows = bf16_bits_from_f32(rows)
    # row 0 of the drawn 33 is h_prev; rows 1..32 are the block's rows
    return dict(h=np.ascontiguousarray(rows[:, 1:]),
                h_prev=np.ascontiguousarray(rows[:, 0]),
                planted_token=t, planted_strength=s)


def make_tokens(cfg: StepConfig, masked_bits: np.ndarray) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(_stream(cfg.seed, 4)))
    tok = rng.integers(0, max(cfg.vocab, 1), size=(cfg.batch, BLOCK)).astype(np.int32)
    for s in range(cfg.batch):
        for i in range(BLOCK):
            if (int(masked_bits[s]) >> i) & 1:
                tok[s, i] = MASK_TOKEN
    return tok


def make_select_inputs(cfg: StepConfig, W=None):
    W = make_lm_weight(cfg) if W is None else W
    bits = make_masked_bits(cfg)
    hid = make_hidden(cfg, W)
    return dict(W=W, masked_bits=bits, tokens=make_tokens(cfg, bits), **hid)


def make_mask_attn_inputs(cfg: MaskAttnConfig):
    """q, k, v ``[N, 2L, H, d]`` for N = samples x views.

    Index ``0..L-1`` is the noisy stream x_t and ``L..2L-1`` the clean stream
    x_0.  The clean half of a sample is shared by both of its views.  View 0
    uses mask m ~ Bernoulli(0.5) per position, view 1 its complement; at a
    masked position the noisy row is a fresh N(0, 1) draw (standing in for
    the projections of the [MASK] embedding), elsewhere it equals the clean
    row.  Returns the tensors and the per-sample mask ``m`` ``[samples, L]``.
    """
    S, V, L = cfg.samples, cfg.views, cfg.L
    Hq, Hkv, d = cfg.n_heads_q, cfg.n_heads_kv, cfg.head_dim
    rng = np.random.Generator(np.random.PCG64(_stream(cfg.seed, 5)))
    m = (rng.random((S, L)) < 0.5)
    out = {}
    for name, H, tag in (("q", Hq, 30), ("k", Hkv, 40), ("v", Hkv, 50)):
        clean = normal(_stream(cfg.seed, tag), (S, L, H, d), 1.0, cfg.dtype)
        mask_rows = normal(_stream(cfg.seed, tag + 1), (S, V, L, H, d), 1.0, cfg.dtype)
        t = np.empty((S, V, 2 * L, H, d), dtype=clean.dtype)
        for smp in range(S):
            for view in range(V):
                mv = m[smp] if view % 2 == 0 else ~m[smp]
                t[smp, view, L:] = clean[smp]
                t[smp, view, :L] = np.where(mv[:, None, None], mask_rows[smp, view], clean[smp])
        out[name] = t.reshape(S * V, 2 * L, H, d)
    out["m"] = m
    return out


def make_ce_inputs(cfg: CeConfig):
    """h ``[N, L, H]``, W ``[V, H]``, targets ``[N, L]``, masked bits
    ``[N, L/32]`` for N = samples x views.

    Targets x_0 ~ U{0..V-1} per sample (shared by its views).  Row i-1 of
    every sequence is a planted peak toward the target of position i,
    h = s * W[y] / ||W[y]|| + N(0, I) with s ~ U(0, s_max), so the losses
    range from about log V down to near 0.  View 0 masks position i with
    probability mask_p, view 1 the complement.
    """
    S, V_, L, H, V = cfg.samples, cfg.views, cfg.L, cfg.hidden, cfg.vocab
    N = S * V_
    W = normal(_stream(cfg.seed, 60), (V, H), cfg.w_std, cfg.dtype)
    rng = np.random.Generator(np.random.PCG64(_stream(cfg.seed, 61)))
    y = rng.integers(0, V, size=(S, L)).astype(np.int32)
    m = rng.random((S, L)) < cfg.mask_p
    strength = rng.uniform(0.0, cfg.s_max, size=(N, L)).astype(np.float32)
    targets = np.repeat(y, V_, axis=0)                       # [N, L]
    # row i-1 points at the target of position i (the last row at a random token)
    nxt = np.concatenate([targets[:, 1:], rng.integers(0, V, size=(N, 1)).astype(np.int32)], 1)
    h = np.empty((N, L, H), dtype=np.uint16 if cfg.dtype == "bf16" else np.float32)
    chunk = max(1, (1 << 22) // H)
    flat_t = nxt.reshape(-1)
    flat_s = strength.reshape(-1)
    out = h.reshape(N * L, H)
    for r0 in range(0, N * L, chunk):
        r1 = min(N * L, r0 + chunk)
        Wt = as_f32(W[flat_t[r0:r1]], cfg.dtype)
        nrm = np.sqrt((Wt.astype(np.float64) ** 2).sum(-1, keepdims=True)).astype(np.float32)
        noise = normal([cfg.seed, 62, r0], (r1 - r0, H), 1.0, "f32")
        rows = (flat_s[r0:r1, None] * Wt / nrm + noise).astype(np.float32)
        out[r0:r1] = bf16_bits_from_f32(rows) if cfg.dtype == "bf16" else rows
    mv = np.empty((N, L), dtype=bool)
    for smp in range(S):
        for view in range(V_):
            mv[smp * V_ + view] = m[smp] if view % 2 == 0 else ~m[smp]
    bits = np.zeros((N, L // BLOCK), dtype=np.uint32)
    for k in range(BLOCK):
        bits |= (mv[:, k::BLOCK].astype(np.uint32) << np.uint32(k))
    return dict(h=h, W=W, targets=targets, masked_bits=bits, mask=mv)
