"""fp64 oracle of the block-diffusion decoding step (test infrastructure).

Plain, slow, float64 restatement of what the Fast-dLLM v2 decoding step
computes.  Inputs are the exact fp32 / bf16 values, widened to float64; no
intermediate rounding, no blocking or fusion beyond the definitions.  A matrix
product (``@``) is the only library primitive used as a step.

Sources (web pages on the method; cited by title and section):

* [N1] "Fast-dLLM v2: Efficient Block-Diffusion LLM" -- paper notes
  (papernotes.org, ICLR 2026), sections "Overall framework" (整体框架) and
  "Key designs" (关键设计) items 1-4.
* [N2] Fast-dLLM (v1) news article (senqingzn.com), section
  "1. Core techniques", item 2 "Confidence-aware parallel decoding".
* [N3] Fast-dLLM v2 abstract (hyper.ai, arXiv 2509.26328).
* [N4] "Fast-dLLM v2: 2.5x inference speedup" article (aigc.bar), sections
  "Core innovation" (block-internal parallel / block-causal) and
  "Acceleration engine" items 1 (hierarchical cache) and 2 (confidence-aware
  parallel decoding).

Readings taken where the pages are silent (each one is listed again, with
its justification, in the repository's design notes):

R1  RoPE: half-split pairing (j, j + d/2), inv_freq_j = theta^(-2j/d), angle
    = position * inv_freq_j (the Qwen2.5 convention; the pages only name the
    Qwen2.5 base models, [N1] "Experiments").
R2  Attention scale 1/sqrt(d); grouped-query heads map q head h to kv head
    floor(h / G), G = Hq / Hkv (contiguous groups, the Qwen convention).
R3  Decode attention: the current block sees every cached key and all 32 of
    its own keys, unmasked ([N1] key design 3; [N4] block-internal
    bidirectional, block-causal across blocks).
R4  2L x 2L training mask ([N1] key design 2): with blk(i) = (i mod L) div D,
    noisy(i) = i < L: noisy->noisy iff same block; noisy->clean iff
    blk(key) < blk(query); clean->clean iff blk(key) <= blk(query);
    clean->noisy never.
R5  Token shift ([N1] key design 2): the prediction for block position i
    reads hidden row i-1; position 0 reads the last row of the previous
    block (h_prev).
R6  Confidence = the probability the model gives the predicted token ([N2]
    item 2): p_max = max_v softmax(l)_v = 1 / sum_v exp(l_v - max l); the
    token is argmax_v l_v, ties to the lowest vocab index.
R7  Selection ([N1] key designs 3 and 4; [N2] item 2; [N4] item 2):
    candidates C are the masked positions of the active sub-block, the
    lowest-index sub-block [kS, (k+1)S) that still holds a masked position.
    Unmask every c in C with p_max(c) > tau (strict); if none, unmask the
    single c with the largest p_max, ties to the lowest position.  The strict
    comparison is the one under which tau = 1.0 reduces to one token per step
    ([N1] key design 3).  Every masked position of the block is scored.
R9  Masked-token cross-entropy of training ([N1] key design 2, the L_block
    equation with the shifted label): in every training sequence (the noisy
    stream x_t, L positions), each position i >= 1 whose token is [MASK]
    contributes -log softmax(W h_{i-1})[x_0^i]; position 0 has no previous
    row in its sequence and contributes nothing.  The equation's
    expectation is left to the caller: the step returns the per-position
    losses and their sum over the scored positions.
R10 Decoding loop ([N1] "Overall framework" and key design 3; [N4]
    "Acceleration engine" item 1): blocks of 32 are decoded left to right;
    a block starts with every position [MASK]; each denoising step runs the
    model on the block over the cache and applies the unmask rule (R7),
    until no position is [MASK]; the finished block is run once more with
    its final tokens and that run's K/V are committed to the cache, its last
    hidden row being the next block's h_prev.  The model is a caller-given
    single layer: x = E[token] (row V of E embeds [MASK]), q/k/v = x Wq /
    Wk / Wv, h = x + attn(q, k, v) Wo, logits = W h.
R11 Sub-block DualCache ([N1] key design 3; [N4] "Acceleration engine"
    item 1: inside the block being decoded, the K/V of its prefix and
    suffix are cached across the iterative refinement; [N1] "Limitations":
    the reuse is approximate).  Per sequence, at the first step of each
    active sub-block (R7) the whole block is run and its K, V and hidden
    rows are cached (a refresh); at the following steps of that sub-block
    only the active sub-block's S rows are fresh: the attention reads the
    cached K/V for the other 32 - S rows, and the shifted hidden rows
    outside the active sub-block are the cached ones.  With S = 32 the
    active sub-block is the whole block, so the loop is the exact one.
R8  Ambiguity: a position's token is ambiguous when its top-2 logit gap is
    < 1e-3; a sequence's unmask decision is ambiguous when some candidate has
    |p_max - tau| < 1e-4 (only for tau < 1: p_max = 1/Z with Z >= 1 never
    exceeds 1, so at tau >= 1 the comparison is false on every side), or when
    it falls back to the single most confident candidate and the two largest
    candidate p_max differ by < 1e-4.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 32
TOKEN_GAP_EPS = 1e-3
TAU_EPS = 1e-4

__all__ = [
    "BLOCK", "TOKEN_GAP_EPS", "TAU_EPS", "widen", "rope", "attention",
    "block_causal_allowed", "OracleCache", "block_attn_seq", "block_attn",
    "full_sequence_attn", "mixed_mask", "mask_attn", "shifted_rows",
    "lm_logits", "softmax_stats", "active_candidates", "select",
    "ambiguity", "confidence_select", "ce_positions", "masked_ce",
    "MASK_TOKEN", "mask_bits", "decode_loop",
]


# ----------------------------------------------------------------------------
# input widening
# ----------------------------------------------------------------------------
def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of fp32 data, or of bf16 data given as uint16 bits."""
    if dtype == "bf16":
        return (np.asarray(a).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# RoPE (reading R1)
# ----------------------------------------------------------------------------
def rope(x: np.ndarray, positions, theta: float) -> np.ndarray:
    """Rotate ``x`` ``[T, H, d]`` at absolute ``positions`` ``[T]``.

    x'_j = x_j cos(a) - x_{j+d/2} sin(a);  x'_{j+d/2} = x_{j+d/2} cos(a) + x_j sin(a),
    a = pos * theta^(-2j/d), j < d/2.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    pos = np.asarray(positions, dtype=np.float64)
    inv_freq = np.array([theta ** (-2.0 * j / d) for j in range(half)], dtype=np.float64)
    ang = pos[:, None] * inv_freq[None, :]                  # [T, d/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ----------------------------------------------------------------------------
# attention (reading R2)
# ----------------------------------------------------------------------------
def attention(q, k, v, allowed=None) -> np.ndarray:
    """softmax(q k^T / sqrt(d)) v per query head; GQA head h uses kv head h // G.

    q ``[Tq, Hq, d]``, k/v ``[Tk, Hkv, d]``, ``allowed`` ``[Tq, Tk]`` bool
    (None: every key visible).  Returns ``[Tq, Hq, d]``.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    Tq, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.empty((Tq, Hq, v.shape[2]), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        s = (q[:, h, :] @ k[:, g, :].T) / math.sqrt(d)
        if allowed is not None:
            s = np.where(allowed, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, g, :]
    return out


def block_causal_allowed(n_q: int, n_k: int, D: int = BLOCK, q_offset: int = 0):
    """Query i (absolute position q_offset + i) may see key j iff blk(j) <= blk(i).

    Bidirectional inside a block, causal across blocks ([N1] overall
    framework; [N4] core innovation).
    """
    qi = (np.arange(n_q) + q_offset) // D
    kj = np.arange(n_k) // D
    return kj[None, :] <= qi[:, None]


# ----------------------------------------------------------------------------
# block-level KV cache and decode attention ([N1] key design 3; [N4] item 1)
# ----------------------------------------------------------------------------
class OracleCache:
    """Per sequence: RoPE'd K and V of every finished block, in order.

    A finished block's keys are rotated at their absolute positions when it is
    committed and are read-only afterwards, like an autoregressive KV cache.
    """

    def __init__(self, batch: int, n_heads_kv: int, head_dim: int, theta: float):
        self.theta = theta
        self.k = [np.zeros((0, n_heads_kv, head_dim)) for _ in range(batch)]
        self.v = [np.zeros((0, n_heads_kv, head_dim)) for _ in range(batch)]

    def length(self, s: int) -> int:
        return self.k[s].shape[0]

    def commit(self, s: int, k_new, v_new):
        """Append finished blocks ``[32 * n, Hkv, d]`` (pre-RoPE k) to sequence s."""
        k_new = np.asarray(k_new, np.float64)
        assert k_new.shape[0] % BLOCK == 0
        P = self.length(s)
        kr = rope(k_new, np.arange(P, P + k_new.shape[0]), self.theta)
        self.k[s] = np.concatenate([self.k[s], kr], axis=0)
        self.v[s] = np.concatenate([self.v[s], np.asarray(v_new, np.float64)], axis=0)


def block_attn_seq(k_cache, v_cache, q, k_blk, v_blk, theta: float) -> np.ndarray:
    """Attention of one sequence's current block over [cache ; block].

    ``k_cache`` is already RoPE'd (``[P, Hkv, d]``); q/k_blk (``[32, H, d]``)
    are rotated here at positions P..P+31.  No mask (reading R3).
    """
    P = k_cache.shape[0]
    pos = np.arange(P, P + BLOCK)
    qr = rope(q, pos, theta)
    kr = rope(k_blk, pos, theta)
    keys = np.concatenate([k_cache, kr], axis=0)
    vals = np.concatenate([v_cache, np.asarray(v_blk, np.float64)], axis=0)
    return attention(qr, keys, vals)


def block_attn(cache: OracleCache, q, k_blk, v_blk) -> np.ndarray:
    """Batched :func:`block_attn_seq`: q ``[B, 32, Hq, d]`` -> ``[B, 32, Hq, d]``."""
    return np.stack([block_attn_seq(cache.k[s], cache.v[s], q[s], k_blk[s], v_blk[s], cache.theta)
                     for s in range(q.shape[0])])


def full_sequence_attn(q_all, k_all, v_all, theta: float, D: int = BLOCK, rows=None):
    """Recompute from scratch: every token of a sequence under the block-causal mask.

    q/k/v ``[T, H, d]`` pre-RoPE; returns the attention output of ``rows``
    (default: all).  The cached decode of the last block must equal its rows.
    """
    T = q_all.shape[0]
    pos = np.arange(T)
    qr = rope(q_all, pos, theta)
    kr = rope(k_all, pos, theta)
    rows = np.arange(T) if rows is None else np.asarray(rows)
    allowed = block_causal_allowed(T, T, D)[rows]
    return attention(qr[rows], kr, v_all, allowed)


# ----------------------------------------------------------------------------
# 2L x 2L complementary-mask attention of the training forward (reading R4)
# ----------------------------------------------------------------------------
def mixed_mask(L: int, D: int) -> np.ndarray:
    """A in {0,1}^{2L x 2L}: rows/cols 0..L-1 noisy x_t, L..2L-1 clean x_0."""
    i = np.arange(2 * L)
    noisy = i < L
    blk = (i % L) // D
    nq, nk = noisy[:, None], noisy[None, :]
    bq, bk = blk[:, None], blk[None, :]
    noisy_noisy = nq & nk & (bk == bq)
    noisy_clean = nq & ~nk & (bk < bq)
    clean_clean = ~nq & ~nk & (bk <= bq)
    return noisy_noisy | noisy_clean | clean_clean


def mask_attn(q, k, v, L: int, D: int, rows=None) -> np.ndarray:
    """Attention of ``[N, 2L, H, d]`` q/k/v under :func:`mixed_mask`.

    No RoPE inside (q/k arrive rotated).  ``rows`` restricts the query rows.
    """
    A = mixed_mask(L, D)
    rows = np.arange(2 * L) if rows is None else np.asarray(rows)
    return np.stack([attention(q[n][rows], k[n], v[n], A[rows]) for n in range(q.shape[0])])


# ----------------------------------------------------------------------------
# token shift, LM head, confidence (readings R5, R6)
# ----------------------------------------------------------------------------
def shifted_rows(h, h_prev, masked_bits):
    """Rows that predict the masked positions: position i <- hidden row i-1.

    h ``[B, 32, H]``, h_prev ``[B, H]``.  Returns (rows ``[M, H]``, list of
    (sequence, position)) in sequence-major, position-ascending order.
    """
    rows, where = [], []
    for s in range(h.shape[0]):
        bits = int(masked_bits[s])
        for i in range(BLOCK):
            if (bits >> i) & 1:
                rows.append(h_prev[s] if i == 0 else h[s, i - 1])
                where.append((s, i))
    H = h.shape[-1]
    return (np.array(rows, dtype=np.float64).reshape(len(rows), H), where)


def lm_logits(rows, W, w_dtype: str = "f32", cols: int = 16384) -> np.ndarray:
    """l = rows @ W^T in float64.  W ``[V, H]`` is widened a column slice at a time."""
    rows = np.asarray(rows, np.float64)
    V = W.shape[0]
    out = np.empty((rows.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, cols):
        out[:, v0:v0 + cols] = rows @ widen(W[v0:v0 + cols], w_dtype).T
    return out


def softmax_stats(logits):
    """Per row: p_max = 1 / sum exp(l - max), argmax (lowest index), top-2 gap."""
    logits = np.asarray(logits, np.float64)
    top = logits.max(axis=1)
    arg = logits.argmax(axis=1)                  # first occurrence: lowest index
    Z = np.exp(logits - top[:, None]).sum(axis=1)
    pmax = 1.0 / Z
    masked_top = logits.copy()
    masked_top[np.arange(logits.shape[0]), arg] = -np.inf
    second = masked_top.max(axis=1) if logits.shape[1] > 1 else np.full_like(top, -np.inf)
    return dict(pmax=pmax, argmax=arg.astype(np.int64), gap=top - second, Z=Z)


# ----------------------------------------------------------------------------
# confidence-aware selection (reading R7)
# ----------------------------------------------------------------------------
def active_candidates(bits: int, sub_block: int):
    """Masked positions of the lowest sub-block that still has a masked position."""
    masked = [i for i in range(BLOCK) if (bits >> i) & 1]
    if not masked:
        return []
    k = masked[0] // sub_block
    return [i for i in masked if k * sub_block <= i < (k + 1) * sub_block]


def select(pmax, argmax, masked_bits, tau: float, sub_block: int, tokens):
    """Unmask decision per sequence.

    pmax/argmax ``[B, 32]`` (read at masked positions).  Returns (tokens out
    ``[B, 32]``, unmask bits ``[B]``).  Positions not unmasked keep their
    input token.
    """
    tokens = np.array(tokens, dtype=np.int64, copy=True)
    B = tokens.shape[0]
    unmask = np.zeros(B, dtype=np.uint32)
    for s in range(B):
        C = active_candidates(int(masked_bits[s]), sub_block)
        if not C:
            continue
        chosen = [c for c in C if pmax[s][c] > tau]
        if not chosen:
            best = C[0]
            for c in C[1:]:
                if pmax[s][c] > pmax[s][best]:
                    best = c
            chosen = [best]
        for c in chosen:
            unmask[s] |= np.uint32(1 << c)
            tokens[s, c] = argmax[s][c]
    return tokens, unmask


def ambiguity(pmax, gap, masked_bits, tau: float, sub_block: int):
    """Flags of reading R8: (token_ambiguous ``[B, 32]``, decision_ambiguous ``[B]``)."""
    B = len(masked_bits)
    tok_amb = np.zeros((B, BLOCK), dtype=bool)
    dec_amb = np.zeros(B, dtype=bool)
    for s in range(B):
        bits = int(masked_bits[s])
        for i in range(BLOCK):
            if (bits >> i) & 1:
                tok_amb[s, i] = gap[s][i] < TOKEN_GAP_EPS
        C = active_candidates(bits, sub_block)
        if not C:
            continue
        if tau < 1.0 and any(abs(pmax[s][c] - tau) < TAU_EPS for c in C):
            dec_amb[s] = True
        elif not any(pmax[s][c] > tau for c in C) and len(C) > 1:
            top2 = sorted((pmax[s][c] for c in C), reverse=True)[:2]
            dec_amb[s] = (top2[0] - top2[1]) < TAU_EPS
    return tok_amb, dec_amb


def confidence_select(h, h_prev, W, masked_bits, tau: float, sub_block: int, tokens,
                      dtype: str = "f32"):
    """Whole unmask step: shift -> LM head -> softmax stats -> selection.

    h ``[B, 32, H]``, h_prev ``[B, H]``, W ``[V, H]``: fp32 arrays, or bf16
    bit patterns when ``dtype == "bf16"``.  Returns a dict with per-position
    ``pmax``/``argmax``/``gap`` (NaN / -1 where not masked), ``tokens``,
    ``unmask``, ambiguity flags and ``n_scored`` (masked positions scored).
    """
    hw = widen(h, dtype)
    hp = widen(h_prev, dtype)
    rows, where = shifted_rows(hw, hp, masked_bits)
    B = hw.shape[0]
    pmax = np.full((B, BLOCK), np.nan)
    gap = np.full((B, BLOCK), np.nan)
    arg = np.full((B, BLOCK), -1, dtype=np.int64)
    if rows.shape[0]:
        st = softmax_stats(lm_logits(rows, W, dtype))
        for r, (s, i) in enumerate(where):
            pmax[s, i] = st["pmax"][r]
            gap[s, i] = st["gap"][r]
            arg[s, i] = st["argmax"][r]
    tok, unmask = select(pmax, arg, masked_bits, tau, sub_block, tokens)
    tok_amb, dec_amb = ambiguity(pmax, gap, masked_bits, tau, sub_block)
    return dict(pmax=pmax, argmax=arg, gap=gap, tokens=tok, unmask=unmask,
                token_ambiguous=tok_amb, decision_ambiguous=dec_amb,
                n_scored=len(where))


# ----------------------------------------------------------------------------
# masked-token cross-entropy of training (reading R9)
# ----------------------------------------------------------------------------
def ce_positions(masked_bits):
    """Scored positions (sequence, i): [MASK] in x_t and i >= 1, in order.

    masked_bits ``[S, L/32]``: bit i % 32 of word i // 32 marks position i.
    """
    bits = np.asarray(masked_bits)
    S, nw = bits.shape
    return [(s, i) for s in range(S) for i in range(1, nw * 32)
            if (int(bits[s, i // 32]) >> (i % 32)) & 1]


def masked_ce(h, W, targets, masked_bits, dtype: str = "f32", positions=None, chunk: int = 256):
    """-log softmax(W h_{i-1})[targets_i] at every scored position (R9).

    h ``[S, L, H]``, W ``[V, H]`` (fp32 arrays or bf16 bit patterns per
    ``dtype``), targets ``[S, L]``, masked_bits ``[S, L/32]``.  ``positions``
    restricts the work to a subset of the scored positions (large cases).
    Returns dict(loss ``[S, L]`` with NaN where not computed, total = sum of
    the computed losses, count).
    """
    S, L = np.asarray(targets).shape
    pos = ce_positions(masked_bits) if positions is None else list(positions)
    loss = np.full((S, L), np.nan)
    for c0 in range(0, len(pos), chunk):
        part = pos[c0:c0 + chunk]
        rows = np.stack([widen(h[s, i - 1], dtype) for s, i in part]).astype(np.float64)
        logits = lm_logits(rows, W, dtype)
        top = logits.max(axis=1)
        lse = top + np.log(np.exp(logits - top[:, None]).sum(axis=1))
        for r, (s, i) in enumerate(part):
            loss[s, i] = lse[r] - logits[r, int(targets[s, i])]
    vals = np.array([loss[s, i] for s, i in pos], dtype=np.float64)
    return dict(loss=loss, total=float(vals.sum()), count=len(pos))


# ----------------------------------------------------------------------------
# the decoding loop, exact and with the sub-block DualCache (readings R10, R11)
# ----------------------------------------------------------------------------
MASK_TOKEN = -1  # id held by a still-masked position (outside [0, V))


def mask_bits(tokens) -> np.ndarray:
    """``[B, 32]`` tokens -> ``[B]`` words, bit i set where position i is [MASK]."""
    tokens = np.asarray(tokens)
    return np.array([sum(1 << i for i in range(BLOCK) if tokens[s, i] == MASK_TOKEN)
                     for s in range(tokens.shape[0])], dtype=np.uint32)


def decode_loop(weights, prompt, n_blocks: int, tau: float, sub_block: int, *,
                n_heads_q: int, n_heads_kv: int, head_dim: int, rope_theta: float,
                dual_cache: bool = False, trace: bool = False):
    """Decode ``n_blocks`` blocks after ``prompt`` (``[B, 32 n]`` tokens) with
    the single-layer model of reading R10, exactly or with the sub-block
    DualCache of reading R11.

    ``weights``: dict of float arrays E ``[V + 1, H]``, Wq ``[H, Hq d]``,
    Wk / Wv ``[H, Hkv d]``, Wo ``[Hq d, H]``, W ``[V, H]``.  Returns dict
    ``tokens`` ``[B, 32 (n + n_blocks)]``, ``steps`` ``[n_blocks, B]`` (steps
    each sequence took per block), ``unmasked`` (per block, per step, the
    ``[B]`` unmask words), ``ambiguous_at`` ((block, step) of the first
    decision flagged by reading R8, or None).  With ``trace``, also
    ``records``: per step (block, step, refresh flags ``[B]``, p_max of the
    step, p_max of the exact step on the same tokens and cache), ``h_prev``
    (per decoded block, the ``[B, H]`` rows its position 0 was read from)
    and ``cache`` (the :class:`OracleCache` after the loop).
    """
    E, Wq, Wk, Wv, Wo, W = (np.asarray(weights[n], np.float64)
                            for n in ("E", "Wq", "Wk", "Wv", "Wo", "W"))
    prompt = np.asarray(prompt)
    B, P = prompt.shape
    V = W.shape[0]
    Hq, Hkv, d = n_heads_q, n_heads_kv, head_dim
    cache = OracleCache(B, Hkv, d, rope_theta)

    def project(tok):
        x = E[np.where(tok == MASK_TOKEN, V, tok)]
        return (x, (x @ Wq).reshape(B, BLOCK, Hq, d), (x @ Wk).reshape(B, BLOCK, Hkv, d),
                (x @ Wv).reshape(B, BLOCK, Hkv, d))

    def hidden(x, q, k, v):
        return x + block_attn(cache, q, k, v).reshape(B, BLOCK, Hq * d) @ Wo

    def commit(k, v):
        for s in range(B):
            cache.commit(s, k[s], v[s])

    h_prev = np.zeros((B, E.shape[1]))
    for b in range(P // BLOCK):  # the prompt, block by block
        x, q, k, v = project(prompt[:, b * BLOCK:(b + 1) * BLOCK])
        h = hidden(x, q, k, v)
        commit(k, v)
        h_prev = h[:, BLOCK - 1]
    toks, logs, records, h_prev_in = [prompt], [], [], []
    steps = np.zeros((n_blocks, B), np.int64)
    ambiguous_at = None
    for b in range(n_blocks):
        h_prev_in.append(h_prev.copy())
        tok = np.full((B, BLOCK), MASK_TOKEN, np.int64)
        log = []
        cached_sub = [None] * B  # active sub-block the DualCache was filled for
        Kc = np.zeros((B, BLOCK, Hkv, d))
        Vc = np.zeros((B, BLOCK, Hkv, d))
        Hc = np.zeros((B, BLOCK, E.shape[1]))
        while (tok == MASK_TOKEN).any():
            bits = mask_bits(tok)
            steps[b] += (tok == MASK_TOKEN).any(axis=1)
            x, q, k, v = project(tok)
            refresh = np.ones(B, bool)
            if dual_cache:
                kb, vb = k.copy(), v.copy()
                rows = np.zeros((B, BLOCK), bool)  # the active sub-block's rows
                for s in range(B):
                    first = min(i for i in range(BLOCK) if tok[s, i] == MASK_TOKEN) \
                        if (tok[s] == MASK_TOKEN).any() else 0
                    a = first // sub_block
                    rows[s, a * sub_block:(a + 1) * sub_block] = True
                    refresh[s] = cached_sub[s] != a
                    if refresh[s]:
                        Kc[s], Vc[s] = k[s], v[s]
                        cached_sub[s] = a
                    kb[s] = np.where(rows[s][:, None, None], k[s], Kc[s])
                    vb[s] = np.where(rows[s][:, None, None], v[s], Vc[s])
                h_new = hidden(x, q, kb, vb)
                h = np.empty_like(h_new)
                for s in range(B):
                    if refresh[s]:
                        Hc[s] = h_new[s]
                    h[s] = np.where(rows[s][:, None], h_new[s], Hc[s])
            else:
                h = hidden(x, q, k, v)
            r = confidence_select(h, h_prev, W, bits, tau, sub_block, tok, "f32")
            if trace:
                exact = r if not dual_cache else confidence_select(
                    hidden(x, q, k, v), h_prev, W, bits, tau, sub_block, tok, "f32")
                records.append(dict(block=b, step=len(log), refresh=refresh.copy(),
                                    pmax=r["pmax"], pmax_exact=exact["pmax"]))
            picked_amb = any(r["token_ambiguous"][s, i] for s in range(B) for i in range(BLOCK)
                             if (int(r["unmask"][s]) >> i) & 1)
            if ambiguous_at is None and (r["decision_ambiguous"].any() or picked_amb):
                ambiguous_at = (b, len(log))
            tok = r["tokens"].astype(np.int64)
            log.append(r["unmask"].astype(np.uint32))
        x, q, k, v = project(tok)  # the finished block with its final tokens
        h = hidden(x, q, k, v)
        commit(k, v)
        h_prev = h[:, BLOCK - 1]
        toks.append(tok)
        logs.append(log)
    out = dict(tokens=np.concatenate(toks, 1), steps=steps, unmasked=logs,
               ambiguous_at=ambiguous_at)
    if trace:
        out.update(records=records, h_prev=h_prev_in, cache=cache)
    return out
