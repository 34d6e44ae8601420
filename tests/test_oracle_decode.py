"""Pins of the oracle's decoding loop (readings R10, R11): the exact loop and
the sub-block DualCache, on a tiny single-layer model with seeded weights.

What fixes the DualCache loop independently of its own code:
* with S = 32 the active sub-block is the whole block, so every step's rows
  are fresh and the loop must equal the exact one;
* at tau = 0 every candidate is unmasked at once, so every step is the first
  of its sub-block (a refresh) and the loop must again equal the exact one;
* each sequence refreshes exactly 32 / S times per block, the refresh steps
  equal the exact step on the same tokens and cache, and the other steps
  do not (the cached rows are stale): the approximation is really there.
The exact loop is pinned by the tau = 1 closed form (one token per step).
"""
import numpy as np
import pytest

import oracle as O

KW = dict(n_heads_q=2, n_heads_kv=1, head_dim=16, rope_theta=1e4)
V, H = 64, 32


def weights(w_std=0.5, seed=3):
    g = np.random.default_rng(seed)
    hq, hk = KW["n_heads_q"] * KW["head_dim"], KW["n_heads_kv"] * KW["head_dim"]
    return dict(E=g.standard_normal((V + 1, H)), Wq=g.standard_normal((H, hq)) * H ** -0.5,
                Wk=g.standard_normal((H, hk)) * H ** -0.5, Wv=g.standard_normal((H, hk)) * H ** -0.5,
                Wo=g.standard_normal((hq, H)) * hq ** -0.5, W=g.standard_normal((V, H)) * w_std)


def prompt(B=2, blocks=1, seed=1):
    return np.random.default_rng(seed).integers(0, V, size=(B, 32 * blocks))


def same(a, b):
    return (np.array_equal(a["tokens"], b["tokens"]) and np.array_equal(a["steps"], b["steps"])
            and all(len(x) == len(y) and all(np.array_equal(u, w) for u, w in zip(x, y))
                    for x, y in zip(a["unmasked"], b["unmasked"])))


@pytest.mark.parametrize("tau", [0.9, 0.3])
def test_dual_cache_whole_block_is_exact(tau):
    w, p = weights(w_std=2.0), prompt()
    exact = O.decode_loop(w, p, 2, tau, 32, **KW)
    dual = O.decode_loop(w, p, 2, tau, 32, dual_cache=True, **KW)
    assert same(exact, dual)


def test_dual_cache_at_tau0_refreshes_every_step_and_is_exact():
    w, p = weights(), prompt()
    exact = O.decode_loop(w, p, 2, 0.0, 8, **KW)
    dual = O.decode_loop(w, p, 2, 0.0, 8, dual_cache=True, trace=True, **KW)
    assert (dual["steps"] == 4).all()            # one step per sub-block of 8
    assert all(rec["refresh"].all() for rec in dual["records"])
    assert same(exact, dual)


def test_dual_cache_refreshes_once_per_sub_block_and_is_approximate():
    w, p = weights(), prompt()
    S = 8
    dual = O.decode_loop(w, p, 2, 0.9, S, dual_cache=True, trace=True, **KW)
    recs = dual["records"]
    for b in range(2):
        n_ref = sum(rec["refresh"].astype(int) for rec in recs if rec["block"] == b)
        assert (n_ref == 32 // S).all()
    stale = []
    for rec in recs:
        for s in range(len(rec["refresh"])):
            m = ~np.isnan(rec["pmax_exact"][s])
            if not m.any():
                continue
            dev = np.abs(rec["pmax"][s][m] - rec["pmax_exact"][s][m]).max()
            if rec["refresh"][s]:
                assert dev <= 1e-12                  # a refresh step is the exact step
            else:
                stale.append(dev)
    assert stale and max(stale) > 1e-3              # the cached rows are stale


def test_exact_loop_tau1_one_token_per_step():
    w, p = weights(w_std=2.0), prompt()
    exact = O.decode_loop(w, p, 2, 1.0, 8, **KW)
    assert (exact["steps"] == 32).all()
    for log in exact["unmasked"]:
        for u in log:
            assert all(bin(int(x)).count("1") == 1 for x in u)


def _recompute(w, tokens):
    """The single layer of reading R10 on whole sequences, without any cache:
    per sequence x = E[tokens], q/k/v projections, the block-causal attention
    recomputed over every token, h = x + attn Wo."""
    E, Wq, Wk, Wv, Wo = (np.asarray(w[n], np.float64) for n in ("E", "Wq", "Wk", "Wv", "Wo"))
    Hq, Hkv, d, th = KW["n_heads_q"], KW["n_heads_kv"], KW["head_dim"], KW["rope_theta"]
    out = []
    for s in range(tokens.shape[0]):
        x = E[tokens[s]]
        T = x.shape[0]
        q = (x @ Wq).reshape(T, Hq, d)
        k = (x @ Wk).reshape(T, Hkv, d)
        v = (x @ Wv).reshape(T, Hkv, d)
        att = O.full_sequence_attn(q, k, v, th)
        out.append(dict(k=O.rope(k, np.arange(T), th), v=v, h=x + att.reshape(T, Hq * d) @ Wo))
    return out


@pytest.mark.parametrize("tau,dual", [(0.9, False), (0.3, False), (0.9, True)])
def test_committed_blocks_and_h_prev_equal_a_full_recompute(tau, dual):
    # [N1] key design 3: a decoded block's K/V become read-only context, as in
    # an AR KV cache.  After the loop, every committed block must hold the
    # rotated K and the V of its FINAL tokens at their absolute positions, and
    # each block's position 0 must have been read from the last hidden row of
    # the block before it, both as a cache-free recompute of the whole
    # sequence under the block-causal mask gives them.  Committing the K/V of
    # the last denoising step (one position still [MASK]) or taking h_prev
    # from that step fails here.
    w, p = weights(w_std=2.0), prompt(blocks=2)
    n_blocks, S = 3, 8
    r = O.decode_loop(w, p, n_blocks, tau, S, dual_cache=dual, trace=True, **KW)
    assert not (r["tokens"] == O.MASK_TOKEN).any()
    ref = _recompute(w, r["tokens"])
    T = r["tokens"].shape[1]
    for s, rs in enumerate(ref):
        np.testing.assert_allclose(r["cache"].k[s], rs["k"], rtol=0, atol=1e-10)
        np.testing.assert_allclose(r["cache"].v[s], rs["v"], rtol=0, atol=1e-12)
        assert r["cache"].length(s) == T
    n_prompt = p.shape[1] // 32
    for b in range(n_blocks):
        want = np.stack([rs["h"][32 * (n_prompt + b) - 1] for rs in ref])
        np.testing.assert_allclose(r["h_prev"][b], want, rtol=0, atol=1e-10)


def test_committed_pin_catches_a_stale_commit(monkeypatch):
    # The pin above must fail on a plausible slip: here the oracle's commit is
    # fed the K/V of the block with one position still [MASK] (as if the last
    # denoising step's projections were committed).
    w, p = weights(w_std=2.0), prompt()
    real_commit = O.OracleCache.commit
    def stale_commit(self, s, k_new, v_new):
        k_new = np.array(k_new, np.float64)
        if self.length(s) >= 32:            # a decoded block, not the prompt
            k_new[-1] += 1.0                # its last position's K changed
        return real_commit(self, s, k_new, v_new)
    monkeypatch.setattr(O.OracleCache, "commit", stale_commit)
    r = O.decode_loop(w, p, 2, 0.9, 8, trace=True, **KW)
    ref = _recompute(w, r["tokens"])
    assert not np.allclose(r["cache"].k[0], ref[0]["k"], atol=1e-10)
