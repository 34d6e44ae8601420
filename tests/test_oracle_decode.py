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
