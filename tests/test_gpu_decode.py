"""The block-diffusion decoding loop (decode.py) on a small synthetic model,
against the same loop run on the oracle in fp64.

Checks the loop's structure (tau = 1 decodes one token per step, so every
block takes 32 steps; a lower tau takes at most 32) and that every token and
every step's unmask bits match the oracle's loop up to the first decision the
oracle flags as ambiguous.
"""
import numpy as np
import pytest

import oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from decoding_bd_block_b200 import bd  # noqa: F401  (fails loudly if libbd.so is missing)


def oracle_decode(model, prompt, n_blocks, tau, S, dual_cache=False):
    """The loop of decode.decode in float64 on the oracle (reading R10; R11
    with ``dual_cache``)."""
    c = model.cfg
    weights = {n: getattr(model, n) for n in ("E", "Wq", "Wk", "Wv", "Wo", "W")}
    return O.decode_loop(weights, prompt, n_blocks, tau, S, n_heads_q=c.n_heads_q,
                         n_heads_kv=c.n_heads_kv, head_dim=c.head_dim, rope_theta=c.rope_theta,
                         dual_cache=dual_cache)


def check_against_oracle(got, ref):
    """Every token, step count and unmask word equal, up to the first decision
    the oracle flags as ambiguous (which must not come too early)."""
    assert ref["ambiguous_at"] is None or ref["ambiguous_at"] >= (0, 8)
    if ref["ambiguous_at"] is None:
        assert np.array_equal(got["tokens"], ref["tokens"])
        assert np.array_equal(got["steps"], ref["steps"])
        for a, b in zip(got["unmasked"], ref["unmasked"]):
            assert len(a) == len(b) and all(np.array_equal(x, y) for x, y in zip(a, b))
    else:                                                      # equal up to the flagged step
        b0, j0 = ref["ambiguous_at"]
        for b in range(b0):
            assert all(np.array_equal(x, y) for x, y in zip(got["unmasked"][b], ref["unmasked"][b]))
        assert all(np.array_equal(x, y)
                   for x, y in zip(got["unmasked"][b0][:j0], ref["unmasked"][b0][:j0]))


@pytest.mark.parametrize("tau,S", [(1.0, 8), (0.9, 8), (0.5, 32)])
def test_decode_loop_matches_oracle_loop(tau, S):
    from decoding_bd_block_b200.decode import TinyModel, TinyModelConfig, decode
    model = TinyModel(TinyModelConfig())
    rng = np.random.default_rng(11)
    prompt = rng.integers(0, model.cfg.vocab, size=(2, 64)).astype(np.int32)
    got = decode(model, prompt, n_blocks=2, tau=tau, sub_block=S)
    ref = oracle_decode(model, prompt, 2, tau, S)
    assert (got["steps"] >= 1).all() and (got["steps"] <= 32).all()
    if tau >= 1.0:
        assert (got["steps"] == 32).all()                    # one token per step
        for log in got["unmasked"]:
            for u in log:
                assert all(bin(int(x)).count("1") == 1 for x in u)
    print("tau", tau, "S", S, "steps", got["steps"].tolist(), "oracle ambiguous at",
          ref["ambiguous_at"])
    check_against_oracle(got, ref)


@pytest.mark.parametrize("tau,S", [(0.9, 8), (1.0, 8), (0.9, 16)])
def test_decode_loop_dual_cache_matches_oracle_loop(tau, S):
    """The sub-block DualCache loop against the oracle's DualCache loop: the
    cache is approximate, so the reference is the oracle's own definition."""
    from decoding_bd_block_b200.decode import TinyModel, TinyModelConfig, decode
    model = TinyModel(TinyModelConfig())
    rng = np.random.default_rng(12)
    prompt = rng.integers(0, model.cfg.vocab, size=(2, 64)).astype(np.int32)
    got = decode(model, prompt, n_blocks=2, tau=tau, sub_block=S, dual_cache=True)
    ref = oracle_decode(model, prompt, 2, tau, S, dual_cache=True)
    assert (got["steps"] >= 32 // S).all() and (got["steps"] <= 32).all()
    # every sequence refreshes once per sub-block and block
    assert got["refreshes"] == 2 * 2 * (32 // S)
    print("dual cache: tau", tau, "S", S, "steps", got["steps"].tolist(), "oracle ambiguous at",
          ref["ambiguous_at"])
    check_against_oracle(got, ref)
