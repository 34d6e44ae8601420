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


def oracle_decode(model, prompt, n_blocks, tau, S):
    """The loop of decode.decode in float64 on the oracle's attention and select."""
    from decoding_bd_block_b200.workloads import BLOCK, MASK_TOKEN
    c = model.cfg
    B, P = prompt.shape
    Hq, Hkv, d, V = c.n_heads_q, c.n_heads_kv, c.head_dim, c.vocab
    E, Wq, Wk, Wv, Wo = (getattr(model, n).astype(np.float64) for n in ("E", "Wq", "Wk", "Wv", "Wo"))
    cache = O.OracleCache(B, Hkv, d, c.rope_theta)

    def forward(tok):
        x = E[np.where(tok == MASK_TOKEN, V, tok)]
        q, k, v = (x @ Wq).reshape(B, BLOCK, Hq, d), (x @ Wk).reshape(B, BLOCK, Hkv, d), \
            (x @ Wv).reshape(B, BLOCK, Hkv, d)
        att = O.block_attn(cache, q, k, v)
        return x + att.reshape(B, BLOCK, Hq * d) @ Wo, k, v

    def commit(k, v):
        for s in range(B):
            cache.commit(s, k[s], v[s])

    h_prev = np.zeros((B, c.hidden))
    for b in range(P // BLOCK):
        h, k, v = forward(prompt[:, b * BLOCK:(b + 1) * BLOCK])
        commit(k, v)
        h_prev = h[:, BLOCK - 1]
    toks, steps, logs, ambiguous_at = [prompt], np.zeros((n_blocks, B), np.int64), [], None
    for b in range(n_blocks):
        tok = np.full((B, BLOCK), MASK_TOKEN, np.int32)
        log = []
        while (tok == MASK_TOKEN).any():
            bits = np.array([sum(1 << i for i in range(BLOCK) if tok[s, i] == MASK_TOKEN)
                             for s in range(B)], dtype=np.uint32)
            steps[b] += (tok == MASK_TOKEN).any(axis=1)
            h, _, _ = forward(tok)
            r = O.confidence_select(h, h_prev, model.W, bits, tau, S, tok, "f32")
            picked_amb = any(r["token_ambiguous"][s, i] for s in range(B) for i in range(BLOCK)
                             if (int(r["unmask"][s]) >> i) & 1)
            if ambiguous_at is None and (r["decision_ambiguous"].any() or picked_amb):
                ambiguous_at = (b, len(log))
            tok = r["tokens"].astype(np.int32)
            log.append(r["unmask"].astype(np.uint32))
        h, k, v = forward(tok)
        commit(k, v)
        h_prev = h[:, BLOCK - 1]
        toks.append(tok)
        logs.append(log)
    return dict(tokens=np.concatenate(toks, 1), steps=steps, unmasked=logs,
                ambiguous_at=ambiguous_at)


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
    # the model must be decisive enough for the comparison to mean something
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
