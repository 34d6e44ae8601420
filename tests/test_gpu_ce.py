"""bd_masked_ce (masked-token cross-entropy of training) against the oracle.

Small cases are compared at every position; the full training batch (16
sequences of 2048 positions, the 1.5B-shaped LM head) at sampled positions.
"""
import dataclasses

import numpy as np
import pytest

import oracle as O
from decoding_bd_block_b200 import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# fp32: LM-head products summed in fp32 over H and V; bf16 inputs are exact
# in both, so the tolerance only covers fp32 accumulation order.
ATOL = {"f32": 2e-4, "bf16": 2e-3}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from decoding_bd_block_b200 import bd  # noqa: F401  (fails loudly if libbd.so is missing)


def _run(cfg, d, loss_out=True):
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import to_device
    N, L = d["targets"].shape
    h = to_device(d["h"], cfg.dtype)
    w = to_device(d["W"], cfg.dtype)
    tg = torch.from_numpy(d["targets"]).cuda()
    mb = torch.from_numpy(d["masked_bits"].view(np.int32)).cuda()
    lo = torch.full((N, L), 7.0, dtype=torch.float32, device="cuda") if loss_out else None
    ls = torch.zeros(1, dtype=torch.float32, device="cuda")
    ns = torch.zeros(1, dtype=torch.int32, device="cuda")
    n = bd.bd_masked_ce_workspace_size(cfg.dtype, N, L, cfg.hidden, cfg.vocab)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    bd.bd_masked_ce(cfg.dtype, N, L, cfg.hidden, cfg.vocab, h, w, tg, mb, lo, ls, ns, ws)
    torch.cuda.synchronize()
    return (lo.cpu().numpy() if loss_out else None), float(ls.item()), int(ns.item())


SMALL = [
    dataclasses.replace(W.MASKED_CE, name="f32_s1x2_L64", samples=1, L=64, hidden=256, vocab=1000,
                        dtype="f32", seed=201),
    dataclasses.replace(W.MASKED_CE, name="bf16_s2x2_L96", samples=2, L=96, hidden=512,
                        vocab=3000, seed=202),
    dataclasses.replace(W.MASKED_CE, name="bf16_vocab_tail_h520", samples=1, L=128, hidden=520,
                        vocab=1001, seed=203),
    dataclasses.replace(W.MASKED_CE, name="bf16_all_masked", samples=1, views=1, L=64, hidden=256,
                        vocab=777, mask_p=1.0, seed=204),
    # >= 2048 packed rows: the rows-as-M LM head; ragged K (264 = 4 x 64 + 8),
    # ragged last W tile (20001 = 78 x 256 + 33), 9 vocab ranges, a partial
    # last row pair
    dataclasses.replace(W.MASKED_CE, name="bf16_rows_s2x2_L1024", samples=2, L=1024, hidden=264,
                        vocab=20001, seed=206),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_masked_ce_parity_small(cfg):
    d = W.make_ce_inputs(cfg)
    ref = O.masked_ce(d["h"], d["W"], d["targets"], d["masked_bits"], cfg.dtype)
    loss, total, count = _run(cfg, d)
    assert count == ref["count"]
    scored = ~np.isnan(ref["loss"])
    assert np.isnan(loss[~scored]).all()                     # position 0 and unmasked: NaN
    err = np.abs(loss[scored] - ref["loss"][scored]).max() if count else 0.0
    print(cfg.name, "count", count, "max abs err", err)
    assert err <= ATOL[cfg.dtype]
    assert total == pytest.approx(ref["total"], rel=1e-4, abs=ATOL[cfg.dtype] * max(count, 1))
    assert total == pytest.approx(float(loss[scored].astype(np.float64).sum()), rel=1e-5, abs=1e-3)


def test_masked_ce_nothing_scored_and_bad_target():
    cfg = dataclasses.replace(W.MASKED_CE, samples=1, views=1, L=64, hidden=256, vocab=500,
                              seed=205)
    d = W.make_ce_inputs(cfg)
    d0 = dict(d, masked_bits=np.zeros_like(d["masked_bits"]))
    loss, total, count = _run(cfg, d0)
    assert count == 0 and total == 0.0 and np.isnan(loss).all()
    d1 = dict(d, masked_bits=np.full_like(d["masked_bits"], 0xFFFFFFFF),
              targets=d["targets"].copy())
    d1["targets"][0, 5] = cfg.vocab                             # outside [0, vocab)
    loss, total, count = _run(cfg, d1)
    assert count == 63 and np.isnan(loss[0, 5]) and np.isnan(total)
    assert not np.isnan(np.delete(loss[0], [0, 5])).any()


def test_masked_ce_rows_path_nothing_scored():
    """>= 2048 packed rows allocated (the rows-as-M LM head) but no position
    scored: no unit of work, count 0, sum 0, every loss NaN."""
    cfg = dataclasses.replace(W.MASKED_CE, samples=2, L=1024, hidden=264, vocab=20001, seed=207)
    d = W.make_ce_inputs(cfg)
    d0 = dict(d, masked_bits=np.zeros_like(d["masked_bits"]))
    loss, total, count = _run(cfg, d0)
    assert count == 0 and total == 0.0 and np.isnan(loss).all()


def test_masked_ce_full_size_sampled_and_deterministic():
    cfg = W.MASKED_CE
    d = W.make_ce_inputs(cfg)
    loss, total, count = _run(cfg, d)
    pos = O.ce_positions(d["masked_bits"])
    assert count == len(pos)
    rng = np.random.default_rng(0)
    sample = [pos[k] for k in sorted(rng.choice(len(pos), 48, replace=False))]
    ref = O.masked_ce(d["h"], d["W"], d["targets"], d["masked_bits"], cfg.dtype, positions=sample)
    err = max(abs(loss[s, i] - ref["loss"][s, i]) for s, i in sample)
    print("full size: count", count, "sampled max abs err", err, "mean loss", total / count)
    assert err <= ATOL["bf16"]
    scored = np.zeros(loss.shape, bool)
    for s, i in pos:
        scored[s, i] = True
    assert np.isnan(loss[~scored]).all() and not np.isnan(loss[scored]).any()
    _, total2, _ = _run(cfg, d, loss_out=False)
    assert total2 == total                                      # fixed summation order
