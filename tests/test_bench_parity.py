"""The bench's parity block (host logic, no GPU): the oracle's own outputs
pass it, and a planted wrong token or decision is counted as a mismatch."""
import dataclasses

import numpy as np

import bench
from decoding_bd_block_b200 import workloads as W


def _case():
    cfg = dataclasses.replace(W.TINY_F32, batch=3, n_masked=0, masked_range=(1, 32), seed=311)
    a_in, s_in = W.make_attn_inputs(cfg), W.make_select_inputs(cfg)
    caches = bench.oracle_caches(cfg, a_in)
    ref = bench.oracle_full_step(cfg, a_in, s_in, 0.9, 8, caches)
    attn, sel = ref
    got = {"out": np.stack([attn[s] for s in range(cfg.batch)]).astype(np.float32),
           "tokens": sel["tokens"].astype(np.int32).copy(), "unmask": sel["unmask"].astype(np.uint32).copy(),
           "pmax": sel["pmax"].astype(np.float32), "argmax": sel["argmax"].astype(np.int32).copy(),
           "masked": np.asarray(s_in["masked_bits"], np.uint32)}
    return cfg, ref, got, sel


def test_oracle_outputs_pass():
    cfg, ref, got, _ = _case()
    p = bench.parity_block(cfg, ref, got, 0.9, 8)
    assert p["pass"] and p["decision_mismatches"] == 0 and p["token_mismatches"] == 0
    assert p["positions_checked"] == sum(bin(int(b)).count("1") for b in got["masked"])
    assert p["attn_max_abs_err"] < 1e-6


def test_planted_mismatches_are_counted():
    cfg, ref, got, sel = _case()
    s = next(s for s in range(cfg.batch) if not sel["decision_ambiguous"][s])
    got["unmask"][s] ^= 1 << 31
    i = next(i for i in range(32) if not sel["token_ambiguous"][s, i])
    got["tokens"][s, i] += 1
    got["out"][0, 0, 0, 0] += 1.0
    p = bench.parity_block(cfg, ref, got, 0.9, 8)
    assert not p["pass"]
    assert p["decision_mismatches"] == 1 and p["token_mismatches"] >= 1
    assert p["attn_max_abs_err"] >= 1.0 - 1e-6


def test_mask_pair_counts_match_the_mask():
    # The bench's algorithmic work for the 2L x 2L attention: its closed-form
    # pair counts against a count of the oracle's mask.  Clean queries see no
    # noisy key, which is why the views of one sample share their clean rows.
    import oracle as O
    for L, D in ((64, 8), (96, 32), (256, 32), (2048, 32)):
        A = O.mixed_mask(L, D)
        assert bench.mask_pairs(L, D) == int(A.sum())
        assert bench.mask_clean_pairs(L, D) == int(A[L:].sum())
        assert not A[L:, :L].any()


def test_nominal_fraction_beside_the_measured_one():
    r = bench.with_nominal({"unit": "GB/s", "achieved": 3850.0, "peak": 6545.0, "frac": 0.588})
    assert r["nominal_peak"] == 7700.0 and abs(r["frac_of_nominal"] - 0.5) < 1e-12
    assert r["frac"] == 0.588  # the measured-peak fraction is left as it is
    t = bench.with_nominal({"unit": "TFLOP/s", "achieved": 1125.0})
    assert abs(t["frac_of_nominal"] - 0.5) < 1e-12
    assert "frac_of_nominal" not in bench.with_nominal({"unit": "x/s", "achieved": 1.0})
