"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Same seeded inputs on both sides.  Unmask decisions and tokens must be
bit-exact outside the ambiguity flags; attention within max-abs 1e-5 (fp32
storage) or 2e-2 (bf16 storage); p_max within 1e-4.
"""
import dataclasses

import numpy as np
import pytest

import oracle as O
from decoding_bd_block_b200 import workloads as W
from parity_util import ATOL, bf16_storage_block_attn, compare_select, oracle_block_attn

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from decoding_bd_block_b200 import bd  # noqa: F401  (fails loudly if libbd.so is missing)
    torch.cuda.init()


def _step(cfg, attn=True, sel=True, prefix=None):
    from decoding_bd_block_b200.step import DecodeStep
    a = W.make_attn_inputs(cfg, prefix) if attn else None
    s = W.make_select_inputs(cfg) if sel else None
    return a, s, DecodeStep(cfg, a, s)


# ------------------------------------------------------------ cache commit
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_commit_pages_match_oracle(dtype):
    from decoding_bd_block_b200.step import BlockCacheState
    cfg = dataclasses.replace(W.TINY_F32, dtype=dtype, batch=3, rope_theta=1e6, seed=77)
    P = np.array([96, 0, 320])
    a = W.make_attn_inputs(cfg, P)
    st = BlockCacheState(cfg, P, a["prefix_k"], a["prefix_v"])
    torch.cuda.synchronize()
    pages = st.cache.pages.float().cpu().numpy()
    pt = st.cache.page_table_host
    assert list(st.cache.n_blocks_host) == [3, 0, 10]
    assert st.cache.n_blocks.cpu().tolist() == [3, 0, 10]
    for s in (0, 2):
        c = O.OracleCache(1, cfg.n_heads_kv, cfg.head_dim, cfg.rope_theta)
        c.commit(0, O.widen(a["prefix_k"][s], dtype), O.widen(a["prefix_v"][s], dtype))
        for b in range(P[s] // 32):
            k_gpu = pages[pt[s, b], 0].transpose(1, 0, 2)   # [32, Hkv, d]
            v_gpu = pages[pt[s, b], 1].transpose(1, 0, 2)
            k_ref = c.k[0][32 * b:32 * (b + 1)]
            tol = 1e-6 if dtype == "f32" else 2.0 ** -8 * np.abs(k_ref) + 1e-6
            assert np.all(np.abs(k_gpu - k_ref) <= tol)
            np.testing.assert_array_equal(v_gpu, c.v[0][32 * b:32 * (b + 1)])


def test_commit_bulk_equals_block_by_block():
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import BlockCacheState, to_device
    cfg = dataclasses.replace(W.QWEN15B_STEP, batch=2, seed=78)
    P = np.array([256, 128])
    a = W.make_attn_inputs(cfg, P)
    bulk = BlockCacheState(cfg, P, a["prefix_k"], a["prefix_v"])
    one = BlockCacheState(cfg, P, None, None)
    for s in range(2):
        for b in range(P[s] // 32):
            k = to_device(a["prefix_k"][s][32 * b:32 * (b + 1)], cfg.dtype)
            v = to_device(a["prefix_v"][s][32 * b:32 * (b + 1)], cfg.dtype)
            bd.bd_cache_commit(one.cache, k, v, [s], 1)
    torch.cuda.synchronize()
    for s in range(2):
        for b in range(P[s] // 32):
            pb = bulk.cache.page_table_host[s, b]
            po = one.cache.page_table_host[s, b]
            assert torch.equal(bulk.cache.pages[pb], one.cache.pages[po])


# --------------------------------------------------------- block attention
ATTN_CASES = [
    W.TINY_F32,
    W.QWEN15B_STEP,
    W.QWEN7B_RAGGED,
    dataclasses.replace(W.TINY_F32, name="f32_d128_ragged", head_dim=128, batch=3,
                        prefix_tokens=(0, 32, 640), seed=91),
    dataclasses.replace(W.QWEN15B_STEP, name="bf16_d64_empty_prefix", head_dim=64,
                        prefix_tokens=(0,), seed=92),
    dataclasses.replace(W.QWEN7B_RAGGED, name="bf16_g7_long_ragged", batch=3,
                        prefix_range=(), prefix_tokens=(4096, 32, 2080), seed=93),
    # one 128-row query tile (G = 4), odd page counts
    dataclasses.replace(W.QWEN15B_STEP, name="bf16_g4_odd_pages", n_heads_q=8, n_heads_kv=2,
                        batch=3, prefix_tokens=(0, 96, 1024), seed=101),
    # G = 1: 32 query rows per CTA
    dataclasses.replace(W.QWEN15B_STEP, name="bf16_g1", n_heads_q=4, n_heads_kv=4,
                        prefix_tokens=(64,), seed=102),
    # CTA pairs: G = 8 fills both 128-row halves; G = 5 leaves three padding
    # warps in the second
    dataclasses.replace(W.QWEN15B_STEP, name="bf16_g8_pair_full", n_heads_q=16, n_heads_kv=2,
                        batch=2, prefix_tokens=(992, 4128), seed=105),
    dataclasses.replace(W.QWEN15B_STEP, name="bf16_g5_pair_pad", n_heads_q=10, n_heads_kv=2,
                        batch=2, prefix_tokens=(32, 2400), seed=106),
]


@pytest.mark.parametrize("cfg", ATTN_CASES, ids=lambda c: c.name)
def test_block_attn_parity(cfg):
    a, _, step = _step(cfg, sel=False)
    step.run_attn()
    torch.cuda.synchronize()
    got = step.out.float().cpu().numpy()
    ref = oracle_block_attn(cfg, a)
    err = max(float(np.abs(got[s] - ref[s]).max()) for s in ref)
    assert err <= ATOL[cfg.dtype], err


def test_block_attn_longctx_sampled():
    cfg = W.LONGCTX_ATTN
    a, _, step = _step(cfg, sel=False)
    step.run_attn()
    torch.cuda.synchronize()
    got = step.out.float().cpu().numpy()
    ref = oracle_block_attn(cfg, a, seqs=[0, 5])
    for s, r in ref.items():
        err = float(np.abs(got[s] - r).max())
        assert err <= ATOL["bf16"], (s, err)


def _growing_case():
    """Keys that grow page by page (up to 4x): the running max keeps rising
    across the KV stream, so the online softmax must rescale its accumulator
    (about one rescale per query row)."""
    cfg = dataclasses.replace(W.QWEN7B_RAGGED, name="bf16_growing", batch=2, prefix_range=(),
                              prefix_tokens=(3072, 1504), seed=103)
    a = W.make_attn_inputs(cfg)
    for s in range(cfg.batch):
        k = W.f32_from_bf16_bits(a["prefix_k"][s])
        ramp = (1.0 + np.arange(k.shape[0]) / 1024.0).astype(np.float32)[:, None, None]
        a["prefix_k"][s] = W.bf16_bits_from_f32(k * ramp)
    a["k_blk"] = W.bf16_bits_from_f32(W.f32_from_bf16_bits(a["k_blk"]) * 4.0)
    return cfg, a


def _run_growing():
    from decoding_bd_block_b200.step import DecodeStep
    cfg, a = _growing_case()
    step = DecodeStep(cfg, a, None)
    step.run_attn()
    torch.cuda.synchronize()
    return cfg, a, step.out.float().cpu().numpy()


def test_block_attn_growing_scores_rescale():
    # Reading: the bf16 path multiplies on the tensor cores, whose operands
    # are bf16, so the rotated q and keys are rounded to bf16 before the
    # products (whether the cache stores keys rotated or not).  Against the
    # oracle with exactly that rounding applied the kernel stays within the
    # bf16 bound; the error of the rounding itself against the fp64 oracle
    # is reported (about 3.4e-2 on this input class, see the strict xfail
    # below; about 2e-3 on the bf16 decoding workloads).
    cfg, a, got = _run_growing()
    ref = oracle_block_attn(cfg, a)
    emu = bf16_storage_block_attn(cfg, a)
    for s in ref:
        err_emu = float(np.abs(got[s] - emu[s]).max())
        print(f"seq {s}: vs bf16-operand oracle {err_emu:.3e}, vs fp64 oracle "
              f"{float(np.abs(got[s] - ref[s]).max()):.3e}, rounding alone "
              f"{float(np.abs(emu[s] - ref[s]).max()):.3e}")
        assert err_emu <= ATOL["bf16"]


@pytest.mark.xfail(strict=True, reason="bf16 tensor-core operands: rounding the rotated q and keys "
                   "alone is 3.4e-2 from the fp64 oracle on these growing keys (stated bound 2e-2)")
def test_block_attn_growing_scores_vs_fp64_oracle():
    cfg, a, got = _run_growing()
    ref = oracle_block_attn(cfg, a)
    assert max(float(np.abs(got[s] - ref[s]).max()) for s in ref) <= ATOL["bf16"]


def test_block_attn_score_spikes():
    """Single keys 100x larger than the rest, deep inside the cache: their
    scores exceed the running max by up to several hundred (base 2), far past
    the range of the FMA-pipe exponential.  Placed at key columns 6, 7 (mod 8)
    of a 128-key stage they fall on the polynomial pairs, elsewhere on the
    MUFU pairs; every row must still match the oracle with bf16 operands."""
    cfg = dataclasses.replace(W.QWEN7B_RAGGED, name="bf16_spikes", batch=2, prefix_range=(),
                              prefix_tokens=(3072, 1504), seed=104)
    a = W.make_attn_inputs(cfg)
    spikes = {0: (1030, 1500, 2055), 1: (700, 1270)}
    for s, toks in spikes.items():
        k = W.f32_from_bf16_bits(a["prefix_k"][s])
        for t in toks:
            k[t] *= 100.0
        a["prefix_k"][s] = W.bf16_bits_from_f32(k)
    from decoding_bd_block_b200.step import DecodeStep
    step = DecodeStep(cfg, a, None)
    step.run_attn()
    torch.cuda.synchronize()
    got = step.out.float().cpu().numpy()
    emu = bf16_storage_block_attn(cfg, a)
    for s in emu:
        assert np.isfinite(got[s]).all()
        err = float(np.abs(got[s] - emu[s]).max())
        print(f"seq {s}: vs bf16-operand oracle {err:.3e}")
        assert err <= ATOL["bf16"], (s, err)


def test_block_attn_repeatable_and_after_commit():
    # The block attention reads n_blocks on the device: commit the current
    # block, attend again with a new block, compare with the oracle.
    from decoding_bd_block_b200 import bd
    cfg = dataclasses.replace(W.TINY_F32, batch=2, prefix_tokens=(64, 0), seed=94)
    a, _, step = _step(cfg, sel=False)
    step.run_attn()
    first = step.out.clone()
    step.run_attn()
    torch.cuda.synchronize()
    assert torch.equal(first, step.out)
    bd.bd_cache_commit(step.cstate.cache, step.k_blk, step.v_blk, [0, 1], 1)
    a2 = W.make_attn_inputs(dataclasses.replace(cfg, seed=95), np.array([96, 32]))
    for key in ("prefix_k", "prefix_v"):
        a2[key] = [np.concatenate([a[key][s], a[{"prefix_k": "k_blk", "prefix_v": "v_blk"}[key]][s]])
                   for s in range(2)]
    from decoding_bd_block_b200.step import to_device
    step.q.copy_(to_device(a2["q"], cfg.dtype))
    step.k_blk.copy_(to_device(a2["k_blk"], cfg.dtype))
    step.v_blk.copy_(to_device(a2["v_blk"], cfg.dtype))
    n = bd.bd_block_attn_workspace_size(step.cstate.cache)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    bd.bd_block_attn(step.cstate.cache, step.q, step.k_blk, step.v_blk, step.out, ws)
    torch.cuda.synchronize()
    ref = oracle_block_attn(cfg, a2)
    got = step.out.cpu().numpy()
    assert max(float(np.abs(got[s] - ref[s]).max()) for s in ref) <= ATOL["f32"]


# ---------------------------------------------------- confidence select
SELECT_CASES = [
    (W.TINY_F32, 0.9, 8), (W.TINY_F32, 1.0, 8), (W.TINY_F32, 0.9, 32), (W.TINY_F32, 1.0, 32),
    (W.TINY_F32_LITERAL, 0.9, 8),
    (W.QWEN15B_STEP, 0.9, 8),
    (W.QWEN7B_RAGGED, 0.9, 8),
    (W.QWEN7B_RAGGED, 0.9, 32),
    (dataclasses.replace(W.QWEN15B_STEP, name="bf16_vocab_tail", vocab=1000, hidden=512, batch=5,
                         n_masked=0, masked_range=(0, 32), seed=96), 0.5, 4),
    (dataclasses.replace(W.TINY_F32, name="f32_all_masked_tau0", batch=4, n_masked=32,
                         seed=97), 0.0, 8),
    (dataclasses.replace(W.TINY_F32, name="f32_subblock1", batch=4, n_masked=0,
                         masked_range=(0, 32), seed=98), 0.9, 1),
    # batch 1: the single-kernel path with the rows resident in shared memory
    (dataclasses.replace(W.QWEN15B_STEP, name="fused_n16_h520_vocab_tail", vocab=1000, hidden=520,
                         n_masked=9, seed=101), 0.5, 4),
    (dataclasses.replace(W.QWEN15B_STEP, name="fused_all_masked_h2304", vocab=3000, hidden=2304,
                         n_masked=32, seed=102), 0.9, 8),
    (dataclasses.replace(W.QWEN15B_STEP, name="fused_none_masked", vocab=1000, hidden=256,
                         n_masked=0, seed=103), 0.9, 8),
    (dataclasses.replace(W.QWEN15B_STEP, name="fused_one_masked_v65536", vocab=65536, hidden=1536,
                         n_masked=1, seed=104), 0.9, 8),
]


@pytest.mark.parametrize("case", SELECT_CASES, ids=lambda c: f"{c[0].name}-tau{c[1]}-S{c[2]}")
def test_confidence_select_parity(case):
    cfg, tau, S = case
    _, s, step = _step(cfg, attn=False)
    step.run_select(tau, S)
    torch.cuda.synchronize()
    ref = O.confidence_select(s["h"], s["h_prev"], s["W"], s["masked_bits"], tau, S,
                              s["tokens"], cfg.dtype)
    res = compare_select(ref, step.tokens.cpu().numpy(), step.unmask.cpu().numpy().view(np.uint32),
                         step.pmax.cpu().numpy(), step.argmax.cpu().numpy(), s["masked_bits"])
    print(cfg.name, tau, S, res)
    if tau == 1.0:
        for b in range(cfg.batch):
            want = 1 if s["masked_bits"][b] else 0
            assert bin(int(step.unmask[b].item()) & 0xFFFFFFFF).count("1") == want


ACTIVE_CASES = [
    (W.TINY_F32, 0.9, 8),                                     # fp32, CUDA-core LM head
    (W.QWEN15B_STEP, 0.9, 8),                                 # batch 1: the single kernel
    (W.QWEN7B_RAGGED, 0.9, 8),                                # tensor-core LM head, packed rows
    (dataclasses.replace(W.QWEN15B_STEP, name="bf16_b5_active", vocab=1000, hidden=512, batch=5,
                         n_masked=0, masked_range=(0, 32), seed=105), 0.5, 4),
    (dataclasses.replace(W.QWEN15B_STEP, name="bf16_b1_s32_active", vocab=3000, hidden=512,
                         n_masked=30, seed=106), 0.9, 32),
]


@pytest.mark.parametrize("case", ACTIVE_CASES, ids=lambda c: f"{c[0].name}-tau{c[1]}-S{c[2]}")
def test_confidence_select_active_parity(case):
    """Scoring only the unmask rule's candidates: the same tokens and unmask
    bits as the full oracle step; p_max / argmax at the candidates only."""
    from decoding_bd_block_b200 import bd
    cfg, tau, S = case
    _, s, step = _step(cfg, attn=False)
    n0 = bd.bd_kernel_launches()
    step.run_select(tau, S, active_only=True)
    torch.cuda.synchronize()
    ref = O.confidence_select(s["h"], s["h_prev"], s["W"], s["masked_bits"], tau, S,
                              s["tokens"], cfg.dtype)
    cand = np.array([sum(1 << i for i in O.active_candidates(int(b), S)) for b in s["masked_bits"]],
                    dtype=np.uint32)
    res = compare_select(ref, step.tokens.cpu().numpy(), step.unmask.cpu().numpy().view(np.uint32),
                         step.pmax.cpu().numpy(), step.argmax.cpu().numpy(), cand)
    print(cfg.name, tau, S, res, "launches", bd.bd_kernel_launches() - n0)


@pytest.mark.parametrize("batch", [1, 3])  # single-kernel and three-kernel paths
def test_select_idempotent_and_masked_untouched(batch):
    cfg = dataclasses.replace(W.QWEN15B_STEP, batch=batch, vocab=4096, seed=99)
    _, s, step = _step(cfg, attn=False)
    step.run_select(0.9, 8)
    t1, u1 = step.tokens.clone(), step.unmask.clone()
    p1 = step.pmax.clone()
    for _ in range(3):  # the workspace header (status, arrivals) is reset by every call
        step.run_select(0.9, 8)
    torch.cuda.synchronize()
    assert torch.equal(t1, step.tokens) and torch.equal(u1, step.unmask)
    assert torch.equal(p1.isnan(), step.pmax.isnan())
    # vocab tiles go to whichever CTA asks first, so the order in which the
    # exp-sums are added, and with it the last bits of p_max, may vary
    torch.testing.assert_close(torch.nan_to_num(p1), torch.nan_to_num(step.pmax), rtol=1e-5,
                               atol=0)
    hdr = step.sel_ws[:16].view(torch.int32).cpu()
    assert hdr[1] == 0 and hdr[2] == 0 and hdr[3] == 0
    assert torch.equal(step.masked.cpu(), torch.from_numpy(s["masked_bits"].view(np.int32)))
    tin = step.tokens_in.cpu().numpy()
    tout = step.tokens.cpu().numpy()
    un = step.unmask.cpu().numpy().view(np.uint32)
    for b in range(batch):
        for i in range(32):
            if not (int(un[b]) >> i) & 1:
                assert tout[b, i] == tin[b, i]


# -------------------------------------------------- 2L x 2L mask attention
def _mask_case(L, D, dtype, n=2, Hq=4, Hkv=2, d=64, seed=5):
    cfg = W.MaskAttnConfig(name="t", samples=n, views=2, L=L, block=D, n_heads_q=Hq,
                           n_heads_kv=Hkv, head_dim=d, seed=seed, dtype=dtype)
    return cfg, W.make_mask_attn_inputs(cfg)


def _run_mask(cfg, t):
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import to_device
    q, k, v = (to_device(t[x], cfg.dtype) for x in ("q", "k", "v"))
    out = torch.empty_like(q)
    shape = bd.make_shape(cfg.n_heads_q, cfg.n_heads_kv, cfg.head_dim, cfg.dtype)
    bd.bd_block_mask_attn(shape, q, k, v, out, cfg.n_seqs, cfg.L, cfg.block)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("L,D,dtype,d,Hq,Hkv", [
    (64, 32, "f32", 64, 4, 2), (96, 16, "f32", 128, 4, 2), (128, 64, "bf16", 64, 4, 2),
    # tensor-core path (bf16, d = 128, L % 128 == 0)
    (256, 32, "bf16", 128, 4, 2),    # G = 2: one head pair per KV group
    (256, 16, "bf16", 128, 6, 2),    # G = 3: a single-head last pair; many partial tiles
    (384, 64, "bf16", 128, 12, 2),   # G = 6
    (512, 128, "bf16", 128, 4, 1),   # D = 128: fully visible noisy diagonal tiles
])
def test_mask_attn_parity_small(L, D, dtype, d, Hq, Hkv):
    cfg, t = _mask_case(L, D, dtype, d=d, Hq=Hq, Hkv=Hkv)
    got = _run_mask(cfg, t)
    ref = O.mask_attn(O.widen(t["q"], dtype), O.widen(t["k"], dtype), O.widen(t["v"], dtype), L, D)
    assert float(np.abs(got - ref).max()) <= ATOL[dtype]


def test_mask_attn_many_items_per_cta():
    """More work items than SMs (4 query tiles x 40 views x 4 head pairs =
    640 items, about four per persistent CTA, single-head pairs among them):
    every row of every view against the oracle."""
    cfg, t = _mask_case(256, 32, "bf16", n=20, d=128, Hq=6, Hkv=2, seed=7)
    got = _run_mask(cfg, t)
    ref = O.mask_attn(O.widen(t["q"], "bf16"), O.widen(t["k"], "bf16"), O.widen(t["v"], "bf16"),
                      cfg.L, cfg.block)
    assert float(np.abs(got - ref).max()) <= ATOL["bf16"]


def _run_mask_views(cfg, t, views):
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import to_device
    q, k, v = (to_device(t[x], cfg.dtype) for x in ("q", "k", "v"))
    out = torch.full_like(q, float("nan"))
    shape = bd.make_shape(cfg.n_heads_q, cfg.n_heads_kv, cfg.head_dim, cfg.dtype)
    bd.bd_block_mask_attn_views(shape, q, k, v, out, cfg.n_seqs, views, cfg.L, cfg.block)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("L,D,dtype,d,Hq,Hkv,samples,views", [
    (256, 32, "bf16", 128, 6, 2, 3, 4),   # tensor-core path, four views per sample
    (384, 16, "bf16", 128, 4, 2, 2, 2),   # tensor-core path, many partly visible tiles
    (96, 32, "f32", 64, 4, 2, 2, 2),      # CUDA-core path: every view computed from its inputs
])
def test_mask_attn_views_parity(L, D, dtype, d, Hq, Hkv, samples, views):
    # Views of one sample share the clean stream (the generator writes the same
    # x_0 rows into each view): the clean rows computed once per sample must be
    # every view's, against the oracle run on each view on its own, and equal
    # bit for bit to the plain call, which computes each view separately.
    cfg = W.MaskAttnConfig(name="t", samples=samples, views=views, L=L, block=D, n_heads_q=Hq,
                           n_heads_kv=Hkv, head_dim=d, seed=11, dtype=dtype)
    t = W.make_mask_attn_inputs(cfg)
    got = _run_mask_views(cfg, t, views)
    ref = O.mask_attn(O.widen(t["q"], dtype), O.widen(t["k"], dtype), O.widen(t["v"], dtype), L, D)
    assert float(np.abs(got - ref).max()) <= ATOL[dtype]
    np.testing.assert_array_equal(got, _run_mask(cfg, t))


def test_mask_attn_views_full_size_equals_plain_call():
    cfg = W.MASK_ATTN
    t = W.make_mask_attn_inputs(cfg)
    np.testing.assert_array_equal(_run_mask_views(cfg, t, cfg.views), _run_mask(cfg, t))


def test_mask_attn_full_size_sampled():
    cfg = W.MASK_ATTN
    t = W.make_mask_attn_inputs(cfg)
    got = _run_mask(cfg, t)
    rows = np.arange(0, 2 * cfg.L, 61)
    for n in (0, 1, cfg.n_seqs - 1):
        ref = O.mask_attn(O.widen(t["q"][n:n + 1], "bf16"), O.widen(t["k"][n:n + 1], "bf16"),
                          O.widen(t["v"][n:n + 1], "bf16"), cfg.L, cfg.block, rows=rows)[0]
        assert float(np.abs(got[n, rows] - ref).max()) <= ATOL["bf16"]


# ------------------------------------------------------------ error paths
def test_host_validation_errors_launch_nothing():
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import BlockCacheState, to_device
    cfg = dataclasses.replace(W.TINY_F32, batch=2, seed=100)
    st = BlockCacheState(cfg, np.array([32, 32]), None, None, extra_blocks=0)
    k = to_device(np.zeros((1, 64, 2, 64), np.float32), "f32")
    with pytest.raises(bd.BdError) as e:            # 2 blocks > max_blocks = 1
        bd.bd_cache_commit(st.cache, k, k, [0], 2)
    assert e.value.status == -3
    with pytest.raises(bd.BdError) as e:            # repeated sequence
        bd.bd_cache_commit(st.cache, k, k, [1, 1], 1)
    assert e.value.status == -1
    st.cache.page_table_host[1, 0] = st.cache.page_table_host[0, 0]
    bd.bd_cache_commit(st.cache, k[:, :32], k[:, :32], [0], 1)
    with pytest.raises(bd.BdError) as e:            # page already holds a block
        bd.bd_cache_commit(st.cache, k[:, :32], k[:, :32], [1], 1)
    assert e.value.status == -1
    assert list(st.cache.n_blocks_host) == [1, 0]
    a = W.make_attn_inputs(cfg, np.array([32, 0]))
    q = to_device(a["q"], "f32")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(bd.BdError) as e:
        bd.bd_block_attn(st.cache, q, q, q, torch.empty_like(q), ws, workspace_bytes=0)
    assert e.value.status == -4


# ------------------------------------------- canary-padded output buffers
CANARY, PAD = 0xA5, 4096


def _canaried(shape, dtype):
    """A tensor of `shape` inside a byte buffer with PAD canary bytes on each
    side (16-byte alignment kept); returns (buffer, tensor)."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    buf = torch.full((n + 2 * PAD,), CANARY, dtype=torch.uint8, device="cuda")
    return buf, buf[PAD:PAD + n].view(dtype).view(*shape)


def _canaries_intact(buf):
    return bool((buf[:PAD] == CANARY).all()) and bool((buf[-PAD:] == CANARY).all())


@pytest.mark.parametrize("cfg", [W.TINY_F32, W.QWEN15B_STEP, ATTN_CASES[5]], ids=lambda c: c.name)
def test_block_attn_writes_only_its_output(cfg):
    # The output of bd_block_attn sits between canary bytes: after the call
    # they are intact and the output equals that of the step's own buffer.
    from decoding_bd_block_b200 import bd
    _, _, step = _step(cfg, sel=False)
    step.run_attn()
    buf, out = _canaried(tuple(step.out.shape), step.out.dtype)
    bd.bd_block_attn(step.cstate.cache, step.q, step.k_blk, step.v_blk, out, step.attn_ws)
    torch.cuda.synchronize()
    assert _canaries_intact(buf)
    assert torch.equal(out, step.out)


@pytest.mark.parametrize("cfg", [W.TINY_F32, W.QWEN15B_STEP, W.QWEN7B_RAGGED], ids=lambda c: c.name)
def test_confidence_select_writes_only_its_outputs(cfg):
    # tokens, unmask bits, p_max and argmax each sit between canary bytes.
    from decoding_bd_block_b200 import bd
    _, s, step = _step(cfg, attn=False)
    step.run_select(0.9, 8)
    torch.cuda.synchronize()
    bt, tok = _canaried(tuple(step.tokens.shape), torch.int32)
    bu, un = _canaried(tuple(step.unmask.shape), torch.int32)
    bp, pm = _canaried(tuple(step.pmax.shape), torch.float32)
    ba, am = _canaried(tuple(step.argmax.shape), torch.int32)
    tok.copy_(step.tokens_in)
    bd.bd_confidence_select(cfg.dtype, cfg.batch, cfg.hidden, cfg.vocab, step.h, step.h_prev,
                            step.W, step.masked, 0.9, 8, tok, un, pm, am, step.sel_ws)
    torch.cuda.synchronize()
    assert all(_canaries_intact(b) for b in (bt, bu, bp, ba))
    assert torch.equal(tok, step.tokens) and torch.equal(un, step.unmask)
    assert torch.equal(am, step.argmax)
    torch.testing.assert_close(torch.nan_to_num(pm), torch.nan_to_num(step.pmax), rtol=1e-5, atol=0)
