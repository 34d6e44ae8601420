"""bd_confidence_select_noalloc against bd_confidence_select, through the C ABI.

The no-alloc entry point is for callers that cannot allocate device memory
when they run the decoding step (a plugin handed only its input and output
buffers, code running while a framework's allocator owns the device, a loop
that must not pay cudaMalloc's device synchronisation).  It keeps its scratch
in a fixed array inside the library instead of a caller workspace, shared by
every call on the device.  These tests check that two calls in a row give the
results of the workspace-taking call, and that a step too large for the
array is refused before anything runs.  This file is collected last so that a
failure here stops a `-x` run only after every other test has run.
"""
import dataclasses

import numpy as np
import pytest

from decoding_bd_block_b200 import workloads as W

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

PMAX_ATOL = 1e-4   # the p_max tolerance of the parity tests

CASES = [
    (W.QWEN15B_STEP, 0.9, 8),
    (W.TINY_F32, 0.9, 8),
    (W.QWEN7B_RAGGED, 0.9, 8),
    (dataclasses.replace(W.TINY_F32, name="f32_b5_tau1", batch=5, n_masked=0,
                         masked_range=(0, 32), seed=201), 1.0, 4),
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from decoding_bd_block_b200 import bd  # noqa: F401  (fails loudly if libbd.so is missing)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].name}-tau{c[1]}-S{c[2]}")
def test_noalloc_matches_workspace_call(case):
    from decoding_bd_block_b200 import bd
    from decoding_bd_block_b200.step import DecodeStep
    cfg, tau, S = case
    step = DecodeStep(cfg, None, W.make_select_inputs(cfg))
    step.run_select(tau, S)                      # existing entry point, caller workspace
    torch.cuda.synchronize()
    want = (step.tokens.cpu().numpy(), step.unmask.cpu().numpy(), step.pmax.cpu().numpy(),
            step.argmax.cpu().numpy())
    for _ in range(2):                           # two calls in a row on the shared array
        tokens = step.tokens_in.clone()
        unmask = torch.full_like(step.unmask, -1)
        pmax = torch.full_like(step.pmax, -7.0)
        argmax = torch.full_like(step.argmax, -7)
        bd.bd_confidence_select_noalloc(cfg.dtype, cfg.batch, cfg.hidden, cfg.vocab, step.h,
                                        step.h_prev, step.W, step.masked, tau, S, tokens,
                                        unmask, pmax, argmax)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(unmask.cpu().numpy(), want[1])
        np.testing.assert_array_equal(tokens.cpu().numpy(), want[0])
        np.testing.assert_array_equal(argmax.cpu().numpy(), want[3])
        got_p = pmax.cpu().numpy()
        np.testing.assert_array_equal(np.isnan(got_p), np.isnan(want[2]))
        m = ~np.isnan(want[2])
        assert np.all(np.abs(got_p[m] - want[2][m]) <= PMAX_ATOL)


def test_noalloc_refuses_step_larger_than_its_array():
    from decoding_bd_block_b200 import bd
    B, H, V = 40, 3584, 152064                  # scratch ~14 MB > BD_NOALLOC_SCRATCH_BYTES
    assert bd.bd_confidence_select_workspace_size("bf16", B, H, V) > bd.BD_NOALLOC_SCRATCH_BYTES
    h = torch.zeros((B, 32, H), dtype=torch.bfloat16, device="cuda")
    hp = torch.zeros((B, H), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((8, H), dtype=torch.bfloat16, device="cuda")
    bits = torch.ones(B, dtype=torch.int32, device="cuda")
    tok = torch.zeros((B, 32), dtype=torch.int32, device="cuda")
    un = torch.zeros(B, dtype=torch.int32, device="cuda")
    n0 = bd.bd_kernel_launches()
    with pytest.raises(bd.BdError) as e:
        bd.bd_confidence_select_noalloc("bf16", B, H, V, h, hp, w, bits, 0.9, 8, tok, un, None,
                                        None)
    assert e.value.status == -4                 # BD_ERR_WORKSPACE
    assert bd.bd_kernel_launches() == n0        # nothing was launched
