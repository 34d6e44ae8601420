"""The FMA-pipe exponential of the attention softmax and the LM-head folds
(poly_exp2 / poly_exp2x2: a degree-4 fit of 2^f on [-1/2, 1/2] after a
round-to-nearest split), held on the device to its stated relative error
bound over [-126, 0], against 2^x in double precision and against CUDA's
exp2f (torch.exp2 on the GPU).  The fitted polynomial is within 2.6e-6 of
2^f in exact arithmetic; its Horner steps round in fp32, which brings the
evaluated error to 2.69e-6 (at f = +-1/2), so the bound is 2.7e-6."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

BOUND = 2.7e-6


def _args():
    g = np.random.default_rng(7)
    x = np.concatenate([
        np.linspace(-126.0, 0.0, 1 << 20),                  # dense sweep
        g.uniform(-126.0, 0.0, 1 << 18),                    # random
        -np.arange(0, 127, dtype=np.float64),               # integers: f = 0
        -np.arange(0, 126, dtype=np.float64) - 0.5,         # ties of the rounding split
    ]).astype(np.float32)
    half = (-np.arange(0, 126) - 0.5).astype(np.float32)
    x = np.concatenate([x, np.nextafter(half, np.float32(0.0)), np.nextafter(half, np.float32(-200.0))])
    if len(x) % 2:
        x = np.append(x, np.float32(-1.0))
    return x


def test_poly_exp2_within_bound():
    from decoding_bd_block_b200 import bd
    x = _args()
    xd = torch.from_numpy(x).cuda()
    yp, y2, ym = (torch.empty_like(xd) for _ in range(3))
    bd.bd_eval_exp2(xd, yp, y2, ym)
    ref_gpu = torch.exp2(xd)
    torch.cuda.synchronize()
    exact = np.exp2(x.astype(np.float64))
    for name, y in (("poly_exp2", yp), ("poly_exp2x2", y2)):
        got = y.cpu().numpy().astype(np.float64)
        rel = np.abs(got - exact) / exact
        assert np.all(np.isfinite(got)), name
        assert rel.max() <= BOUND, (name, float(rel.max()), float(x[np.argmax(rel)]))
        # and against CUDA's own exp2f (itself within a few ulp of 2^x)
        rel_cuda = np.abs(got - ref_gpu.cpu().numpy()) / exact
        assert rel_cuda.max() <= BOUND + 2.5e-7, (name, float(rel_cuda.max()))
    # the paired form computes each lane as the scalar form does
    np.testing.assert_array_equal(yp.cpu().numpy(), y2.cpu().numpy())
    # the hardware approximation the rest of the exponentials use
    relm = np.abs(ym.cpu().numpy().astype(np.float64) - exact) / exact
    assert relm.max() <= 2.0 ** -21, float(relm.max())


def test_poly_exp2_below_range_clamps():
    # arguments below -126 return 2^-126 (the polynomial's input is clamped)
    from decoding_bd_block_b200 import bd
    x = torch.tensor([-126.0, -127.0, -150.0, -1e30, float("-inf")], device="cuda")
    yp, y2, ym = (torch.empty(6, device="cuda") for _ in range(3))
    xx = torch.cat([x, torch.tensor([0.0], device="cuda")])
    bd.bd_eval_exp2(xx, yp, y2, ym)
    torch.cuda.synchronize()
    want = np.float32(2.0 ** -126)
    got = yp.cpu().numpy()[:5]
    assert np.all(np.abs(got - want) <= want * BOUND), got
