"""Host-side checks of the precision claims the tensor-core assignment rests on
(no GPU): the two-bf16-plane split of an fp32 centroid and its error bound.

The kernel rounds with round-to-nearest-even to bf16 (h = bf16(c), then
m = bf16(c - h) with c - h exact in fp32); torch's float32 -> bfloat16
conversion is the same rounding."""
import numpy as np
import torch

U32 = 2.0 ** -24


def _split(c):
    t = torch.from_numpy(c)
    h = t.to(torch.bfloat16).to(torch.float32)
    r = t - h                       # exact in fp32
    m = r.to(torch.bfloat16).to(torch.float32)
    return h.numpy(), m.numpy(), r.numpy()


def test_two_plane_residual_is_below_2_pow_minus_17():
    g = np.random.default_rng(7)
    c = (g.standard_normal(500_000) * np.exp(g.uniform(-30, 30, 500_000))).astype(np.float32)
    h, m, r = _split(c)
    # c - h is exact: the planes reproduce c up to the second rounding
    assert np.array_equal((h.astype(np.float64) + r.astype(np.float64)).astype(np.float32), c)
    left = np.abs(c.astype(np.float64) - h.astype(np.float64) - m.astype(np.float64))
    assert np.all(left <= 2.0 ** -17 * np.abs(c.astype(np.float64)))
    # the first rounding alone leaves up to 2^-8: the second plane is needed
    assert np.max(np.abs(r.astype(np.float64)) / np.abs(c.astype(np.float64))) > 2.0 ** -9


def test_two_plane_distances_stay_inside_the_parity_band():
    # worst-case error of each computed distance |c|^2 - 2 x.(h + m) against the
    # exact one: split 2^-17 S, accumulation of 2d exact products 2d u S, and the
    # norm d u |c|^2 (S = sum_k |x_k c_k|); two candidates' errors together must
    # stay below the band 8 d u (|x|^2 + |c1|^2 + |c2|^2) that check_assign uses
    g = np.random.default_rng(11)
    for d in (64, 128):
        worst = 0.0
        cases = []
        for _ in range(2000):
            cases.append([g.standard_normal(d) * np.exp(g.uniform(-3, 3)) for _ in range(3)])
        # the worst geometry: x parallel to both centroids (S = |x||c|), |x| = sqrt(2)|c|
        c = np.abs(g.standard_normal(d))
        for k in np.linspace(0.25, 4.0, 64):
            cases.append([k * c, c, c])
        for x, c1, c2 in cases:
            err = 0.0
            for c in (c1, c2):
                S = np.abs(x * c).sum()
                err += 2 * (2.0 ** -17 + 2 * d * U32) * S + d * U32 * (c @ c)
            band = 8 * d * U32 * (x @ x + c1 @ c1 + c2 @ c2)
            worst = max(worst, err / band)
        assert worst < 1.0, (d, worst)
