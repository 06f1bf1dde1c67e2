"""Host-side checks of the precision claims the tensor-core assignment rests on
(no GPU): the two-bf16-plane split of an fp32 centroid, the three-part bf16
split of -|c|^2/2 that the kernel folds into its contraction, and the error
bound of the resulting distances.

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


def _split3(n):
    """-|c|^2/2 as the kernel's norm step: three bf16 parts, each the rounding
    of what the previous ones leave (every difference exact in fp32)."""
    t = torch.from_numpy(n)
    p0 = t.to(torch.bfloat16).to(torch.float32)
    r1 = t - p0
    p1 = r1.to(torch.bfloat16).to(torch.float32)
    p2 = (r1 - p1).to(torch.bfloat16).to(torch.float32)
    return p0.numpy(), p1.numpy(), p2.numpy()


def test_three_part_norm_split_holds_the_fp32_norm_to_2_pow_minus_24():
    g = np.random.default_rng(5)
    n = (-np.abs(g.standard_normal(500_000)) * np.exp(g.uniform(-20, 20, 500_000))).astype(np.float32)
    p0, p1, p2 = _split3(n)
    s = p0.astype(np.float64) + p1.astype(np.float64) + p2.astype(np.float64)
    rel = np.abs(s - n.astype(np.float64)) / np.abs(n.astype(np.float64))
    assert rel.max() <= 2.0 ** -24
    # two parts are not enough: the third carries bits
    assert (np.abs(p0.astype(np.float64) + p1 - n) / np.abs(n)).max() > 2.0 ** -20


def test_folded_norm_distances_stay_inside_the_parity_band():
    # the kernel's distance is -2 (x.(h + m) - |c|^2/2), accumulated in fp32
    # over the 2d plane products and the three norm parts: per candidate at
    # most 2 (2^-17 + (2d+3) u) S + ((2d+3) u + d u + 2 u) |c|^2 (S = sum_k
    # |x_k c_k|; d u |c|^2 for the fp32 norm itself, 2 u for its split and
    # halving); two candidates' errors together must stay below the band
    # 8 d u (|x|^2 + |c1|^2 + |c2|^2) that check_assign uses
    g = np.random.default_rng(13)
    for d in (64, 128):
        worst = 0.0
        cases = []
        for _ in range(2000):
            cases.append([g.standard_normal(d) * np.exp(g.uniform(-3, 3)) for _ in range(3)])
        c = np.abs(g.standard_normal(d))
        for k in np.linspace(0.25, 4.0, 64):
            cases.append([k * c, c, c])
        for x, c1, c2 in cases:
            err = 0.0
            for c in (c1, c2):
                S = np.abs(x * c).sum()
                err += 2 * (2.0 ** -17 + (2 * d + 3) * U32) * S + ((3 * d + 5) * U32) * (c @ c)
            band = 8 * d * U32 * (x @ x + c1 @ c1 + c2 @ c2)
            worst = max(worst, err / band)
        assert worst < 1.0, (d, worst)
