"""Pins for the CPU oracle: every routine is checked against something other
than itself -- a library routine on a special case, a closed form, an
invariant, brute force on tiny inputs, or the numbers the pages print.

Sources: "SVG-EAR measured error" (frontier-cs.org blog) worked example and
probe paragraph; SVG2 summary (paper-graph) section 3.4 on clustering,
permutation validity and k-means++; the SVG-EAR review (pith.science) on greedy
error-to-cost routing under a density budget.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Philox4x64-10 and the uniform draws
# --------------------------------------------------------------------------
@pytest.mark.parametrize("key,counter", [(0, (0, 0, 0, 0)), (5, (0, 0, 0, 0)),
                                         (2**64 - 1, (7, 3, 0, 0)),
                                         (123456789, (41, 9, 2, 5))])
def test_philox_matches_numpy_bit_generator(key, counter):
    # numpy's Philox increments its 256-bit counter before each block.
    bg = np.random.Philox(key=key, counter=np.array(counter, dtype=np.uint64))
    ref = bg.random_raw(4)
    ctr = list(counter)
    ctr[0] = (ctr[0] + 1) % 2**64
    got = oracle.philox4x64_10(ctr, [key % 2**64, key >> 64])
    assert [int(x) for x in got] == [int(x) for x in ref]


def test_uniform_is_top53_bits_of_first_word():
    for j in range(5):
        ctr = np.array([(j - 1) % 2**64, 3 if j else 2, 0, 0], dtype=np.uint64)
        bg = np.random.Philox(key=77, counter=ctr)
        w0 = int(bg.random_raw(1)[0])
        assert oracle.uniform(77, 3, j) == (w0 >> 11) * 2.0**-53
    u = [oracle.uniform(1, 0, j) for j in range(2000)]
    assert min(u) >= 0.0 and max(u) < 1.0
    assert abs(np.mean(u) - 0.5) < 0.03


# --------------------------------------------------------------------------
# k-means++ seeding
# --------------------------------------------------------------------------
def _kpp_numpy(X, C, seed, stream):
    N = X.shape[0]
    idx = [int(math.floor(oracle.uniform(seed, stream, 0) * N))]
    for j in range(1, C):
        D2 = np.min(((X[:, None, :] - X[idx][None]) ** 2).sum(-1), axis=1)
        cs = np.cumsum(D2)
        target = oracle.uniform(seed, stream, j) * cs[-1]
        idx.append(int(np.searchsorted(cs, target, side="right")))
    return np.array(idx)


@pytest.mark.parametrize("seed", [0, 1, 99])
def test_kmeanspp_matches_cumsum_searchsorted(seed):
    g = np.random.default_rng(seed)
    X = g.standard_normal((64, 4))
    idx, margin = oracle.kmeanspp(X, 12, seed, 5)
    ref = _kpp_numpy(X, 12, seed, 5)
    ok = margin[1:] > 1e-12
    assert np.array_equal(idx[0], ref[0])
    assert np.array_equal(idx[1:][ok], ref[1:][ok])
    assert len(set(idx.tolist())) == 12


def test_kmeanspp_d2_sampling_finds_every_separated_blob():
    # 10 tight blobs 1000 apart: D^2 sampling puts one seed in each blob
    # (uniform sampling would collide with probability ~ 1 - 10!/10^10).
    g = np.random.default_rng(3)
    centres = g.standard_normal((10, 8)) * 1000.0
    blob = np.repeat(np.arange(10), 50)
    X = centres[blob] + g.standard_normal((500, 8))
    for seed in range(5):
        idx, _ = oracle.kmeanspp(X, 10, seed, 0)
        assert sorted(blob[idx].tolist()) == list(range(10))


def test_kmeanspp_follow_reproduces_own_choices():
    g = np.random.default_rng(4)
    X = g.standard_normal((300, 6))
    own, _ = oracle.kmeanspp(X, 20, 11, 2)
    chk, margin = oracle.kmeanspp(X, 20, 11, 2, follow=own)
    assert np.array_equal(own, chk)
    assert np.all(margin[1:] >= 0)


def test_kmeanspp_all_identical_takes_lowest_unchosen():
    X = np.ones((8, 3))
    idx, _ = oracle.kmeanspp(X, 4, 0, 0)
    first = int(idx[0])
    rest = [t for t in range(8) if t != first][:3]
    assert idx[1:].tolist() == rest


# --------------------------------------------------------------------------
# assign / update / sort / segment mean
# --------------------------------------------------------------------------
def test_assign_matches_numpy_argmin_bruteforce():
    g = np.random.default_rng(0)
    X = g.standard_normal((500, 16))
    cent = g.standard_normal((23, 16))
    labels, second, best, gap = oracle.assign(X, cent)
    D = ((X[:, None, :] - cent[None]) ** 2).sum(-1)
    assert np.array_equal(labels, np.argmin(D, axis=1))
    assert np.allclose(best, D.min(1))
    Ds = np.sort(D, axis=1)
    assert np.allclose(gap, Ds[:, 1] - Ds[:, 0])
    assert np.all(second != labels)


def test_assign_exact_tie_goes_to_lowest_index():
    X = np.array([[0.0, 0.0], [1.0, 1.0]])
    cent = np.array([[1.0, 0.0], [0.0, 1.0], [-1.0, 0.0], [5.0, 5.0]])
    labels, second, _, gap = oracle.assign(X, cent)
    assert labels[0] == 0 and second[0] == 1 and gap[0] == 0.0
    assert labels[1] == 0 and second[1] == 1


def test_update_means_and_empty_cluster_keeps_previous():
    g = np.random.default_rng(1)
    X = g.standard_normal((200, 5))
    labels = g.integers(0, 6, 200)
    labels[labels == 4] = 5           # cluster 4 is empty
    prev = g.standard_normal((6, 5))
    out = oracle.update(X, labels, prev)
    cnt = np.bincount(labels, minlength=6)
    for c in range(6):
        if cnt[c]:
            assert np.allclose(out[c], X[labels == c].mean(0))
    assert np.array_equal(out[4], prev[4])
    assert np.allclose((out * cnt[:, None]).sum(0), X.sum(0))


def test_stable_sort_matches_numpy_stable_argsort():
    g = np.random.default_rng(2)
    for C in (1, 7, 50):
        labels = g.integers(0, C, 1000).astype(np.int32)
        perm, off = oracle.stable_sort(labels, C)
        assert np.array_equal(perm, np.argsort(labels, kind="stable"))
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(labels, minlength=C))]))
        assert np.array_equal(np.sort(perm), np.arange(1000))


def test_segment_mean_matches_reduceat_singletons_and_empties():
    g = np.random.default_rng(5)
    sizes = np.array([3, 1, 0, 7, 1, 0, 4])
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    Xp = g.standard_normal((sizes.sum(), 9))
    out = oracle.segment_mean(Xp, off)
    nz = sizes > 0
    ref = np.add.reduceat(Xp, off[:-1][nz], axis=0) / sizes[nz][:, None]
    assert np.allclose(out[nz], ref)
    assert np.array_equal(out[1], Xp[3]) and np.array_equal(out[4], Xp[11])
    assert np.all(out[2] == 0) and np.all(out[5] == 0)
    prev = np.full((7, 9), 3.5)
    assert np.all(oracle.segment_mean(Xp, off, prev)[5] == 3.5)


def test_cluster_recovers_separated_blobs_and_centroids_are_member_means():
    g = np.random.default_rng(6)
    centres = g.standard_normal((8, 16)) * 50
    truth = g.integers(0, 8, 2000)
    X = centres[truth] + g.standard_normal((2000, 16))
    out = oracle.cluster(X, 8, 10, seed=3, stream=0)
    # a bijection between found and true clusters
    pairs = set(zip(out["labels"].tolist(), truth.tolist()))
    assert len(pairs) == 8
    for c in range(8):
        members = X[out["labels"] == c]
        assert np.allclose(out["centroids"][c], members.mean(0))
    assert np.array_equal(out["Xp"], X[out["perm"]])


# --------------------------------------------------------------------------
# The worked toy example (golden numbers printed on the blog page)
# --------------------------------------------------------------------------
def _toy(vA=(1.0,), vB=((1.0,), (3.0,)), d=64):
    """q = 8 e1 so that q.k/sqrt(64) = k_1: keys score 1, 1 (A) and 0, 2 (B)."""
    q = np.zeros((1, d)); q[0, 0] = 8.0
    K = np.zeros((4, d)); K[:, 0] = [1.0, 1.0, 0.0, 2.0]
    V = np.zeros((4, d))
    V[0, 1] = V[1, 1] = vA[0]
    V[2, 1], V[3, 1] = vB[0][0], vB[1][0]
    k_off = np.array([0, 2, 4], dtype=np.int32)
    q_off = np.array([0, 1], dtype=np.int32)
    kbar = oracle.segment_mean(K, k_off)
    vbar = oracle.segment_mean(V, k_off)
    return q, K, V, q_off, k_off, kbar, vbar


def test_toy_example_weights_match_the_page():
    gold = json.load(open(os.path.join(GOLDEN, "toy_example.json")))["printed"]
    q, K, V, q_off, k_off, kbar, vbar = _toy()
    scale = 1.0 / 8.0
    perm = np.zeros(1, dtype=np.int32)
    # exact (both clusters computed): weight = e^lse
    _, lse_all = oracle.attend(q, K, V, q_off, k_off, np.array([0, 2], np.int32),
                               np.array([0, 1], np.int32), kbar, vbar, perm, scale)
    # A computed, B compensated / B computed, A compensated / both compensated
    _, lse_a = oracle.attend(q, K, V, q_off, k_off, np.array([0, 1], np.int32),
                             np.array([0], np.int32), kbar, vbar, perm, scale)
    _, lse_b = oracle.attend(q, K, V, q_off, k_off, np.array([0, 1], np.int32),
                             np.array([1], np.int32), kbar, vbar, perm, scale)
    _, lse_0 = oracle.attend(q, K, V, q_off, k_off, np.array([0, 0], np.int32),
                             np.zeros(0, np.int32), kbar, vbar, perm, scale)
    total = math.exp(lse_all[0])
    est_a = est_b = math.exp(lse_0[0]) / 2.0
    true_b = math.exp(lse_a[0]) - est_b       # A exact + B estimated
    true_a = total - (math.exp(lse_b[0]) - est_a)
    assert abs(total - gold["weight_total"]) < 0.05
    assert abs(true_a - gold["weight_A"]) < 0.05
    assert abs((total - true_a) - gold["weight_B"]) < 0.05
    assert abs(est_a - gold["centroid_estimate_A"]) < 0.05
    assert abs(est_b - gold["centroid_estimate_B"]) < 0.05
    assert abs((total - true_a) - est_b - gold["shortfall_B"]) < 0.1
    # "For A that is exact": computing B alone already gives the exact weight
    assert math.isclose(math.exp(lse_b[0]), total, rel_tol=1e-12)
    del true_b


def test_toy_example_error_aware_routing_picks_b_and_is_exact():
    q, K, V, q_off, k_off, kbar, vbar = _toy()
    scale = 1.0 / 8.0
    E = oracle.probe(q, K, V, kbar, vbar, k_off, scale)
    assert E[0, 0] == 0.0 and E[0, 1] > 0.0
    # room for one cluster: density 0.5 of Nk=4 keys = 2 keys
    pair_off, pair_kc = oracle.route(E.astype(np.float32), q_off, k_off, 4, 0.5)
    assert pair_kc.tolist() == [1]
    O, _ = oracle.attend(q, K, V, q_off, k_off, pair_off, pair_kc, kbar, vbar,
                         np.zeros(1, np.int32), scale)
    dense = softmax(q @ K.T * scale, axis=-1) @ V
    assert np.allclose(O, dense, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# Probe closed forms
# --------------------------------------------------------------------------
def test_probe_identical_keys_is_shifted_value_variance():
    # keys identical inside each cluster: e^{s_t} = e^{sbar}, so
    # E_ic = e^{2(s_c - m)} * sum_t |v_t - vbar_c|^2 = e^{2(s_c-m)} n_c sum var.
    g = np.random.default_rng(7)
    d, sizes = 8, [5, 3, 9, 1]
    kc = g.standard_normal((4, d))
    K = np.repeat(kc, sizes, axis=0)
    V = g.standard_normal((sum(sizes), d))
    k_off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    qbar = g.standard_normal((3, d))
    scale = 0.7
    E = oracle.probe(qbar, K, V, kc, oracle.segment_mean(V, k_off), k_off, scale)
    for i in range(3):
        s = scale * kc @ qbar[i]
        m = s.max()
        for c in range(4):
            Vc = V[k_off[c]:k_off[c + 1]]
            ref = math.exp(2 * (s[c] - m)) * sizes[c] * np.var(Vc, axis=0).sum()
            assert math.isclose(E[i, c], ref, rel_tol=1e-10, abs_tol=1e-300)
    assert np.all(E[:, 3] == 0.0)          # a singleton is exact


def test_probe_scales_with_value_square_and_ignores_key_order():
    g = np.random.default_rng(8)
    d = 6
    K = g.standard_normal((20, d)); V = g.standard_normal((20, d))
    k_off = np.array([0, 4, 11, 20], dtype=np.int32)
    kbar = oracle.segment_mean(K, k_off); vbar = oracle.segment_mean(V, k_off)
    qbar = g.standard_normal((2, d))
    E = oracle.probe(qbar, K, V, kbar, vbar, k_off, 0.5)
    E3 = oracle.probe(qbar, K, 3 * V, kbar, 3 * vbar, k_off, 0.5)
    assert np.allclose(E3, 9 * E, rtol=1e-12)
    p = np.concatenate([g.permutation(np.arange(a, b)) for a, b in zip(k_off[:-1], k_off[1:])])
    Ep = oracle.probe(qbar, K[p], V[p], kbar, vbar, k_off, 0.5)
    assert np.allclose(Ep, E, rtol=1e-12)


def test_probe_shift_is_the_global_row_max():
    # Two identical-key clusters: the ratio E_1/E_0 must carry e^{2(s1-s0)};
    # a per-cluster shift would cancel it.
    d = 2
    K = np.array([[0.0, 0.0]] * 2 + [[1.0, 0.0]] * 2)
    V = np.array([[1.0, 0.0], [-1.0, 0.0], [1.0, 0.0], [-1.0, 0.0]])
    k_off = np.array([0, 2, 4], dtype=np.int32)
    qbar = np.array([[2.0, 0.0]])
    E = oracle.probe(qbar, K, V, oracle.segment_mean(K, k_off),
                     oracle.segment_mean(V, k_off), k_off, 1.0)
    assert math.isclose(E[0, 1] / E[0, 0], math.exp(4.0), rel_tol=1e-12)
    assert math.isclose(E[0, 1], 2.0, rel_tol=1e-12)   # m = s_1 = 2: e^0 * 2 * 1


# --------------------------------------------------------------------------
# Greedy routing
# --------------------------------------------------------------------------
def _best_subset(E_row, sizes, budget):
    best = 0.0
    idx = [c for c in range(len(sizes)) if sizes[c] > 0]
    for r in range(len(idx) + 1):
        for S in itertools.combinations(idx, r):
            if sum(sizes[c] for c in S) <= budget:
                best = max(best, float(sum(E_row[c] for c in S)))
    return best


def test_route_equal_sizes_equals_exhaustive_optimum():
    g = np.random.default_rng(9)
    for trial in range(20):
        Ck, n = 10, 4
        k_off = np.arange(0, (Ck + 1) * n, n, dtype=np.int32)
        E = g.random((1, Ck)).astype(np.float32)
        density = g.random()
        po, pk = oracle.route(E, np.array([0, 3], np.int32), k_off, Ck * n, density)
        budget = math.floor(density * Ck * n)
        got = float(E[0, pk].astype(np.float64).sum())
        assert math.isclose(got, _best_subset(E[0].astype(np.float64), [n] * Ck, budget), rel_tol=1e-6)


def test_route_unequal_sizes_within_fractional_knapsack_bound():
    g = np.random.default_rng(10)
    for trial in range(30):
        Ck = 9
        sizes = g.integers(0, 8, Ck)
        k_off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
        Nk = int(sizes.sum())
        E = g.random((1, Ck)).astype(np.float32) * 10
        density = g.random()
        po, pk = oracle.route(E, np.array([0, 5], np.int32), k_off, Nk, density)
        budget = math.floor(density * Nk)
        assert sizes[pk].sum() <= budget
        assert np.all(sizes[pk] > 0) and np.all(np.diff(pk) > 0)
        got = float(E[0, pk].astype(np.float64).sum())
        opt = _best_subset(E[0].astype(np.float64), sizes.tolist(), budget)
        assert got >= opt - float(E[0][sizes > 0].max()) - 1e-6
        assert got <= opt + 1e-6


def test_route_skips_a_misfit_and_continues():
    # ratios: c1 = 9/2, c0 = 10/3, c2 = 1/1; budget 4 keys: take c1, c0 does
    # not fit (5 > 4) and is skipped, c2 still fits.
    E = np.array([[10.0, 9.0, 1.0]], dtype=np.float32)
    k_off = np.array([0, 3, 5, 6], dtype=np.int32)
    po, pk = oracle.route(E, np.array([0, 2], np.int32), k_off, 8, 0.5)
    assert pk.tolist() == [1, 2]


def test_route_density_one_takes_everything_and_ties_go_low():
    k_off = np.array([0, 2, 2, 5, 6], dtype=np.int32)         # cluster 1 empty
    q_off = np.array([0, 3, 3, 4], dtype=np.int32)            # query cluster 1 empty
    E = np.ones((3, 4), dtype=np.float32)
    po, pk = oracle.route(E, q_off, k_off, 6, 1.0)
    assert po.tolist() == [0, 3, 3, 6]
    assert pk.tolist() == [0, 2, 3, 0, 2, 3]
    # equal ratio everywhere, room for two of three size-2 clusters -> 0 and 1
    k2 = np.array([0, 2, 4, 6], dtype=np.int32)
    po, pk = oracle.route(np.ones((1, 3), np.float32) * 2, np.array([0, 1], np.int32), k2, 6, 0.7)
    assert pk.tolist() == [0, 1]


# --------------------------------------------------------------------------
# Attention with compensation
# --------------------------------------------------------------------------
def _random_clustered_head(g, Nq=40, Nk=50, d=8, Cq=5, Ck=7):
    Q = g.standard_normal((Nq, d)); K = g.standard_normal((Nk, d)); V = g.standard_normal((Nk, d))
    lq = g.integers(0, Cq, Nq); lk = g.integers(0, Ck, Nk)
    pq, oq = oracle.stable_sort(lq, Cq)
    pk, ok = oracle.stable_sort(lk, Ck)
    return Q, K, V, pq, oq, pk, ok


def _all_pairs(q_off, k_off):
    Cq, Ck = len(q_off) - 1, len(k_off) - 1
    po, pk = [0], []
    for i in range(Cq):
        if q_off[i + 1] > q_off[i]:
            pk += [c for c in range(Ck) if k_off[c + 1] > k_off[c]]
        po.append(len(pk))
    return np.array(po, np.int32), np.array(pk, np.int32)


def test_density_one_is_dense_softmax_attention_in_original_order():
    g = np.random.default_rng(11)
    Q, K, V, pq, oq, pk, ok = _random_clustered_head(g)
    Kp, Vp = K[pk], V[pk]
    kbar, vbar = oracle.segment_mean(Kp, ok), oracle.segment_mean(Vp, ok)
    po, pkc = _all_pairs(oq, ok)
    scale = 0.35
    O, lse = oracle.attend(Q[pq], Kp, Vp, oq, ok, po, pkc, kbar, vbar, pq, scale)
    S = Q @ K.T * scale
    assert np.allclose(O, softmax(S, axis=-1) @ V, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, np.log(np.exp(S).sum(-1)), rtol=1e-12)


def test_identical_keys_or_singletons_make_compensation_exact():
    g = np.random.default_rng(12)
    d, Ck = 8, 6
    sizes = np.array([4, 1, 6, 1, 3, 5])
    kc = g.standard_normal((Ck, d))
    Kp = np.repeat(kc, sizes, axis=0)
    Vp = g.standard_normal((sizes.sum(), d))
    ok = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    Q = g.standard_normal((30, d))
    oq = np.array([0, 10, 30], np.int32)
    pq = g.permutation(30).astype(np.int32)
    kbar, vbar = oracle.segment_mean(Kp, ok), oracle.segment_mean(Vp, ok)
    po = np.array([0, 2, 3], np.int32); pkc = np.array([1, 4, 2], np.int32)
    O, _ = oracle.attend(Q[pq], Kp, Vp, oq, ok, po, pkc, kbar, vbar, pq, 0.5)
    dense = softmax(Q @ Kp.T * 0.5, axis=-1) @ Vp
    assert np.allclose(O, dense, rtol=1e-11, atol=1e-12)


def test_output_is_invariant_under_token_relabelling():
    g = np.random.default_rng(13)
    Q, K, V, pq, oq, pk, ok = _random_clustered_head(g)
    lq = np.repeat(np.arange(len(oq) - 1), np.diff(oq))[np.argsort(pq)]
    lk = np.repeat(np.arange(len(ok) - 1), np.diff(ok))[np.argsort(pk)]
    po, pkc = np.array([0, 2, 3, 3, 5, 6], np.int32), np.array([0, 3, 6, 1, 5, 2], np.int32)

    def run(Q, K, V, lq, lk):
        pq, oq = oracle.stable_sort(lq, 5)
        pk, ok = oracle.stable_sort(lk, 7)
        Kp, Vp = K[pk], V[pk]
        kbar, vbar = oracle.segment_mean(Kp, ok), oracle.segment_mean(Vp, ok)
        return oracle.attend(Q[pq], Kp, Vp, oq, ok, po, pkc, kbar, vbar, pq, 0.4)[0]

    O = run(Q, K, V, lq, lk)
    sq, sk = g.permutation(len(Q)), g.permutation(len(K))
    O2 = run(Q[sq], K[sk], V[sk], lq[sq], lk[sk])
    assert np.allclose(O2, O[sq], rtol=1e-11, atol=1e-12)


def test_centroid_estimate_never_exceeds_true_weight():
    # mean(e^s) >= e^{mean s} (Jensen): compensated denominators under-count.
    g = np.random.default_rng(14)
    Q, K, V, pq, oq, pk, ok = _random_clustered_head(g, d=16)
    Kp, Vp = K[pk], V[pk]
    kbar, vbar = oracle.segment_mean(Kp, ok), oracle.segment_mean(Vp, ok)
    po_all, pk_all = _all_pairs(oq, ok)
    _, lse_dense = oracle.attend(Q[pq], Kp, Vp, oq, ok, po_all, pk_all, kbar, vbar, pq, 0.5)
    po = np.array([0, 1, 1, 3, 3, 4], np.int32); pkc = np.array([2, 0, 6, 4], np.int32)
    _, lse = oracle.attend(Q[pq], Kp, Vp, oq, ok, po, pkc, kbar, vbar, pq, 0.5)
    assert np.all(lse <= lse_dense + 1e-12)
    assert np.any(lse < lse_dense - 1e-3)


def test_row_subset_matches_full_output():
    g = np.random.default_rng(15)
    Q, K, V, pq, oq, pk, ok = _random_clustered_head(g)
    Kp, Vp = K[pk], V[pk]
    kbar, vbar = oracle.segment_mean(Kp, ok), oracle.segment_mean(Vp, ok)
    po = np.array([0, 2, 3, 3, 5, 6], np.int32); pkc = np.array([0, 3, 6, 1, 5, 2], np.int32)
    O, lse = oracle.attend(Q[pq], Kp, Vp, oq, ok, po, pkc, kbar, vbar, pq, 0.4)
    rows = np.array([39, 0, 17, 5])
    Or, lr = oracle.attend(Q[pq], Kp, Vp, oq, ok, po, pkc, kbar, vbar, pq, 0.4, rows=rows)
    assert np.array_equal(Or, O[pq[rows]]) and np.array_equal(lr, lse[pq[rows]])


def test_layer_at_density_one_equals_dense_attention():
    g = np.random.default_rng(16)
    Q = g.standard_normal((96, 8)); K = g.standard_normal((80, 8)); V = g.standard_normal((80, 8))
    out = oracle.layer(Q, K, V, Cq=4, Ck=6, iters=3, density=1.0, scale=0.3,
                       seed_q=1, seed_k=2, stream=0)
    assert np.allclose(out["O"], softmax(Q @ K.T * 0.3, axis=-1) @ V, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------------------
# Top-p budget (SVG2 summary, section 3.4, "Top-p selection for dynamic budget
# allocation"; SVG-EAR blog, budget paragraph)
# ---------------------------------------------------------------------------
def _offsets(sizes):
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)


def test_topp_identical_centroids_rank_clusters_by_size():
    # every centroid scores the same, so P'_j = n_j / N: sizes 5, 1, 3, 1 hold
    # 0.5, 0.1, 0.3, 0.1 of the weight; worked by hand
    k_off = _offsets([5, 1, 3, 1])
    q_off = np.array([0, 7], dtype=np.int32)
    qbar = np.full((1, 8), 0.25)
    kbar = np.full((4, 8), -0.5)
    for p, want in ((0.5, 5), (0.55, 8), (0.8, 8), (0.85, 9), (0.95, 10), (1.0, 10), (0.01, 5)):
        b, _ = oracle.topp_budget(qbar, kbar, q_off, k_off, p, 0.3)
        assert b[0] == want, (p, b[0], want)


def test_topp_dominant_cluster_alone_holds_the_mass():
    g = np.random.default_rng(40)
    d = 16
    kbar = g.standard_normal((6, d)) * 0.1
    kbar[3] = 4.0 * np.ones(d) / np.sqrt(d)          # the key cluster q points at
    qbar = (4.0 * np.ones(d) / np.sqrt(d))[None]
    k_off = _offsets([30, 30, 30, 2, 30, 30])        # small cluster, but e^{16} outweighs size
    b, _ = oracle.topp_budget(qbar, kbar, np.array([0, 3]), k_off, 0.9, 1.0)
    assert b[0] == 2
    # with the score flipped the cluster is the least attended one
    b, _ = oracle.topp_budget(-qbar, kbar, np.array([0, 3]), k_off, 0.9, 1.0)
    assert b[0] > 0 and b[0] <= 150 and b[0] != 2


def test_topp_p_one_takes_every_nonempty_cluster_and_empties_take_none():
    g = np.random.default_rng(41)
    sizes = np.array([4, 0, 7, 3, 0, 9, 1])
    k_off = _offsets(sizes)
    q_off = np.array([0, 5, 5, 9], dtype=np.int32)   # query cluster 1 is empty
    qbar = g.standard_normal((3, 8)) * 0.3
    kbar = g.standard_normal((7, 8)) * 0.3
    b, _ = oracle.topp_budget(qbar, kbar, q_off, k_off, 1.0, 0.5)
    assert list(b) == [sizes.sum(), 0, sizes.sum()]


def test_topp_prefix_has_the_fewest_clusters_reaching_p_brute_force():
    # the descending order makes the taken prefix the smallest number of key
    # clusters whose weight reaches p: checked over every subset
    import itertools
    g = np.random.default_rng(42)
    for trial in range(30):
        Ck = 6
        sizes = g.integers(1, 9, Ck)
        k_off = _offsets(sizes)
        qbar = g.standard_normal((1, 5))
        kbar = g.standard_normal((Ck, 5))
        p = float(g.uniform(0.2, 0.97))
        b, margin = oracle.topp_budget(qbar, kbar, np.array([0, 4]), k_off, p, 0.7)
        w = sizes * np.exp(0.7 * kbar @ qbar[0])
        w = w / w.sum()
        kmin = min(len(T) for r in range(1, Ck + 1) for T in itertools.combinations(range(Ck), r)
                   if w[list(T)].sum() >= p - 1e-12)
        # the prefix of that length: its sizes must sum to the budget
        top = np.argsort(-w, kind="stable")[:kmin]
        if margin[0] > 1e-9:
            assert b[0] == sizes[top].sum(), (trial, b[0], sizes[top].sum())


def test_topp_budget_grows_with_p():
    g = np.random.default_rng(43)
    sizes = g.integers(0, 20, 40)
    k_off = _offsets(sizes)
    qbar = g.standard_normal((3, 16)) * 0.5
    kbar = g.standard_normal((40, 16)) * 0.5
    q_off = np.array([0, 10, 20, 30], dtype=np.int32)
    prev = np.zeros(3, dtype=np.int64)
    for p in np.linspace(0.05, 1.0, 20):
        b, _ = oracle.topp_budget(qbar, kbar, q_off, k_off, p, 0.25)
        assert np.all(b >= prev)
        prev = b
    assert np.all(prev == sizes.sum())


def test_route_with_budgets_equals_route_with_the_same_density_per_row():
    g = np.random.default_rng(44)
    Cq, Ck, Nk = 5, 12, 100
    sizes = g.multinomial(Nk, np.ones(Ck) / Ck)
    k_off = _offsets(sizes)
    q_off = _offsets([3, 0, 4, 2, 5])
    E = g.random((Cq, Ck)).astype(np.float32)
    budgets = np.array([0, 37, 55, 100, 12], dtype=np.int64)
    off, kc = oracle.route(E, q_off, k_off, Nk, 0.5, budgets=budgets)
    for i in range(Cq):
        o1, k1 = oracle.route(E[i:i + 1], q_off[i:i + 2] - q_off[i], k_off, Nk,
                              (budgets[i] + 0.5) / Nk)
        assert np.array_equal(kc[off[i]:off[i + 1]], k1)


# ---------------------------------------------------------------------------
# Variance-corrected compensation (SVG-EAR blog, variance paragraph)
# ---------------------------------------------------------------------------
def test_segment_variance_closed_forms():
    Xp = np.array([[0.0, 5.0], [2.0, 5.0],          # segment 0: var 1, 0
                   [1.0, -3.0], [4.0, 1.0], [7.0, 2.0],  # segment 1
                   [3.0, 3.0]])                      # segment 2: single row
    off = np.array([0, 2, 2, 5, 6], dtype=np.int32)  # segment 1 empty
    v = oracle.segment_var(Xp, off)
    assert np.allclose(v[0], [1.0, 0.0])
    assert np.all(v[1] == 0.0)
    # {1, 4, 7}: mean 4, var (9+0+9)/3 = 6;  {-3, 1, 2}: mean 0, var (9+1+4)/3
    assert np.allclose(v[2], [6.0, 14.0 / 3.0])
    assert np.all(v[3] == 0.0)


def _weight_of_one_skipped_cluster(keys, q, lam, scale=1.0):
    """exp(lse) of one query row whose only key cluster is skipped: the
    cluster's (corrected) estimated weight."""
    keys = np.asarray(keys, dtype=np.float64)
    n, d = keys.shape
    q = np.asarray(q, dtype=np.float64)[None]
    k_off = np.array([0, n], dtype=np.int32)
    kbar = keys.mean(0, keepdims=True)
    kvar = oracle.segment_var(keys, k_off)
    vbar = np.ones((1, d))
    _, lse = oracle.attend(q, keys, np.ones((n, d)), np.array([0, 1]), k_off,
                           np.array([0, 0]), np.zeros(0, np.int32), kbar, vbar,
                           np.array([0]), scale, kvar=kvar, lam=lam)
    return float(np.exp(lse[0]))


def test_variance_toy_cluster_b_matches_the_printed_estimate():
    g = json.load(open(os.path.join(GOLDEN, "variance_example.json")))
    # cluster B of the toy example: scores 0 and 2 for q = 1, d = 1, scale 1
    w_corr = _weight_of_one_skipped_cluster([[0.0], [2.0]], [1.0], lam=1.0)
    w_plain = _weight_of_one_skipped_cluster([[0.0], [2.0]], [1.0], lam=0.0)
    assert abs(w_corr - 2 * math.exp(1.5)) < 1e-12
    assert abs(w_corr - g["corrected_estimate_B_printed"]) <= g["printed_precision"]
    assert abs(w_plain - g["uncorrected_estimate_B_printed"]) <= g["printed_precision"]
    true_b = math.exp(0.0) + math.exp(2.0)
    assert abs(true_b - g["true_weight_B_printed"]) <= g["printed_precision"]
    # the corrected estimate lands closer to the truth, from above
    assert abs(w_corr - true_b) < abs(w_plain - true_b) and w_corr > true_b > w_plain


def test_variance_term_vanishes_for_identical_keys_and_scales_with_lambda():
    g = np.random.default_rng(45)
    d = 8
    k = g.standard_normal(d)
    q = g.standard_normal(d)
    same = np.tile(k, (5, 1))
    base = _weight_of_one_skipped_cluster(same, q, lam=0.0, scale=0.4)
    for lam in (0.5, 1.0, 1.5):
        assert abs(_weight_of_one_skipped_cluster(same, q, lam, scale=0.4) - base) < 1e-12 * base
    # spread keys: log-weight grows linearly in lambda by scale^2/2 sum q^2 var
    keys = g.standard_normal((6, d))
    var = keys.var(axis=0)
    w0 = _weight_of_one_skipped_cluster(keys, q, 0.0, scale=0.4)
    for lam in (0.5, 1.5):
        w = _weight_of_one_skipped_cluster(keys, q, lam, scale=0.4)
        want = lam * 0.4 ** 2 / 2 * float((q ** 2 * var).sum())
        assert abs(math.log(w / w0) - want) < 1e-12


# ---------------------------------------------------------------------------
# Value-free probe error and the recall / MSE diagnostics
# ---------------------------------------------------------------------------
def test_value_free_error_is_the_value_aware_error_with_unit_values():
    g = np.random.default_rng(46)
    d, N, Cq, Ck = 8, 60, 3, 5
    Kp = g.standard_normal((N, d))
    k_off = _offsets([10, 0, 25, 5, 20])
    kbar = np.stack([Kp[k_off[c]:k_off[c + 1]].mean(0) if k_off[c + 1] > k_off[c]
                     else np.zeros(d) for c in range(Ck)])
    qbar = g.standard_normal((Cq, d))
    u = np.zeros(d)
    u[3] = 1.0                                          # one unit value vector for all
    Eaware = oracle.probe(qbar, Kp, np.tile(u, (N, 1)), kbar, np.tile(u, (Ck, 1)), k_off, 0.5)
    Efree = oracle.probe_value_free(qbar, Kp, kbar, k_off, 0.5)
    assert np.allclose(Efree, Eaware, rtol=1e-12, atol=1e-300)
    assert np.all(Efree[:, 1] == 0.0)                   # empty cluster


def test_value_free_error_closed_form_and_identical_keys():
    # cluster B of the toy example: scores 0 and 2 for q = 1, centroid score 1;
    # the row maximum over the keys is 2
    E = oracle.probe_value_free(np.array([[1.0]]), np.array([[0.0], [2.0]]), np.array([[1.0]]),
                                np.array([0, 2], dtype=np.int32), 1.0)
    want = (math.exp(-1) - math.exp(-2)) ** 2 + (math.exp(-1) - 1.0) ** 2
    assert abs(E[0, 0] - want) < 1e-15
    same = np.tile(np.array([0.3, -1.2, 0.5]), (7, 1))
    E = oracle.probe_value_free(np.array([[0.4, 0.1, -2.0]]), same, same[:1],
                                np.array([0, 7], dtype=np.int32), 0.8)
    assert E[0, 0] == 0.0


def _toy_setup():
    # one query (q = 1, d = 1, scale 1); cluster A keys score 1, 1; B keys 0, 2
    Kp = np.array([[1.0], [1.0], [0.0], [2.0]])
    Vp = np.array([[0.5], [-1.0], [2.0], [3.0]])
    k_off = np.array([0, 2, 4], dtype=np.int32)
    kbar = np.array([[1.0], [1.0]])
    vbar = np.array([[-0.25], [2.5]])
    return np.array([[1.0]]), Kp, Vp, np.array([0, 1], dtype=np.int32), k_off, kbar, vbar


def test_diagnostics_toy_recall_and_exact_output_when_b_is_computed():
    gold = json.load(open(os.path.join(GOLDEN, "toy_example.json")))["printed"]
    Qp, Kp, Vp, q_off, k_off, kbar, vbar = _toy_setup()
    perm = np.array([0], dtype=np.int32)
    for sel, recall_want in (([1], (1 + math.e ** 2) / (2 * math.e + 1 + math.e ** 2)),
                             ([0, 1], 1.0), ([], 0.0)):
        pair_off = np.array([0, len(sel)], dtype=np.int32)
        pair_kc = np.array(sel, dtype=np.int32)
        O, _ = oracle.attend(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, kbar, vbar, perm, 1.0)
        rec, err2, ref2 = oracle.diagnostics(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, O, perm,
                                             1.0, [0])
        assert abs(rec[0] - recall_want) < 1e-12
        if sel:   # B computed: A's keys are identical, so its estimate is exact
            assert err2[0] < 1e-28 and ref2[0] > 0
    # the printed weights give the same share for B
    assert abs(gold["weight_B"] / gold["weight_total"] -
               (1 + math.e ** 2) / (2 * math.e + 1 + math.e ** 2)) < 0.01


def test_diagnostics_full_selection_is_dense_attention():
    g = np.random.default_rng(47)
    N, d = 40, 6
    Qp, Kp, Vp = (g.standard_normal((N, d)) for _ in range(3))
    q_off, k_off = _offsets([15, 25]), _offsets([12, 8, 20])
    kbar = np.stack([Kp[k_off[c]:k_off[c + 1]].mean(0) for c in range(3)])
    vbar = np.stack([Vp[k_off[c]:k_off[c + 1]].mean(0) for c in range(3)])
    pair_off = np.array([0, 3, 6], dtype=np.int32)
    pair_kc = np.array([0, 1, 2, 0, 1, 2], dtype=np.int32)
    perm = g.permutation(N).astype(np.int32)
    O, _ = oracle.attend(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, kbar, vbar, perm, 0.7)
    rows = np.arange(N)
    rec, err2, ref2 = oracle.diagnostics(Qp, Kp, Vp, q_off, k_off, pair_off, pair_kc, O, perm, 0.7,
                                         rows)
    assert np.allclose(rec, 1.0) and np.all(err2 < 1e-25)
    S = Qp @ Kp.T * 0.7
    ref = softmax(S, axis=1) @ Vp
    assert np.allclose(ref2, (ref ** 2).sum(1))

def test_probe_error_equals_its_expansion_and_parts_bound_the_terms():
    """E_ic = sum_t |a vbar - b v_t|^2 equals, term by term, the expansion
    (a-b)^2|vbar|^2 - 2(a-b) b vbar.w_t + b^2|w_t|^2 with w_t = v_t - vbar
    (brute force on a tiny case), and P_ic bounds the terms' absolute values."""
    rng = np.random.default_rng(11)
    d, Nk, Cq, Ck = 8, 40, 3, 4
    q = rng.normal(size=(Cq, d))
    K = rng.normal(size=(Nk, d))
    V = rng.normal(size=(Nk, d)) + 2.0
    off = np.array([0, 7, 7, 22, 40], np.int32)
    kb = np.stack([K[off[c]:off[c + 1]].mean(0) if off[c + 1] > off[c] else np.zeros(d)
                   for c in range(Ck)])
    vb = np.stack([V[off[c]:off[c + 1]].mean(0) if off[c + 1] > off[c] else np.zeros(d)
                   for c in range(Ck)])
    scale = 0.3
    E, S, P = oracle.probe(q, K, V, kb, vb, off, scale, with_parts=True)
    for i in range(Cq):
        m = max(scale * float(q[i] @ K[t]) for t in range(Nk))
        for c in range(Ck):
            a = np.exp(scale * float(q[i] @ kb[c]) - m)
            terms, absum = 0.0, 0.0
            for t in range(off[c], off[c + 1]):
                b = np.exp(scale * float(q[i] @ K[t]) - m)
                w = V[t] - vb[c]
                t1 = (a - b) ** 2 * float(vb[c] @ vb[c])
                t2 = -2.0 * (a - b) * b * float(vb[c] @ w)
                t3 = b * b * float(w @ w)
                terms += t1 + t2 + t3
                absum += abs(t1) + abs(t2) + abs(t3)
            assert abs(E[i, c] - terms) <= 1e-12 * max(1.0, abs(terms))
            assert P[i, c] >= absum * (1 - 1e-12) and P[i, c] >= E[i, c] * (1 - 1e-12)
            if off[c + 1] == off[c]:
                assert E[i, c] == 0.0 and P[i, c] == 0.0
