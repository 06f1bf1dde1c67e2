"""CUDA path vs the CPU oracle, stage by stage, through the C ABI.

Labels, permutations, offsets and routed pairs must be bit-exact when the
oracle is fed the GPU stage's inputs (labels up to documented fp32 near-ties);
floating-point outputs must lie within bounds derived from the fp32 arithmetic
(tests/helpers.py); the final O within rel-L2 1e-2 and max-abs 2e-2 for bf16
and 1e-5 for fp32.
"""
import math

import numpy as np
import pytest

import oracle
from clustered_sparse_attention_b200 import synth
from tests.helpers import (U32, check_assign, np64, probe_tolerance, to_torch,
                           update_tolerance)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _csa():
    import clustered_sparse_attention_b200 as csa
    return csa


SMALL_BF16 = synth.custom_workload("small_bf16", H=2, frames=2, grid_h=32, grid_w=40, d=128,
                                   dtype="bf16", Cq=20, Ck=50, iters=5, density=0.3,
                                   n_centres=32, sigma=0.5, index=50)
RAGGED_BF16_64 = synth.custom_workload("ragged_bf16_d64", H=3, frames=1, grid_h=25, grid_w=41,
                                       d=64, dtype="bf16", Cq=7, Ck=33, iters=3, density=0.25,
                                       n_centres=12, sigma=0.4, index=51)
TINY = synth.WORKLOADS["tiny"]
# the SVG-EAR paper's cluster counts (300 query, 1000 key clusters) on a short
# clip: query clusters of ~16 rows leave most 128-row tiles partial
EAR_COUNTS = synth.custom_workload("ear_counts", H=2, frames=2, grid_h=40, grid_w=60, d=128,
                                   dtype="bf16", Cq=300, Ck=1000, iters=3, density=0.25,
                                   n_centres=64, sigma=0.5, index=54)
# many seeds over few tokens: most tokens of the late k-means++ passes are
# screened out by the triangle bound, so the picks exercise the pruned path
MANY_SEEDS = synth.custom_workload("many_seeds", H=2, frames=2, grid_h=48, grid_w=64, d=128,
                                   dtype="bf16", Cq=16, Ck=600, iters=2, density=0.3,
                                   n_centres=48, sigma=0.5, index=52)


def _inputs(w, heads=None):
    t = {n: synth.layer_tensor(w, n, heads=heads) for n in ("q", "k", "v")}
    return t, {n: to_torch(a, w.dtype) for n, a in t.items()}


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64, MANY_SEEDS],
                         ids=lambda w: w.name)
def test_kmeanspp_stagewise(w):
    csa = _csa()
    host, dev = _inputs(w)
    C = w.Ck
    cent, idx = csa.svgear_kmeanspp_init(dev["k"], C, seed=7)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    cent = cent.cpu().numpy()
    band = 4 * (w.d + 2) * U32
    flips = 0
    for h in range(w.H):
        X = host["k"][0, h]
        own, margin = oracle.kmeanspp(X, C, seed=7, stream=h, follow=idx[0, h])
        assert own[0] == idx[0, h, 0]
        diff = np.nonzero(own != idx[0, h])[0]
        for j in diff:
            assert margin[j] < band, "seed %d of head %d: gpu %d oracle %d margin %.3g" % (
                j, h, idx[0, h, j], own[j], margin[j])
        flips += len(diff)
        assert np.array_equal(cent[0, h], X[idx[0, h]])
    assert flips <= 2


# more heads than resident CTAs, 640 tokens (one partial block) each: many heads have no
# CTA of their own and are served by CTAs homed on other heads
MANY_HEADS = synth.custom_workload("many_heads", H=1200, frames=1, grid_h=16, grid_w=40, d=64,
                                   dtype="bf16", Cq=4, Ck=12, iters=2, density=0.5,
                                   n_centres=8, sigma=0.5, index=55)


def test_kmeanspp_with_more_heads_than_ctas():
    csa = _csa()
    w = MANY_HEADS
    heads = list(range(0, w.H, 97)) + [w.H - 1]
    host, dev = _inputs(w)
    C = w.Ck
    cent, idx = csa.svgear_kmeanspp_init(dev["k"], C, seed=3)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    cent = cent.cpu().numpy()
    band = 4 * (w.d + 2) * U32
    flips = 0
    for h in heads:
        X = host["k"][0, h]
        own, margin = oracle.kmeanspp(X, C, seed=3, stream=h, follow=idx[0, h])
        assert own[0] == idx[0, h, 0]
        diff = np.nonzero(own != idx[0, h])[0]
        for j in diff:
            assert margin[j] < band
        flips += len(diff)
        assert np.array_equal(cent[0, h], X[idx[0, h]])
    assert flips <= 2
    # every head: distinct seeds, all of them tokens of the head
    assert np.all((idx >= 0) & (idx < w.N))
    assert all(len(set(idx[0, h].tolist())) == C for h in range(w.H))


@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64], ids=lambda w: w.name)
def test_assign_matches_oracle(w):
    csa = _csa()
    host, dev = _inputs(w)
    g = np.random.default_rng(1)
    for C in (w.Cq, w.Ck, 129):
        C = min(C, w.N)
        cent = np.stack([host["q"][0, h][g.choice(w.N, C, replace=False)] for h in range(w.H)])[None]
        cent = cent + 0.01 * g.standard_normal(cent.shape).astype(np.float32)
        lab = csa.svgear_kmeans_assign(dev["q"], torch.from_numpy(cent).cuda()).cpu().numpy()
        flips = sum(check_assign(host["q"][0, h], cent[0, h], lab[0, h]) for h in range(w.H))
        assert flips <= max(2, w.N * w.H // 5000)


def test_assign_exact_ties_take_lowest_index():
    csa = _csa()
    X = torch.zeros((1, 1, 300, 64), device="cuda")
    X[0, 0, :, 0] = torch.arange(300, device="cuda").float() % 3
    cent = torch.zeros((1, 1, 200, 64), device="cuda")
    cent[0, 0, :, 0] = (torch.arange(200, device="cuda") % 3).float()   # 3 values, many duplicates
    lab = csa.svgear_kmeans_assign(X, cent).cpu().numpy()[0, 0]
    assert np.array_equal(lab, np.arange(300) % 3)


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("C", [16, 100, 256, 257, 500, 1000])
def test_tensor_core_assign_over_centroid_chunks(d, C):
    # bf16 tokens take the tcgen05 kernel: one to four centroid chunks of up
    # to 256 columns, widths rounded to 16, a ragged last token tile
    csa = _csa()
    w = synth.custom_workload("assign_tc_d%d" % d, H=2, frames=2, grid_h=30, grid_w=50, d=d,
                              dtype="bf16", Cq=C, Ck=C, iters=1, density=0.3, n_centres=40,
                              sigma=0.5, index=53)
    host, dev = _inputs(w)
    g = np.random.default_rng(C + d)
    cent = np.stack([host["k"][0, h][g.choice(w.N, C, replace=False)] for h in range(w.H)])[None]
    cent = cent + 0.01 * g.standard_normal(cent.shape).astype(np.float32)
    lab = csa.svgear_kmeans_assign(dev["k"], torch.from_numpy(cent).cuda(),
                                   check_status=True).cpu().numpy()
    flips = sum(check_assign(host["k"][0, h], cent[0, h], lab[0, h]) for h in range(w.H))
    assert flips <= max(2, w.N * w.H // 5000)


def test_tensor_core_assign_exact_ties_take_lowest_index():
    csa = _csa()
    X = torch.zeros((1, 1, 300, 128), dtype=torch.bfloat16, device="cuda")
    X[0, 0, :, 0] = (torch.arange(300, device="cuda") % 3).to(torch.bfloat16)
    cent = torch.zeros((1, 1, 300, 128), device="cuda")
    cent[0, 0, :, 0] = (torch.arange(300, device="cuda") % 3).float()   # two chunks of duplicates
    cent[0, 0, :, 5] = 1.0 / 3.0                                        # not on the bf16 grid
    lab = csa.svgear_kmeans_assign(X, cent, check_status=True).cpu().numpy()[0, 0]
    assert np.array_equal(lab, np.arange(300) % 3)


@pytest.mark.parametrize("N,C", [(5000, 300), (1024, 1), (777, 777), (5000, 4096), (3000, 129)])
def test_label_sort_bit_exact(N, C):
    csa = _csa()
    g = np.random.default_rng(N + C)
    labels = g.integers(0, C, (2, 3, N)).astype(np.int32)
    if C > 10:
        labels[labels % 7 == 3] = 0          # leaves some clusters empty
    perm, off = csa.svgear_label_sort(torch.from_numpy(labels).cuda(), C)
    perm, off = perm.cpu().numpy(), off.cpu().numpy()
    for b in range(2):
        for h in range(3):
            p_o, o_o = oracle.stable_sort(labels[b, h], C)
            assert np.array_equal(perm[b, h], p_o)
            assert np.array_equal(off[b, h], o_o)


@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64], ids=lambda w: w.name)
def test_update_matches_oracle(w):
    csa = _csa()
    host, dev = _inputs(w)
    g = np.random.default_rng(2)
    C = w.Ck
    labels = g.integers(0, C - 3, (1, w.H, w.N)).astype(np.int32)   # last clusters empty
    prev = g.standard_normal((1, w.H, C, w.d)).astype(np.float32)
    out = csa.svgear_kmeans_update(dev["k"], torch.from_numpy(labels).cuda(),
                                   torch.from_numpy(prev).cuda()).cpu().numpy()
    for h in range(w.H):
        ref = oracle.update(host["k"][0, h], labels[0, h], prev[0, h])
        tol = update_tolerance(host["k"][0, h], labels[0, h], C)
        assert np.all(np.abs(out[0, h] - ref) <= tol)
        assert np.array_equal(out[0, h, C - 3:], prev[0, h, C - 3:])


@pytest.mark.parametrize("w", [TINY, SMALL_BF16], ids=lambda w: w.name)
def test_cluster_iteration_chain(w):
    """cluster(iters=k) returns centroids c^k; cluster(iters=k+1) must hold
    labels = argmin against c^k, centroids = means of those labels, and the
    stable sort of those labels; Xp = X[perm]."""
    csa = _csa()
    host, dev = _inputs(w)
    C = w.Ck
    prev = csa.svgear_cluster(dev["k"], C, 1, seed=11)
    for k in (1, 2, 3):
        nxt = csa.svgear_cluster(dev["k"], C, k + 1, seed=11)
        torch.cuda.synchronize()
        for h in range(w.H):
            X = host["k"][0, h]
            cprev = prev.centroids.cpu().numpy()[0, h]
            lab = nxt.labels.cpu().numpy()[0, h]
            check_assign(X, cprev, lab)
            p_o, o_o = oracle.stable_sort(lab, C)
            assert np.array_equal(nxt.perm.cpu().numpy()[0, h], p_o)
            assert np.array_equal(nxt.offsets.cpu().numpy()[0, h], o_o)
            ref = oracle.update(X, lab, cprev)
            assert np.all(np.abs(nxt.centroids.cpu().numpy()[0, h] - ref)
                          <= update_tolerance(X, lab, C))
            Xp = np64(nxt.Xp)[0, h]
            assert np.array_equal(Xp, X[p_o].astype(np.float64))
        prev = nxt


def test_warm_start_is_one_round_from_the_cache():
    csa = _csa()
    w = SMALL_BF16
    host, dev = _inputs(w)
    cold = csa.svgear_cluster(dev["q"], w.Cq, 3, seed=5)
    warm = csa.svgear_cluster(dev["q"], w.Cq, 1, warm_centroids=cold.centroids.clone())
    torch.cuda.synchronize()
    for h in range(w.H):
        check_assign(host["q"][0, h], cold.centroids.cpu().numpy()[0, h],
                     warm.labels.cpu().numpy()[0, h])


WARM_SEQ = synth.custom_workload("warm_seq", H=2, frames=2, grid_h=32, grid_w=40, d=128,
                                  dtype="bf16", Cq=20, Ck=50, iters=5, density=0.25,
                                  n_centres=32, sigma=0.5, index=55)


@pytest.mark.parametrize("density", [0.1, 0.3])
def test_warm_sequence_stagewise(density):
    """The centroid cache over a drifting sequence (SVG2 section 3.4, fast
    k-means with centroid cache): step 0 clusters cold; each later step's
    inputs drift by 0.05 N(0,1) per element and Q and K are clustered with one
    round from the previous step's centroids, then routed and attended.  Every
    stage of every step is checked against the oracle fed that stage's GPU
    inputs: labels against the cached centroids, the sort, the centroid
    update, the permuted copies, the value centroids, the pairs given the
    GPU's errors, and O."""
    csa = _csa()
    w = WARM_SEQ
    warm = {"q": None, "k": None}
    for step in range(4):
        host = {n: synth.layer_tensor(w, n, step=step) for n in ("q", "k", "v")}
        dev = {n: to_torch(a, w.dtype) for n, a in host.items()}
        cl = {}
        for name, C, sd in (("q", w.Cq, 0), ("k", w.Ck, 1)):
            if step == 0:
                cl[name] = csa.svgear_cluster(dev[name], C, w.iters, seed=sd, check_status=True)
            else:
                cl[name] = csa.svgear_cluster(dev[name], C, 1, warm_centroids=warm[name].clone(),
                                              check_status=True)
        cq, ck = cl["q"], cl["k"]
        Vp = csa.svgear_permute(dev["v"], ck.perm)
        vbar = csa.svgear_centroids(Vp, ck.offsets, w.Ck)
        po, pk, E = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets,
                                     ck.Xp, Vp, density, w.scale, return_errors=True)
        O = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids,
                              vbar, cq.perm, w.scale, check_status=True)
        torch.cuda.synchronize()
        for h in range(w.H):
            for name, C in (("q", w.Cq), ("k", w.Ck)):
                c = cl[name]
                X = host[name][0, h]
                lab = c.labels.cpu().numpy()[0, h]
                cents = c.centroids.cpu().numpy()[0, h]
                if step > 0:   # one round from the cache: argmin against it
                    check_assign(X, warm[name].cpu().numpy()[0, h], lab)
                p_o, o_o = oracle.stable_sort(lab, C)
                assert np.array_equal(c.perm.cpu().numpy()[0, h], p_o)
                assert np.array_equal(c.offsets.cpu().numpy()[0, h], o_o)
                prev = warm[name].cpu().numpy()[0, h] if step > 0 else cents
                ref = oracle.update(X, lab, prev)
                assert np.all(np.abs(cents - ref) <= update_tolerance(X, lab, C))
                assert np.array_equal(np64(c.Xp)[0, h], X[p_o].astype(np.float64))
            k_off = ck.offsets.cpu().numpy()[0, h]
            V = host["v"][0, h][ck.perm.cpu().numpy()[0, h]]
            lab_k = np.repeat(np.arange(w.Ck), np.diff(k_off))
            assert np.all(np.abs(vbar.cpu().numpy()[0, h] - oracle.segment_mean(V, k_off))
                          <= update_tolerance(V, lab_k, w.Ck))
            ref_off, ref_kc = oracle.route(E.cpu().numpy()[0, h], cq.offsets.cpu().numpy()[0, h],
                                           k_off, w.N, density)
            got_off = po.cpu().numpy()[0, h]
            assert np.array_equal(got_off, ref_off)
            assert np.array_equal(pk.cpu().numpy()[0, h][:got_off[-1]], ref_kc)
            Oo, _ = oracle.attend(np64(cq.Xp)[0, h], np64(ck.Xp)[0, h], np64(Vp)[0, h],
                                  cq.offsets.cpu().numpy()[0, h], k_off, got_off,
                                  pk.cpu().numpy()[0, h], ck.centroids.cpu().numpy()[0, h],
                                  vbar.cpu().numpy()[0, h], cq.perm.cpu().numpy()[0, h], w.scale)
            Og = np64(O)[0, h]
            assert _rel_l2(Og, Oo) <= 1e-2 and np.abs(Og - Oo).max() <= 2e-2
        warm = {"q": cq.centroids, "k": ck.centroids}


def _hand_offsets(N, C, g):
    """Segment sizes that stress the position split (chunks of 512): long
    segments over several chunks, ends exactly on chunk edges, empty
    segments first, in the middle and last, a single segment of one row."""
    sizes = np.zeros(C, dtype=np.int64)
    fixed = [0, 1, 511, 1, 1536, 0, 512, 0, 3000, 7]
    sizes[:len(fixed)] = fixed[:C]
    rest = N - int(sizes.sum())
    free = np.arange(len(fixed), C - 1)             # the last segment stays empty
    cut = np.sort(g.choice(rest + 1, len(free) - 1, replace=True)) if len(free) > 1 else []
    parts = np.diff(np.concatenate([[0], cut, [rest]]))
    sizes[free] = parts
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    assert off[-1] == N and sizes[-1] == 0
    return off


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 128)])
def test_segment_means_across_position_chunks(dtype, d):
    """Means of segments that cross the 512-position chunks of the split
    kernel: the gathered form (k-means update, rows perm[p]) and the
    contiguous form (value centroids on X[perm]) sum the same values in the
    same order, so they agree bit for bit; both within the fp32 bound of the
    oracle's means, and identical from run to run."""
    csa = _csa()
    g = np.random.default_rng(17)
    B, H, N, C = 1, 2, 9000 + 77, 40
    X = g.standard_normal((B, H, N, d)).astype(np.float32)
    if dtype == "bf16":
        X = synth.round_to_bf16(X)
    offs = np.stack([_hand_offsets(N, C, g) for _ in range(H)])[None]
    labels = np.zeros((B, H, N), dtype=np.int32)
    perm = np.zeros((B, H, N), dtype=np.int32)
    for h in range(H):
        sizes = np.diff(offs[0, h])
        lab_sorted = np.repeat(np.arange(C), sizes).astype(np.int32)
        p = g.permutation(N).astype(np.int32)          # token perm[i] sits at position i
        perm[0, h] = p
        labels[0, h, p] = lab_sorted
    Xd = to_torch(X, dtype)
    prev = g.standard_normal((B, H, C, d)).astype(np.float32)
    upd = csa.svgear_kmeans_update(Xd, torch.from_numpy(labels).cuda(),
                                   torch.from_numpy(prev).cuda())
    upd2 = csa.svgear_kmeans_update(Xd, torch.from_numpy(labels).cuda(),
                                    torch.from_numpy(prev).cuda())
    Xp = csa.svgear_permute(Xd, torch.from_numpy(perm).cuda())
    cen = csa.svgear_centroids(Xp, torch.from_numpy(offs).cuda(), C)
    torch.cuda.synchronize()
    assert torch.equal(upd, upd2)
    u, c = upd.cpu().numpy(), cen.cpu().numpy()
    for h in range(H):
        sizes = np.diff(offs[0, h])
        full = sizes > 0
        # the update's sort is stable, so its perm lists tokens of a cluster in
        # increasing index; compare with the contiguous form on that order
        ref = oracle.segment_mean(X[0, h][perm[0, h]], offs[0, h])
        lab_sorted = np.repeat(np.arange(C), sizes)
        tol = update_tolerance(X[0, h][perm[0, h]], lab_sorted, C)
        assert np.all(np.abs(c[0, h] - ref) <= tol)
        assert np.all(np.abs(u[0, h][full] - ref[full]) <= tol[full])
        assert np.all(c[0, h][~full] == 0)                       # empty: zeros
        assert np.array_equal(u[0, h][~full], prev[0, h][~full])  # empty: previous row
        p_o, o_o = oracle.stable_sort(labels[0, h], C)
        assert np.array_equal(o_o, offs[0, h])
    # the gathered form in the sort's own order equals the contiguous form
    # on the same order, bit for bit
    ps, _ = csa.svgear_label_sort(torch.from_numpy(labels).cuda(), C)
    cen_s = csa.svgear_centroids(csa.svgear_permute(Xd, ps), torch.from_numpy(offs).cuda(), C)
    torch.cuda.synchronize()
    full = np.diff(offs[0], axis=-1) > 0
    assert np.array_equal(cen_s.cpu().numpy()[0][full], u[0][full])


@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64], ids=lambda w: w.name)
def test_permute_and_value_centroids(w):
    csa = _csa()
    host, dev = _inputs(w)
    ck = csa.svgear_cluster(dev["k"], w.Ck, 2, seed=3)
    Vp = csa.svgear_permute(dev["v"], ck.perm)
    vbar = csa.svgear_centroids(Vp, ck.offsets, w.Ck)
    torch.cuda.synchronize()
    for h in range(w.H):
        perm = ck.perm.cpu().numpy()[0, h]
        off = ck.offsets.cpu().numpy()[0, h]
        V = host["v"][0, h]
        assert np.array_equal(np64(Vp)[0, h], V[perm].astype(np.float64))
        ref = oracle.segment_mean(V[perm], off)
        lab = np.repeat(np.arange(w.Ck), np.diff(off))
        tol = update_tolerance(V[perm], lab, w.Ck)
        got = vbar.cpu().numpy()[0, h]
        assert np.all(np.abs(got - ref) <= tol)
        assert np.all(got[np.diff(off) == 0] == 0)


def _clustered(w, dev, seed=3):
    csa = _csa()
    cq = csa.svgear_cluster(dev["q"], w.Cq, 2, seed=2 * seed)
    ck = csa.svgear_cluster(dev["k"], w.Ck, 2, seed=2 * seed + 1)
    Vp = csa.svgear_permute(dev["v"], ck.perm)
    vbar = csa.svgear_centroids(Vp, ck.offsets, w.Ck)
    return cq, ck, Vp, vbar


@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64, EAR_COUNTS],
                         ids=lambda w: w.name)
def test_probe_matches_oracle(w):
    csa = _csa()
    host, dev = _inputs(w)
    cq, ck, Vp, vbar = _clustered(w, dev)
    E = csa.svgear_probe(cq.centroids, ck.Xp, Vp, ck.centroids, vbar, ck.offsets, w.scale)
    torch.cuda.synchronize()
    for h in range(w.H):
        qbar = cq.centroids.cpu().numpy()[0, h]
        Kp, Vph = np64(ck.Xp)[0, h], np64(Vp)[0, h]
        Eo, So, Po = oracle.probe(qbar, Kp, Vph, ck.centroids.cpu().numpy()[0, h],
                                  vbar.cpu().numpy()[0, h], ck.offsets.cpu().numpy()[0, h],
                                  w.scale, with_parts=True)
        Eg = E.cpu().numpy()[0, h].astype(np.float64)
        tol = probe_tolerance(qbar, Kp, Eo, So, w.scale, P=Po)
        assert np.all(np.abs(Eg - Eo) <= tol), float(np.max(np.abs(Eg - Eo) / tol))
        empty = np.diff(ck.offsets.cpu().numpy()[0, h]) == 0
        assert np.all(Eg[:, empty] == 0)


@pytest.mark.parametrize("density", [0.05, 0.25, 0.5, 1.0])
@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64, EAR_COUNTS],
                         ids=lambda w: w.name)
def test_route_bit_exact_given_gpu_errors(w, density):
    csa = _csa()
    host, dev = _inputs(w)
    cq, ck, Vp, vbar = _clustered(w, dev)
    po, pk, E = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets, ck.Xp,
                                 Vp, density, w.scale, return_errors=True)
    torch.cuda.synchronize()
    for h in range(w.H):
        ref_off, ref_kc = oracle.route(E.cpu().numpy()[0, h], cq.offsets.cpu().numpy()[0, h],
                                       ck.offsets.cpu().numpy()[0, h], w.N, density)
        got_off = po.cpu().numpy()[0, h]
        assert np.array_equal(got_off, ref_off)
        assert np.array_equal(pk.cpu().numpy()[0, h][:got_off[-1]], ref_kc)
    # the standalone select on the same errors gives the same pairs
    po2, pk2 = csa.svgear_route_select(E, cq.offsets, ck.offsets, w.N, density)
    assert torch.equal(po2, po)
    n = int(po[0, 0, -1])
    assert torch.equal(pk2[0, 0, :n], pk[0, 0, :n])


def _check_attend(w, dev, density, rows=None):
    csa = _csa()
    cq, ck, Vp, vbar = _clustered(w, dev)
    po, pk = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets, ck.Xp,
                              Vp, density, w.scale)
    O = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids, vbar,
                          cq.perm, w.scale, check_status=True)
    torch.cuda.synchronize()
    Og = np64(O)
    worst = (0.0, 0.0)
    for h in range(w.H):
        args = (np64(cq.Xp)[0, h], np64(ck.Xp)[0, h], np64(Vp)[0, h],
                cq.offsets.cpu().numpy()[0, h], ck.offsets.cpu().numpy()[0, h],
                po.cpu().numpy()[0, h], pk.cpu().numpy()[0, h],
                ck.centroids.cpu().numpy()[0, h], vbar.cpu().numpy()[0, h],
                cq.perm.cpu().numpy()[0, h])
        if rows is None:
            Oo, _ = oracle.attend(*args, w.scale)
            Gh = Og[0, h]
        else:
            Oo, _ = oracle.attend(*args, w.scale, rows=rows)
            Gh = Og[0, h][cq.perm.cpu().numpy()[0, h][rows]]
        worst = (max(worst[0], _rel_l2(Gh, Oo)), max(worst[1], float(np.abs(Gh - Oo).max())))
    return worst


def test_attend_fp32_tiny_within_1e5():
    host, dev = _inputs(TINY)
    rel, mx = _check_attend(TINY, dev, TINY.density)
    assert rel <= 1e-5 and mx <= 1e-5, (rel, mx)


@pytest.mark.parametrize("density", [0.1, 0.3, 1.0])
@pytest.mark.parametrize("w", [SMALL_BF16, RAGGED_BF16_64, EAR_COUNTS], ids=lambda w: w.name)
def test_attend_bf16_within_tolerance(w, density):
    host, dev = _inputs(w)
    rel, mx = _check_attend(w, dev, density)
    assert rel <= 1e-2 and mx <= 2e-2, (rel, mx)


def test_density_one_equals_dense_attention():
    csa = _csa()
    w = SMALL_BF16
    host, dev = _inputs(w)
    out = csa.layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, 3, 1.0, w.scale, seed=1)
    torch.cuda.synchronize()
    O = np64(out["O"])
    for h in range(w.H):
        Q, K, V = (host[n][0, h].astype(np.float64) for n in ("q", "k", "v"))
        S = Q @ K.T * w.scale
        S -= S.max(1, keepdims=True)
        P = np.exp(S)
        ref = (P / P.sum(1, keepdims=True)) @ V
        assert _rel_l2(O[0, h], ref) <= 1e-2 and np.abs(O[0, h] - ref).max() <= 2e-2


def test_singleton_key_clusters_make_compensation_exact():
    csa = _csa()
    g = np.random.default_rng(4)
    N, d = 256, 64
    Q = g.standard_normal((1, 1, N, d)).astype(np.float32)
    K = g.standard_normal((1, 1, N, d)).astype(np.float32)
    V = g.standard_normal((1, 1, N, d)).astype(np.float32)
    dq, dk, dv = (torch.from_numpy(a).cuda() for a in (Q, K, V))
    out = csa.layer(dq, dk, dv, 8, N, 2, 0.2, d ** -0.5, seed=2)   # Ck = N: all singletons
    torch.cuda.synchronize()
    S = Q[0, 0].astype(np.float64) @ K[0, 0].T.astype(np.float64) * d ** -0.5
    S -= S.max(1, keepdims=True)
    P = np.exp(S)
    ref = (P / P.sum(1, keepdims=True)) @ V[0, 0]
    got = np64(out["O"])[0, 0]
    assert _rel_l2(got, ref) <= 1e-5 and np.abs(got - ref).max() <= 1e-5


def test_tiny_layer_end_to_end_stagewise():
    """The tiny fp32 workload through csa.layer, every stage checked."""
    csa = _csa()
    w = TINY
    host, dev = _inputs(w)
    out = csa.layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, w.iters, w.density, w.scale, seed=0)
    torch.cuda.synchronize()
    cq, ck = out["q"], out["k"]
    for name, cl, X, C in (("q", cq, host["q"][0, 0], w.Cq), ("k", ck, host["k"][0, 0], w.Ck)):
        lab = cl.labels.cpu().numpy()[0, 0]
        p_o, o_o = oracle.stable_sort(lab, C)
        assert np.array_equal(cl.perm.cpu().numpy()[0, 0], p_o)
        assert np.array_equal(cl.offsets.cpu().numpy()[0, 0], o_o)
        ref = oracle.segment_mean(X[p_o], o_o, prev=cl.centroids.cpu().numpy()[0, 0])
        assert np.all(np.abs(cl.centroids.cpu().numpy()[0, 0] - ref)
                      <= update_tolerance(X, lab, C))
    pairs = int(out["pair_off"][0, 0, -1])
    assert pairs > 0
    Oo, _ = oracle.attend(np64(cq.Xp)[0, 0], np64(ck.Xp)[0, 0], np64(out["Vp"])[0, 0],
                          cq.offsets.cpu().numpy()[0, 0], ck.offsets.cpu().numpy()[0, 0],
                          out["pair_off"].cpu().numpy()[0, 0],
                          out["pair_kc"].cpu().numpy()[0, 0][:pairs],
                          ck.centroids.cpu().numpy()[0, 0], out["vbar"].cpu().numpy()[0, 0],
                          cq.perm.cpu().numpy()[0, 0], w.scale)
    Og = np64(out["O"])[0, 0]
    assert _rel_l2(Og, Oo) <= 1e-5 and np.abs(Og - Oo).max() <= 1e-5


def test_invalid_arguments_are_rejected_before_launch():
    csa = _csa()
    from clustered_sparse_attention_b200 import _lib
    X = torch.zeros((1, 1, 100, 96), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(_lib.SvgearError) as e:
        csa.svgear_kmeans_assign(X, torch.zeros((1, 1, 4, 96), device="cuda"))
    assert e.value.status == _lib.ERR_UNSUPPORTED
    X = torch.zeros((1, 1, 100, 64), device="cuda")
    with pytest.raises(_lib.SvgearError) as e:
        csa.svgear_cluster(X, 101, 1)
    assert e.value.status == _lib.ERR_INVALID_ARG
    with pytest.raises(_lib.SvgearError):
        csa.svgear_cluster(X, 10, 0)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("case", [
    # (query cluster sizes, key cluster sizes, selected key clusters per query cluster)
    ([128], [64, 64], [[0, 1]]),                       # one key tile, no compensation
    ([128], [64, 64], [[1]]),                          # partial key tile + one compensation tile
    ([200], [100, 150, 7, 300], [[0, 1, 3]]),          # 5 key tiles, ragged query tile
    ([1, 129, 0, 300], [130, 1, 0, 250, 40], [[2], [0, 1, 3], [], [4]]),
    ([64, 64], [5] * 300, [list(range(0, 300, 2)), []]),   # 3 compensation tiles
    ([128], [128, 128, 128], [[0, 1, 2]], "spiky"),    # half the rows rescale O mid-row
    ([256], [100, 60, 200], [[2], [0]], "spiky"),
    # one key tile of 60 keys, no compensation: the upper 64-key half of the
    # tile never holds a key (its softmax state stays empty and merges as zero)
    ([100], [10, 50], [[0, 1]]),
    # 20 keys and one compensated cluster: both tiles only in the lower half
    ([130], [20, 30], [[0]]),
    # 40 keys, then 100 compensated singletons: the upper half meets its first
    # valid column in the second tile, with nothing summed before it
    ([128], [40] + [1] * 100, [[0]]),
])
def test_attend_kernel_on_handmade_layouts(D, case):
    """The attention kernel alone on hand-built segments and pair lists,
    against the oracle (bf16 inputs, fp32 centroids)."""
    csa = _csa()
    qs, ks, sel = case[:3]
    spiky = len(case) > 3
    g = np.random.default_rng(len(qs) * 7 + D)
    Nq, Nk = sum(qs), sum(ks)
    Cq, Ck = len(qs), len(ks)
    if spiky:    # route pairs per query cluster: the spiky cases use one list per cluster
        sel = sel[:Cq]
    from clustered_sparse_attention_b200.synth import round_to_bf16
    Q0 = g.standard_normal((Nq, D)).astype(np.float32)
    K0 = g.standard_normal((Nk, D)).astype(np.float32)
    if spiky:
        # rows with an even index see a score jump of ~8.2 (log2 units) in the
        # keys after the first tile; odd rows do not -> divergent rescales
        Q0[::2, 0] = 20.0
        K0[:, 0] = 0.0
        K0[128:, 0] = 4.0 * (D / 128) ** 0.5
    Qp = round_to_bf16(Q0)
    Kp = round_to_bf16(K0)
    Vp = round_to_bf16(g.standard_normal((Nk, D)).astype(np.float32))
    q_off = np.concatenate([[0], np.cumsum(qs)]).astype(np.int32)
    k_off = np.concatenate([[0], np.cumsum(ks)]).astype(np.int32)
    pair_off = np.concatenate([[0], np.cumsum([len(s) for s in sel])]).astype(np.int32)
    pair_kc = np.zeros(Cq * Ck, np.int32)
    flat = [c for s in sel for c in s]
    pair_kc[:len(flat)] = flat
    kbar = oracle.segment_mean(Kp, k_off).astype(np.float32)
    vbar = oracle.segment_mean(Vp, k_off).astype(np.float32)
    q_perm = g.permutation(Nq).astype(np.int32)
    scale = D ** -0.5

    def dev(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.to(dt) if dt is not None else t).cuda()

    O = csa.svgear_attend(dev(Qp[None, None], torch.bfloat16), dev(Kp[None, None], torch.bfloat16),
                          dev(Vp[None, None], torch.bfloat16), dev(q_off[None, None]),
                          dev(k_off[None, None]), dev(pair_off[None, None]), dev(pair_kc[None, None]),
                          dev(kbar[None, None]), dev(vbar[None, None]), dev(q_perm[None, None]),
                          scale, check_status=True)
    torch.cuda.synchronize()
    Oo, _ = oracle.attend(Qp, Kp, Vp, q_off, k_off, pair_off, np.array(flat, np.int32), kbar, vbar,
                          q_perm, scale)
    Og = np64(O)[0, 0]
    assert _rel_l2(Og, Oo) <= 1e-2 and np.abs(Og - Oo).max() <= 2e-2, (_rel_l2(Og, Oo),
                                                                        np.abs(Og - Oo).max())


def test_cluster_fixed_point_gives_the_same_result_as_more_rounds():
    """Once a round moves no label, later rounds are exact no-ops: 60 and 120
    rounds must agree bit for bit, and one more oracle round moves nothing."""
    csa = _csa()
    w = SMALL_BF16
    host, dev = _inputs(w)
    a = csa.svgear_cluster(dev["k"], w.Ck, 60, seed=4)
    b = csa.svgear_cluster(dev["k"], w.Ck, 120, seed=4)
    torch.cuda.synchronize()
    for f in ("labels", "perm", "offsets", "centroids", "Xp"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    for h in range(w.H):
        check_assign(host["k"][0, h], b.centroids.cpu().numpy()[0, h], b.labels.cpu().numpy()[0, h])


# ---------------------------------------------------------------------------
# Top-p budget (SVG2 summary, section 3.4, top-p selection; SVG-EAR blog,
# budget paragraph)
# ---------------------------------------------------------------------------
def _check_budgets(gpu, qbar, kbar, q_off, k_off, p, scale):
    """GPU budgets equal the oracle's except where the running weight crosses
    p within fp64 rounding of it (counted and returned)."""
    ref, margin = oracle.topp_budget(qbar, kbar, q_off, k_off, p, scale)
    bad = np.nonzero(ref != gpu)[0]
    for i in bad:
        assert margin[i] < 1e-9, (i, int(gpu[i]), int(ref[i]), margin[i])
    return len(bad)


@pytest.mark.parametrize("p", [0.3, 0.9, 1.0])
@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64, EAR_COUNTS], ids=lambda w: w.name)
def test_topp_budget_matches_oracle(w, p):
    csa = _csa()
    host, dev = _inputs(w)
    cq, ck, Vp, vbar = _clustered(w, dev)
    budget = csa.svgear_topp_budget(cq.centroids, cq.offsets, ck.centroids, ck.offsets, w.N, p,
                                    w.scale).cpu().numpy()
    qb, kb = cq.centroids.cpu().numpy(), ck.centroids.cpu().numpy()
    qo, ko = cq.offsets.cpu().numpy(), ck.offsets.cpu().numpy()
    flips = sum(_check_budgets(budget[0, h], qb[0, h], kb[0, h], qo[0, h], ko[0, h], p, w.scale)
                for h in range(w.H))
    assert flips <= 1
    if p == 1.0:
        nonempty_rows = np.diff(qo, axis=-1) > 0
        assert np.all(budget[nonempty_rows] == w.N)


@pytest.mark.parametrize("w", [SMALL_BF16, EAR_COUNTS], ids=lambda w: w.name)
def test_route_topp_bit_exact_given_gpu_errors_and_budgets(w):
    csa = _csa()
    host, dev = _inputs(w)
    cq, ck, Vp, vbar = _clustered(w, dev)
    po, pk, budget, E = csa.svgear_route_topp(cq.centroids, cq.offsets, ck.centroids, vbar,
                                              ck.offsets, ck.Xp, Vp, 0.9, w.scale,
                                              return_errors=True)
    torch.cuda.synchronize()
    b = budget.cpu().numpy()
    for h in range(w.H):
        ref_off, ref_kc = oracle.route(E.cpu().numpy()[0, h], cq.offsets.cpu().numpy()[0, h],
                                       ck.offsets.cpu().numpy()[0, h], w.N, 1.0,
                                       budgets=b[0, h].astype(np.int64))
        got = po.cpu().numpy()[0, h]
        assert np.array_equal(got, ref_off)
        assert np.array_equal(pk.cpu().numpy()[0, h][:got[-1]], ref_kc)
        # every taken set fits its budget
        sizes = np.diff(ck.offsets.cpu().numpy()[0, h])
        for i in range(w.Cq):
            assert sizes[ref_kc[ref_off[i]:ref_off[i + 1]]].sum() <= b[0, h, i]
    # the standalone select with the same budgets gives the same pairs
    po2, pk2 = csa.svgear_route_select_budget(E, cq.offsets, ck.offsets, w.N, budget)
    assert torch.equal(po2, po)


def test_layer_with_topp_budget_end_to_end():
    csa = _csa()
    w = SMALL_BF16
    host, dev = _inputs(w)
    out = csa.layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, 3, None, w.scale, seed=2, topp=0.9)
    torch.cuda.synchronize()
    cq, ck = out["q"], out["k"]
    for h in range(w.H):
        args = (np64(cq.Xp)[0, h], np64(ck.Xp)[0, h], np64(out["Vp"])[0, h],
                cq.offsets.cpu().numpy()[0, h], ck.offsets.cpu().numpy()[0, h],
                out["pair_off"].cpu().numpy()[0, h], out["pair_kc"].cpu().numpy()[0, h],
                ck.centroids.cpu().numpy()[0, h], out["vbar"].cpu().numpy()[0, h],
                cq.perm.cpu().numpy()[0, h])
        Oo, _ = oracle.attend(*args, w.scale)
        Og = np64(out["O"])[0, h]
        assert _rel_l2(Og, Oo) <= 1e-2 and np.abs(Og - Oo).max() <= 2e-2


@pytest.mark.parametrize("w", [TINY, SMALL_BF16], ids=lambda w: w.name)
def test_layer_from_host_buffers_equals_the_device_layer(w):
    """layer_host (inputs copied on a side stream while the first stages run)
    returns exactly the device layer's O, and the same every time."""
    csa = _csa()
    host, dev = _inputs(w)
    ref = csa.layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, w.iters, w.density, w.scale,
                    seed=1)["O"].cpu()
    hp = {n: t.cpu().pin_memory() for n, t in dev.items()}
    out = torch.empty(ref.shape, dtype=ref.dtype).pin_memory()
    for _ in range(3):
        res = csa.layer_host(hp["q"], hp["k"], hp["v"], w.Cq, w.Ck, w.iters, w.density,
                             w.scale, seed=1, out=out)
        torch.cuda.synchronize()
        assert res["O_host"] is out
        assert torch.equal(out, ref)


# ---------------------------------------------------------------------------
# Variance-corrected compensation (SVG-EAR blog, variance paragraph)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64], ids=lambda w: w.name)
def test_key_variance_matches_oracle(w):
    csa = _csa()
    host, dev = _inputs(w)
    cq, ck, Vp, vbar = _clustered(w, dev)
    kvar = csa.svgear_key_variance(ck.Xp, ck.offsets, w.Ck).cpu().numpy()
    for h in range(w.H):
        Kp = np64(ck.Xp)[0, h]
        off = ck.offsets.cpu().numpy()[0, h]
        ref = oracle.segment_var(Kp, off)
        # fp32 two-pass sums: relative to the segment's second moment
        m2 = oracle.segment_mean(Kp ** 2, off, prev=np.zeros_like(ref))
        assert np.all(np.abs(kvar[0, h] - ref) <= 2e-5 * m2 + 1e-7)


def _check_attend_var(w, dev, lam, density=None, zero_budget=False):
    csa = _csa()
    cq, ck, Vp, vbar = _clustered(w, dev)
    if zero_budget:   # every cluster compensated: no exact tile at all
        po, pk = csa.svgear_route_select_budget(
            torch.zeros((1, w.H, w.Cq, w.Ck), dtype=torch.float32, device="cuda"), cq.offsets,
            ck.offsets, w.N, torch.zeros((1, w.H, w.Cq), dtype=torch.int32, device="cuda"))
    else:
        po, pk = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets, ck.Xp,
                                  Vp, density, w.scale)
    kvar = csa.svgear_key_variance(ck.Xp, ck.offsets, w.Ck)
    O = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids, vbar,
                          cq.perm, w.scale, check_status=True, kvar=kvar, lam=lam)
    O0 = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids, vbar,
                           cq.perm, w.scale, check_status=True)
    torch.cuda.synchronize()
    Og, O0g = np64(O), np64(O0)
    worst = (0.0, 0.0)
    for h in range(w.H):
        Oo, _ = oracle.attend(np64(cq.Xp)[0, h], np64(ck.Xp)[0, h], np64(Vp)[0, h],
                              cq.offsets.cpu().numpy()[0, h], ck.offsets.cpu().numpy()[0, h],
                              po.cpu().numpy()[0, h], pk.cpu().numpy()[0, h],
                              ck.centroids.cpu().numpy()[0, h], vbar.cpu().numpy()[0, h],
                              cq.perm.cpu().numpy()[0, h], w.scale,
                              kvar=kvar.cpu().numpy()[0, h], lam=lam)
        worst = (max(worst[0], _rel_l2(Og[0, h], Oo)),
                 max(worst[1], float(np.abs(Og[0, h] - Oo).max())))
    # the term moves the output well beyond the parity tolerance of the path
    assert _rel_l2(Og, O0g) > (5e-5 if w.dtype == "f32" else 1e-3)
    return worst


@pytest.mark.parametrize("lam", [0.5, 1.0])
def test_attend_variance_fp32_tiny_within_1e5(lam):
    host, dev = _inputs(TINY)
    rel, mx = _check_attend_var(TINY, dev, lam, density=0.1)
    assert rel <= 1e-5 and mx <= 1e-5, (rel, mx)


@pytest.mark.parametrize("lam", [0.5, 1.5])
@pytest.mark.parametrize("w", [SMALL_BF16, RAGGED_BF16_64, EAR_COUNTS], ids=lambda w: w.name)
def test_attend_variance_bf16_within_tolerance(w, lam):
    host, dev = _inputs(w)
    rel, mx = _check_attend_var(w, dev, lam, density=0.2)
    assert rel <= 1e-2 and mx <= 2e-2, (rel, mx)


@pytest.mark.parametrize("w", [TINY, SMALL_BF16], ids=lambda w: w.name)
def test_attend_variance_with_every_cluster_compensated(w):
    host, dev = _inputs(w)
    rel, mx = _check_attend_var(w, dev, 1.0, zero_budget=True)
    tol = (1e-5, 1e-5) if w.dtype == "f32" else (1e-2, 2e-2)
    assert rel <= tol[0] and mx <= tol[1], (rel, mx)


# ---------------------------------------------------------------------------
# Value-free probe error and the recall / MSE diagnostics
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [TINY, SMALL_BF16, RAGGED_BF16_64], ids=lambda w: w.name)
def test_value_free_probe_matches_oracle(w):
    csa = _csa()
    host, dev = _inputs(w)
    cq, ck, Vp, vbar = _clustered(w, dev)
    E = csa.svgear_probe_value_free(cq.centroids, ck.Xp, ck.centroids, ck.offsets, w.scale)
    torch.cuda.synchronize()
    for h in range(w.H):
        qbar = cq.centroids.cpu().numpy()[0, h]
        Kp = np64(ck.Xp)[0, h]
        off = ck.offsets.cpu().numpy()[0, h]
        kb = ck.centroids.cpu().numpy()[0, h]
        Eo = oracle.probe_value_free(qbar, Kp, kb, off, w.scale)
        # error scale of the bound: the value-aware probe with unit values
        u = np.zeros(w.d)
        u[0] = 1.0
        _, So = oracle.probe(qbar, Kp, np.tile(u, (w.N, 1)), kb, np.tile(u, (w.Ck, 1)), off,
                             w.scale, with_scale=True)
        tol = probe_tolerance(qbar, Kp, Eo, So, w.scale)
        Eg = E.cpu().numpy()[0, h].astype(np.float64)
        assert np.all(np.abs(Eg - Eo) <= tol), float(np.max(np.abs(Eg - Eo) / tol))


@pytest.mark.parametrize("density", [0.2, 1.0])
@pytest.mark.parametrize("w", [TINY, SMALL_BF16], ids=lambda w: w.name)
def test_diagnostics_match_oracle(w, density):
    csa = _csa()
    host, dev = _inputs(w)
    cq, ck, Vp, vbar = _clustered(w, dev)
    po, pk = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets, ck.Xp,
                              Vp, density, w.scale)
    O = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids, vbar,
                          cq.perm, w.scale, check_status=True)
    g = np.random.default_rng(9)
    R = 48
    rows = np.stack([np.sort(g.choice(w.N, R, replace=False)) for _ in range(w.H)])[None]
    rec, e2, r2 = csa.svgear_diagnostics(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, O,
                                         cq.perm, w.scale,
                                         torch.from_numpy(rows.astype(np.int32)).cuda())
    torch.cuda.synchronize()
    rec, e2, r2 = (t.cpu().numpy().astype(np.float64) for t in (rec, e2, r2))
    for h in range(w.H):
        ro, eo, fo = oracle.diagnostics(np64(cq.Xp)[0, h], np64(ck.Xp)[0, h], np64(Vp)[0, h],
                                        cq.offsets.cpu().numpy()[0, h],
                                        ck.offsets.cpu().numpy()[0, h], po.cpu().numpy()[0, h],
                                        pk.cpu().numpy()[0, h], np64(O)[0, h],
                                        cq.perm.cpu().numpy()[0, h], w.scale, rows[0, h])
        assert np.all(np.abs(rec[0, h] - ro) <= 1e-5)
        assert np.all(np.abs(r2[0, h] - fo) <= 1e-5 * fo + 1e-9)
        # fp32 dense output against fp64: |d err2| <= 2 |O - O_d| |dO_d| + |dO_d|^2
        assert np.all(np.abs(e2[0, h] - eo) <= 4e-5 * np.sqrt(eo * fo) + 1e-9 * fo + 1e-12)
        if density == 1.0:
            assert np.allclose(rec[0, h], 1.0, atol=1e-6)
