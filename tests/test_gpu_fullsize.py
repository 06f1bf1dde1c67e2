"""The two 720p layers at full size, run through the C ABI exactly as bench.py
times them -- Wan 2.1 (B=1, H=40, N=75600) and HunyuanVideo (B=1, H=24,
N=118800), both d=128, Cq=100, Ck=500, 40 rounds, density 0.25, and the Wan
shape at the SVG-EAR paper's cluster counts (Cq=300, Ck=1000) -- then
checked against the oracle on what the oracle can compute one piece at a
time: sampled heads for the sort, means and routing (whole heads), sampled
tokens for the assignment, sampled query clusters for the probe and sampled
rows for the attention output (every 128-row tile boundary of four query
clusters, plus random rows); k-means++ is followed seed by seed on one head.
"""
import os

import numpy as np
import pytest

import oracle
from clustered_sparse_attention_b200 import synth
from tests.helpers import U32, check_assign, np64, probe_tolerance, update_tolerance

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

# sampled heads of each workload: first, one inside, last.  The third is the
# Wan shape at the SVG-EAR paper's cluster counts (300 query, 1000 key
# clusters): query clusters of ~250 rows, 1000 k-means++ seeds.
SHAPES = {"wan720p": (0, 17, 39), "hunyuan720p": (0, 11, 23), "wan720p_q300_k1000": (0, 23, 39)}


def _rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module", params=sorted(SHAPES))
def run(request):
    import clustered_sparse_attention_b200 as csa
    W = synth.WORKLOADS[request.param]
    threads = min(16, os.cpu_count() or 1)
    bits = {n: synth.layer_tensor_bits(W, n, threads=threads) for n in ("q", "k", "v")}
    dev = {n: torch.from_numpy(b).view(torch.bfloat16).cuda() for n, b in bits.items()}
    cq = csa.svgear_cluster(dev["q"], W.Cq, W.iters, seed=0, check_status=True)
    ck = csa.svgear_cluster(dev["k"], W.Ck, W.iters, seed=1, check_status=True)
    Vp = csa.svgear_permute(dev["v"], ck.perm)
    vbar = csa.svgear_centroids(Vp, ck.offsets, W.Ck)
    po, pk, E = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets, ck.Xp,
                                 Vp, W.density, W.scale, return_errors=True)
    O = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids, vbar,
                          cq.perm, W.scale, check_status=True)
    torch.cuda.synchronize()

    def host(name, h):
        b = bits[name][0, h].astype(np.uint32) << 16
        return b.view(np.float32)

    res = {"csa": csa, "W": W, "HEADS": SHAPES[W.name], "dev": dev, "host": host, "cq": cq,
           "ck": ck, "Vp": Vp, "vbar": vbar, "po": po, "pk": pk, "E": E, "O": O}
    yield res
    res.clear()
    torch.cuda.empty_cache()


def test_fullsize_kmeanspp_follows_the_oracle_on_one_head(run):
    W, HEADS = run["W"], run["HEADS"]
    csa = run["csa"]
    h = HEADS[1]
    cent, idx = csa.svgear_kmeanspp_init(run["dev"]["k"], W.Ck, seed=1)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()[0, h]
    X = run["host"]("k", h)
    own, margin = oracle.kmeanspp(X, W.Ck, seed=1, stream=h, follow=idx)
    assert own[0] == idx[0]
    band = 4 * (W.d + 2) * U32
    diff = np.nonzero(own != idx)[0]
    for j in diff:
        assert margin[j] < band, (j, idx[j], own[j], margin[j])
    assert len(diff) <= max(3, W.Ck // 200)   # every flip is inside the band (above)
    assert np.array_equal(cent.cpu().numpy()[0, h], X[idx])


@pytest.mark.parametrize("name", ["q", "k"])
def test_fullsize_sort_means_and_permuted_copy(run, name):
    W, HEADS = run["W"], run["HEADS"]
    C = W.Cq if name == "q" else W.Ck
    cl = run["cq"] if name == "q" else run["ck"]
    labels = cl.labels.cpu().numpy()
    perm = cl.perm.cpu().numpy()
    offs = cl.offsets.cpu().numpy()
    cents = cl.centroids.cpu().numpy()
    g = np.random.default_rng(5)
    for h in HEADS:
        X = run["host"](name, h)
        p_o, o_o = oracle.stable_sort(labels[0, h], C)
        assert np.array_equal(perm[0, h], p_o)
        assert np.array_equal(offs[0, h], o_o)
        ref = oracle.segment_mean(X[p_o], o_o, prev=cents[0, h])
        assert np.all(np.abs(cents[0, h] - ref) <= update_tolerance(X, labels[0, h], C))
        pos = g.choice(W.N, 4096, replace=False)
        Xp = cl.Xp[0, h][torch.from_numpy(pos).cuda()].float().cpu().numpy()
        assert np.array_equal(Xp, X[perm[0, h][pos]])


def test_fullsize_assignment_on_sampled_tokens(run):
    W, HEADS = run["W"], run["HEADS"]
    csa = run["csa"]
    ck = run["ck"]
    lab = csa.svgear_kmeans_assign(run["dev"]["k"], ck.centroids, check_status=True).cpu().numpy()
    cents = ck.centroids.cpu().numpy()
    g = np.random.default_rng(6)
    flips = 0
    for h in HEADS:
        tok = np.sort(g.choice(W.N, 6000, replace=False))
        X = run["host"]("k", h)
        flips += check_assign(X[tok], cents[0, h], lab[0, h][tok])
    assert flips <= 12   # 0.07 % of the sampled tokens; each one inside the band (check_assign)


def test_fullsize_probe_on_sampled_query_clusters(run):
    W, HEADS = run["W"], run["HEADS"]
    cq, ck = run["cq"], run["ck"]
    E = run["E"].cpu().numpy()
    qbar = cq.centroids.cpu().numpy()
    kbar = ck.centroids.cpu().numpy()
    vbar = run["vbar"].cpu().numpy()
    k_off = ck.offsets.cpu().numpy()
    for h in HEADS[:2]:
        rows = np.array([0, 37, W.Cq - 1])
        Kp, Vp = np64(ck.Xp[0, h]), np64(run["Vp"][0, h])
        Eo, So, Po = oracle.probe(qbar[0, h][rows], Kp, Vp, kbar[0, h], vbar[0, h], k_off[0, h],
                                  W.scale, with_parts=True)
        tol = probe_tolerance(qbar[0, h][rows], Kp, Eo, So, W.scale, P=Po)
        Eg = E[0, h][rows].astype(np.float64)
        assert np.all(np.abs(Eg - Eo) <= tol), float(np.max(np.abs(Eg - Eo) / tol))


def test_fullsize_route_bit_exact_given_gpu_errors(run):
    W, HEADS = run["W"], run["HEADS"]
    cq, ck = run["cq"], run["ck"]
    E = run["E"].cpu().numpy()
    po, pk = run["po"].cpu().numpy(), run["pk"].cpu().numpy()
    for h in HEADS:
        ref_off, ref_kc = oracle.route(E[0, h], cq.offsets.cpu().numpy()[0, h],
                                       ck.offsets.cpu().numpy()[0, h], W.N, W.density)
        assert np.array_equal(po[0, h], ref_off)
        assert np.array_equal(pk[0, h][:ref_off[-1]], ref_kc)


def test_fullsize_attention_on_sampled_rows(run):
    W, HEADS = run["W"], run["HEADS"]
    cq, ck = run["cq"], run["ck"]
    q_off = cq.offsets.cpu().numpy()
    g = np.random.default_rng(7)
    O = run["O"]
    for h in HEADS[:2]:
        qo = q_off[0, h]
        # the first and last row of every 128-row tile of four query clusters
        # (every CTA's tile, the partial last one included) plus random rows
        rows = set(g.choice(W.N, 32, replace=False).tolist())
        for i in (0, 1, W.Cq // 2, W.Cq - 1):
            a, b = int(qo[i]), int(qo[i + 1])
            for r0 in range(a, b, 128):
                rows.update((r0, min(r0 + 127, b - 1)))
        rows = np.array(sorted(rows))
        args = (np64(cq.Xp[0, h]), np64(ck.Xp[0, h]), np64(run["Vp"][0, h]), qo,
                ck.offsets.cpu().numpy()[0, h], run["po"].cpu().numpy()[0, h],
                run["pk"].cpu().numpy()[0, h], ck.centroids.cpu().numpy()[0, h],
                run["vbar"].cpu().numpy()[0, h], cq.perm.cpu().numpy()[0, h])
        Oo, _ = oracle.attend(*args, W.scale, rows=rows)
        dst = cq.perm.cpu().numpy()[0, h][rows]
        Og = np64(O[0, h][torch.from_numpy(dst).cuda()])
        assert _rel_l2(Og, Oo) <= 1e-2 and np.abs(Og - Oo).max() <= 2e-2


def test_fullsize_topp_budget_and_routing(run):
    W, HEADS = run["W"], run["HEADS"]
    csa = run["csa"]
    cq, ck = run["cq"], run["ck"]
    budget = csa.svgear_topp_budget(cq.centroids, cq.offsets, ck.centroids, ck.offsets, W.N, 0.9,
                                    W.scale)
    po, pk = csa.svgear_route_select_budget(run["E"], cq.offsets, ck.offsets, W.N, budget)
    b = budget.cpu().numpy()
    qb, kb = cq.centroids.cpu().numpy(), ck.centroids.cpu().numpy()
    qo, ko = cq.offsets.cpu().numpy(), ck.offsets.cpu().numpy()
    E = run["E"].cpu().numpy()
    for h in HEADS:
        ref, margin = oracle.topp_budget(qb[0, h], kb[0, h], qo[0, h], ko[0, h], 0.9, W.scale)
        bad = np.nonzero(ref != b[0, h])[0]
        assert all(margin[i] < 1e-9 for i in bad) and len(bad) <= 1
        ref_off, ref_kc = oracle.route(E[0, h], qo[0, h], ko[0, h], W.N, 1.0,
                                       budgets=b[0, h].astype(np.int64))
        assert np.array_equal(po.cpu().numpy()[0, h], ref_off)
        assert np.array_equal(pk.cpu().numpy()[0, h][:ref_off[-1]], ref_kc)
