"""The whole-layer entry points (svgear_layer on device buffers,
svgear_layer_host on host buffers) against the stage-by-stage composition of
the same C calls, and O against the oracle.  Every kernel is deterministic,
so the two routes must agree bit for bit: cold and warm starts, fixed density
and top-p budgets, plain and variance-corrected compensation, bf16 and fp32."""
import numpy as np
import pytest

import oracle
from clustered_sparse_attention_b200 import synth
from tests.helpers import np64, to_torch

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SMALL = synth.custom_workload("layer_small", H=3, frames=2, grid_h=24, grid_w=40, d=128,
                              dtype="bf16", Cq=16, Ck=40, iters=4, density=0.3, n_centres=24,
                              sigma=0.5, index=71)
TINY = synth.WORKLOADS["tiny"]
# enough heads for the host-buffer call to pipeline Q and O over head groups
# (2 groups of 17 heads for Q, 4 of 8-9 heads for attention and O)
MANY = synth.custom_workload("layer_many_heads", H=34, frames=1, grid_h=24, grid_w=32, d=64,
                             dtype="bf16", Cq=8, Ck=20, iters=3, density=0.25, n_centres=12,
                             sigma=0.5, index=72)


def _inputs(w):
    host = {n: synth.layer_tensor(w, n) for n in ("q", "k", "v")}
    return host, {n: to_torch(a, w.dtype) for n, a in host.items()}


@pytest.mark.parametrize("topp,lam", [(None, 0.0), (0.9, 0.0), (None, 1.0)])
@pytest.mark.parametrize("w", [SMALL, TINY, MANY], ids=lambda w: w.name)
def test_layer_call_equals_stagewise_composition(w, topp, lam):
    import clustered_sparse_attention_b200 as csa
    host, dev = _inputs(w)
    ref = csa.layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, w.iters, w.density, w.scale,
                    seed=3, topp=topp, var_lambda=lam)
    O, cq, ck = csa.svgear_layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, w.iters, w.density,
                                 w.scale, seed=3, topp=topp, var_lambda=lam)
    torch.cuda.synchronize()
    assert torch.equal(O, ref["O"])
    assert torch.equal(cq, ref["q"].centroids) and torch.equal(ck, ref["k"].centroids)
    # host buffers in, host buffer out, copies inside the call
    hq, hk, hv = (dev[n].cpu().pin_memory() for n in ("q", "k", "v"))
    res = csa.layer_host(hq, hk, hv, w.Cq, w.Ck, w.iters, w.density, w.scale, seed=3, topp=topp,
                         var_lambda=lam)
    torch.cuda.synchronize()
    assert torch.equal(res["O_host"], ref["O"].cpu())
    assert torch.equal(res["cent_k"], ref["k"].centroids)
    # warm step from the returned centroids, in place (cent aliases warm)
    wq, wk = cq.clone(), ck.clone()
    ref2 = csa.layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, 1, w.density, w.scale,
                     warm_q=wq.clone(), warm_k=wk.clone(), topp=topp, var_lambda=lam)
    O2, cq2, ck2 = csa.svgear_layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, 1, w.density,
                                    w.scale, warm_q=wq, warm_k=wk, cent_q=wq, cent_k=wk,
                                    topp=topp, var_lambda=lam)
    torch.cuda.synchronize()
    assert cq2.data_ptr() == wq.data_ptr()
    assert torch.equal(O2, ref2["O"]) and torch.equal(wq, ref2["q"].centroids)
    assert torch.equal(wk, ref2["k"].centroids)


def test_layer_call_output_matches_the_oracle_and_records_stage_events():
    import clustered_sparse_attention_b200 as csa
    w = SMALL
    host, dev = _inputs(w)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in evs:
        e.record()          # the CUDA events exist from their first record
    O, cq, ck = csa.svgear_layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, w.iters, w.density,
                                 w.scale, seed=0, stage_events=evs)
    torch.cuda.synchronize()
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
    assert all(t >= 0 for t in times) and sum(times) > 0
    # the stage-wise intermediates of the same (deterministic) call feed the oracle
    ref = csa.layer(dev["q"], dev["k"], dev["v"], w.Cq, w.Ck, w.iters, w.density, w.scale, seed=0)
    torch.cuda.synchronize()
    assert torch.equal(O, ref["O"])
    for h in range(w.H):
        n = int(ref["pair_off"][0, h, -1])
        Oo, _ = oracle.attend(np64(ref["q"].Xp)[0, h], np64(ref["k"].Xp)[0, h],
                              np64(ref["Vp"])[0, h], ref["q"].offsets.cpu().numpy()[0, h],
                              ref["k"].offsets.cpu().numpy()[0, h],
                              ref["pair_off"].cpu().numpy()[0, h],
                              ref["pair_kc"].cpu().numpy()[0, h][:n],
                              ck.cpu().numpy()[0, h], ref["vbar"].cpu().numpy()[0, h],
                              ref["q"].perm.cpu().numpy()[0, h], w.scale)
        Og = np64(O)[0, h]
        assert np.linalg.norm(Og - Oo) / np.linalg.norm(Oo) <= 1e-2
        assert np.abs(Og - Oo).max() <= 2e-2
