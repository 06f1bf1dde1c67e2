"""The bounded device wait and the tensor-memory guard, exercised on the GPU
without faulting or hanging it.

Every wait in the tensor-core kernels gives up after a time limit, records
SVGEAR_ERR_TIMEOUT with the wait's site and CTA in the device status words
and returns, so the CUDA context stays usable.  svgear_selftest_wait runs that
same wait on a barrier nothing arrives on (a short limit, no tensor memory, no
MMA, no copy).  A kernel that gives up with an MMA possibly still running
keeps its tensor memory and sets the device's lost word; later tensor-core
kernels then refuse to start.  That state lasts for the CUDA context, so its
test runs in a child process of its own.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle
from clustered_sparse_attention_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SITE_SELFTEST, SITE_REFUSED = 60, 61


def test_bounded_wait_gives_up_reports_and_leaves_the_gpu_usable():
    import clustered_sparse_attention_b200 as csa
    from clustered_sparse_attention_b200 import _lib
    st = _lib.selftest_wait(arrive=False, timeout_us=2000)
    assert st[0] == _lib.ERR_TIMEOUT
    assert st[1] >> 16 == SITE_SELFTEST and st[2] == 0 and st[3] == 0
    # the same wait completes when its arrival is made, and the words clear
    assert _lib.selftest_wait(arrive=True, timeout_us=2000) == [0, 0, 0, 0]
    # the GPU is unaffected: a small tensor-core layer still matches the oracle
    w = synth.custom_workload("after_timeout", H=2, frames=1, grid_h=24, grid_w=40, d=128,
                              dtype="bf16", Cq=8, Ck=24, iters=3, density=0.3, n_centres=16,
                              sigma=0.5, index=70)
    host = {n: synth.layer_tensor(w, n) for n in ("q", "k", "v")}
    dev = {n: torch.from_numpy(a).to(torch.bfloat16).cuda() for n, a in host.items()}
    cq = csa.svgear_cluster(dev["q"], w.Cq, w.iters, seed=0, check_status=True)
    ck = csa.svgear_cluster(dev["k"], w.Ck, w.iters, seed=1, check_status=True)
    Vp = csa.svgear_permute(dev["v"], ck.perm)
    vbar = csa.svgear_centroids(Vp, ck.offsets, w.Ck)
    po, pk = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets, ck.Xp, Vp,
                              w.density, w.scale)
    O = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids, vbar,
                          cq.perm, w.scale, check_status=True)
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()  # noqa: E731
    for h in range(w.H):
        n = int(po[0, h, -1])
        Oo, _ = oracle.attend(f64(cq.Xp)[0, h], f64(ck.Xp)[0, h], f64(Vp)[0, h],
                              cq.offsets.cpu().numpy()[0, h], ck.offsets.cpu().numpy()[0, h],
                              po.cpu().numpy()[0, h], pk.cpu().numpy()[0, h][:n],
                              ck.centroids.cpu().numpy()[0, h], vbar.cpu().numpy()[0, h],
                              cq.perm.cpu().numpy()[0, h], w.scale)
        Og = f64(O)[0, h]
        assert np.linalg.norm(Og - Oo) / np.linalg.norm(Oo) <= 1e-2
        assert np.abs(Og - Oo).max() <= 2e-2


_CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, %(root)r)
import clustered_sparse_attention_b200 as csa
from clustered_sparse_attention_b200 import _lib
torch.cuda.set_device(0)
g = np.random.default_rng(3)
X = torch.from_numpy(g.standard_normal((1, 2, 2048, 128)).astype(np.float32)).to(torch.bfloat16).cuda()
C = torch.from_numpy(g.standard_normal((1, 2, 40, 128)).astype(np.float32)).cuda()
out = {}
lab = csa.svgear_kmeans_assign(X, C, check_status=True)
out["before"] = "ok"
# a wait that gives up and marks the tensor memory lost (it allocated none)
ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
rc = _lib.lib().svgear_selftest_wait(_lib._ptr(ws), 256, 0, 2000, 1, _lib._stream())
torch.cuda.synchronize()
out["selftest_rc"] = rc
# the device word alone (not yet seen by the host) stops the next kernel
# before it allocates: it launches and returns SVGEAR_ERR_TMEM_LOST
l0 = csa.kernel_launches()
try:
    csa.svgear_kmeans_assign(X, C, check_status=True)
    out["device_refusal"] = None
except _lib.SvgearError as e:
    out["device_refusal"] = e.status
    out["device_refusal_msg"] = str(e)
out["device_refusal_launched"] = csa.kernel_launches() - l0
# svgear_device_status has now seen the word: calls return without launching
l0 = csa.kernel_launches()
for name, fn in (("assign", lambda: csa.svgear_kmeans_assign(X, C)),
                 ("cluster", lambda: csa.svgear_cluster(X, 40, 2, seed=0))):
    try:
        fn()
        out[name] = None
    except _lib.SvgearError as e:
        out[name] = e.status
out["host_refusal_launched"] = csa.kernel_launches() - l0
# work without tensor memory still runs: the fp32 assignment and the label sort
lab32 = csa.svgear_kmeans_assign(X.float(), C)
perm, off = csa.svgear_label_sort(lab32, 40)
torch.cuda.synchronize()
out["fp32_ok"] = bool(torch.equal(off[..., -1], torch.full_like(off[..., -1], 2048)))
print("RESULT " + json.dumps(out))
"""


def test_lost_tensor_memory_refuses_later_tensor_core_calls():
    from clustered_sparse_attention_b200 import _lib
    r = subprocess.run([sys.executable, "-c", _CHILD % {"root": ROOT}], capture_output=True,
                       text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    out = json.loads(line[len("RESULT "):])
    assert out["before"] == "ok" and out["selftest_rc"] == _lib.OK
    assert out["device_refusal"] == _lib.ERR_TMEM_LOST, out
    assert "wait site %d" % SITE_REFUSED in out["device_refusal_msg"]
    assert "tensor memory lost 1" in out["device_refusal_msg"]
    assert out["device_refusal_launched"] >= 1
    assert out["assign"] == _lib.ERR_TMEM_LOST and out["cluster"] == _lib.ERR_TMEM_LOST
    assert out["host_refusal_launched"] == 0
    assert out["fp32_ok"] is True
