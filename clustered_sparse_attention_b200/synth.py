"""Seeded synthetic Q/K/V generators for the clustered sparse attention layer.

This module holds no part of the method's arithmetic: it only draws the
inputs that both the CUDA path and the CPU oracle consume, so that neither
has to import the other.  Shapes follow the video workloads the method is
evaluated on (Wan 2.1 / HunyuanVideo 720p latents of 45x80 tokens per frame,
SVG2 summary, "Experimental Setup"); the value distribution is a Gaussian
mixture with patch-coherent centre assignment, which stands in for the
models' real activations (no weights are available).

Recipe (per tensor Q, K or V, per batch b and head h):
  * centres ~ N(0, 1)^d, ``n_centres`` of them;
  * each 8x8 patch of a frame's latent grid draws one patch centre uniformly;
    a token takes its patch centre with probability ``p_patch`` (0.8), else a
    uniform centre.  Edge patches of grids that 8 does not divide are partial.
    The tiny workload instead assigns every token a uniform centre.
  * token = centre + sigma * N(0, 1)^d, stored as float32 or rounded to
    bfloat16 (round to nearest even).
  * the warm-start sequence drifts every element: x_{t+1} = x_t + 0.05 N(0,1).
Every draw comes from numpy's PCG64 seeded by SeedSequence([workload, tensor,
b, h(, step)]), so any single head can be regenerated on its own.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

TENSORS = {"q": 0, "k": 1, "v": 2}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int          # position in the workload list; part of every seed
    B: int
    H: int
    frames: int
    grid_h: int
    grid_w: int
    d: int
    dtype: str          # "f32" or "bf16"
    Cq: int
    Ck: int
    iters: int          # k-means iterations of the cold call
    density: float
    n_centres: int
    sigma: float
    patch_coherent: bool
    p_patch: float = 0.8
    patch: int = 8
    warm_steps: int = 0
    drift: float = 0.05

    @property
    def N(self) -> int:
        return self.frames * self.grid_h * self.grid_w

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 1, 4, 32, 32, 64, "f32", 16, 32, 10, 0.25,
                     16, 0.3, False),
    "mid": Workload("mid", 1, 1, 8, 16, 32, 32, 128, "bf16", 100, 250, 20, 0.3,
                    64, 0.5, True),
    "wan720p": Workload("wan720p", 2, 1, 40, 21, 45, 80, 128, "bf16", 100, 500,
                        40, 0.25, 256, 0.5, True),
    "hunyuan720p": Workload("hunyuan720p", 3, 1, 24, 33, 45, 80, 128, "bf16",
                            100, 500, 40, 0.25, 256, 0.5, True),
    "wan720p_warm": Workload("wan720p_warm", 4, 1, 40, 21, 45, 80, 128, "bf16",
                             100, 500, 1, 0.25, 256, 0.5, True, warm_steps=10),
    # the SVG-EAR paper's own cluster counts (review page, "What carries the
    # argument"): 300 or 400 query clusters, 1000 key clusters
    "wan720p_q300_k1000": Workload("wan720p_q300_k1000", 5, 1, 40, 21, 45, 80, 128, "bf16",
                                   300, 1000, 40, 0.25, 256, 0.5, True),
    "wan720p_q400_k1000": Workload("wan720p_q400_k1000", 6, 1, 40, 21, 45, 80, 128, "bf16",
                                   400, 1000, 40, 0.25, 256, 0.5, True),
}


def custom_workload(name: str, *, H: int, frames: int, grid_h: int, grid_w: int,
                    d: int, dtype: str, Cq: int, Ck: int, iters: int,
                    density: float, n_centres: int, sigma: float,
                    patch_coherent: bool = True, index: int = 99,
                    B: int = 1) -> Workload:
    """A workload of arbitrary size with the same recipe (for tests)."""
    return Workload(name, index, B, H, frames, grid_h, grid_w, d, dtype, Cq,
                    Ck, iters, density, n_centres, sigma, patch_coherent)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = (u << 16).astype(np.uint32).view(np.float32)
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 values already on the bf16 grid."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _rng(*words: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(words))))


def _centre_assignment(w: Workload, g: np.random.Generator) -> np.ndarray:
    if not w.patch_coherent:
        return g.integers(0, w.n_centres, size=w.N)
    ph = -(-w.grid_h // w.patch)
    pw = -(-w.grid_w // w.patch)
    rows = np.arange(w.grid_h) // w.patch
    cols = np.arange(w.grid_w) // w.patch
    patch_of = (rows[:, None] * pw + cols[None, :]).reshape(-1)
    out = np.empty(w.N, dtype=np.int64)
    per_frame = w.grid_h * w.grid_w
    for f in range(w.frames):
        patch_centre = g.integers(0, w.n_centres, size=ph * pw)
        own = patch_centre[patch_of]
        keep = g.random(per_frame) < w.p_patch
        other = g.integers(0, w.n_centres, size=per_frame)
        out[f * per_frame:(f + 1) * per_frame] = np.where(keep, own, other)
    return out


def head_tensor(w: Workload, tensor: str, b: int, h: int, step: int = 0) -> np.ndarray:
    """One head's [N, d] float32 tensor (values on the bf16 grid for bf16 workloads)."""
    t = TENSORS[tensor]
    g = _rng(w.index, t, b, h)
    centres = g.standard_normal((w.n_centres, w.d), dtype=np.float32)
    assign = _centre_assignment(w, g)
    x = centres[assign]
    x += np.float32(w.sigma) * g.standard_normal((w.N, w.d), dtype=np.float32)
    for s in range(1, step + 1):
        gs = _rng(w.index, t, b, h, 1000 + s)
        x += np.float32(w.drift) * gs.standard_normal((w.N, w.d), dtype=np.float32)
    if w.dtype == "bf16":
        x = round_to_bf16(x)
    return np.ascontiguousarray(x, dtype=np.float32)


def layer_tensor(w: Workload, tensor: str, step: int = 0, heads=None,
                 threads: int = 8) -> np.ndarray:
    """[B, H', N, d] float32 for the listed heads (all heads by default)."""
    heads = list(range(w.H)) if heads is None else list(heads)
    jobs = [(b, h) for b in range(w.B) for h in heads]
    out = np.empty((w.B, len(heads), w.N, w.d), dtype=np.float32)

    def one(i):
        b, h = jobs[i]
        out[b, heads.index(h)] = head_tensor(w, tensor, b, h, step)

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(one, range(len(jobs))))
    return out


def layer_tensor_bits(w: Workload, tensor: str, step: int = 0, heads=None,
                      threads: int = 8, batch_offset: int = 0) -> np.ndarray:
    """Like layer_tensor, but bfloat16 bit patterns (uint16) for bf16
    workloads -- half the host memory at the 720p shapes.  Batch index b of
    the result is drawn as batch b + batch_offset (independent replicas)."""
    if w.dtype != "bf16":
        raise ValueError("layer_tensor_bits is for bf16 workloads")
    heads = list(range(w.H)) if heads is None else list(heads)
    jobs = [(b + batch_offset, h) for b in range(w.B) for h in heads]
    out = np.empty((w.B, len(heads), w.N, w.d), dtype=np.uint16)

    def one(i):
        b, h = jobs[i]
        out[b - batch_offset, heads.index(h)] = bf16_bits(head_tensor(w, tensor, b, h, step))

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(one, range(len(jobs))))
    return out
