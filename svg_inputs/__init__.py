"""Seeded synthetic inputs for the sparse spatial/temporal video attention path.

This module is shared by the CPU oracle (``oracle/``), the tests and ``bench.py``.
It holds only input generation: workload shapes, a seeded Gaussian generator,
bf16 round-to-nearest-even encoding and the sampled-query draw.  None of the
method's arithmetic (attention, masks, permutation, profiling, calibration)
lives here.

Workloads follow the shapes of the video DiT layers the Sparse VideoGen article
(m.jxzklqfsx.com/article/815093.html) and the CalibAtt article
(lpnh.cn/news/568491) name: CogVideoX, Wan 2.1 (480p, 720p) and HunyuanVideo
720p, plus one tiny fp32 case.  No model weights, prompts or datasets are used;
q/k/v are synthetic:

    u ~ N(0, 1)                        [H, F, d]      (one vector per frame)
    w ~ N(0, 1)                        [H, P, d]      (one vector per position)
    z_q, z_k, z_v ~ N(0, 1)            [B, H, N, d]   (one stream per (tensor, b, h) slab)
    x[b,h,n] = z[b,h,n] + 2.0 * u[h, n // P]    for a spatial-type head
    x[b,h,n] = z[b,h,n] + 2.0 * w[h, n %  P]    for a temporal-type head

The same bias vector is added to q, k and v, so q.k is large between tokens of
one frame (spatial-type heads) or of one spatial position (temporal-type
heads).  Tokens are frame-major: n = f * P + s with P = ph * pw tokens per frame.
QK-Norm weights and 3D rotary tables for the fused QK-Norm + RoPE step are
synthetic inputs too (``qk_norm_weights``, ``rope_tables``).
All draws use numpy's PCG64 in float32: u and w come from ``default_rng(seed)``,
each (N, d) slab of z from its own ``default_rng((seed, tensor, b, h))`` (tensor
0, 1, 2 for q, k, v), so slabs are drawn in parallel threads and the result does
not depend on the thread count.  bf16 workloads are rounded to bf16 with
round-to-nearest-even and both sides consume the rounded values.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np
import torch

SPATIAL_TYPE = 0
TEMPORAL_TYPE = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-layer shape.  ``kind`` says where the per-head key-block
    lists come from: "profiled" (online profiling picks spatial or temporal per
    head) or "calibrated" (energy-threshold lists, one per head)."""

    name: str
    B: int
    H: int
    F: int          # latent frames
    ph: int         # latent height (tokens)
    pw: int         # latent width (tokens)
    d: int          # head dim
    dtype: str      # "bf16" or "fp32"
    S: int          # sampled queries for profiling
    width: int      # spatial band: keys with |f - f'| <= width
    head_types: str  # "alternate" | "half" | "random"
    kind: str = "profiled"
    eps: float = 0.90        # calibrated only: cumulative-energy threshold
    rho: float = 0.5         # calibrated only: keep-frequency threshold
    calib_seeds: tuple = ()  # calibrated only: inputs the lists are built from
    seed: int = 0            # seed of the timed / parity input
    block: int = 128

    @property
    def P(self) -> int:
        return self.ph * self.pw

    @property
    def N(self) -> int:
        return self.F * self.P

    @property
    def n_blocks(self) -> int:
        return (self.N + self.block - 1) // self.block

    def scaled(self, name: str, **kw) -> "Workload":
        return dataclasses.replace(self, name=name, **kw)


WORKLOADS = {
    # tiny fp32 case: head 0 spatial-type, head 1 temporal-type
    "tiny": Workload("tiny", B=1, H=2, F=4, ph=8, pw=8, d=64, dtype="fp32", S=16,
                     width=1, head_types="alternate"),
    # CogVideoX-shaped layer
    "cogvideox": Workload("cogvideox", B=1, H=48, F=13, ph=30, pw=45, d=64,
                          dtype="bf16", S=64, width=1, head_types="half"),
    # Wan 2.1 480p-shaped layer
    "wan480": Workload("wan480", B=1, H=40, F=21, ph=30, pw=52, d=128, dtype="bf16",
                       S=64, width=1, head_types="random"),
    # Wan 2.1 720p-shaped layer with calibrated per-head block lists
    "wan720": Workload("wan720", B=1, H=40, F=21, ph=45, pw=80, d=128, dtype="bf16",
                       S=64, width=1, head_types="random", kind="calibrated",
                       eps=0.90, rho=0.5, calib_seeds=(0, 1, 2, 3), seed=4),
    # HunyuanVideo 720p-shaped layer, band 2
    "hunyuan720": Workload("hunyuan720", B=1, H=24, F=33, ph=45, pw=80, d=128,
                           dtype="bf16", S=64, width=2, head_types="random"),
}

ORDER = ["tiny", "cogvideox", "wan480", "wan720", "hunyuan720"]


def small(name: str) -> Workload:
    """A reduced copy of a workload with the same head dim, dtype, band and
    head-type rule, small enough for the float64 oracle to finish in seconds
    while still spanning several 128-row tiles and a ragged last tile."""
    base = WORKLOADS[name]
    shrink = {
        "tiny": dict(),
        "cogvideox": dict(H=4, F=5, ph=10, pw=13),     # N = 650
        "wan480": dict(H=4, F=6, ph=9, pw=14),         # N = 756
        "wan720": dict(H=4, F=5, ph=11, pw=17),        # N = 935
        "hunyuan720": dict(H=4, F=7, ph=8, pw=13),     # N = 728
    }[name]
    return base.scaled(base.name + "-small", **shrink)


# --------------------------------------------------------------------------
# bf16 encoding (input preparation only)
# --------------------------------------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even (torch's
    float32 -> bfloat16 cast, which rounds to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# generator
# --------------------------------------------------------------------------

def head_types(wl: Workload, seed: Optional[int] = None) -> np.ndarray:
    """Bias type of each head: SPATIAL_TYPE (per-frame bias) or TEMPORAL_TYPE
    (per-position bias).  ``random`` draws a permutation from
    default_rng(1000 + seed) and makes its first H/2 heads spatial-type."""
    seed = wl.seed if seed is None else seed
    t = np.full(wl.H, TEMPORAL_TYPE, dtype=np.int32)
    if wl.head_types == "alternate":
        t[0::2] = SPATIAL_TYPE
    elif wl.head_types == "half":
        t[: wl.H // 2] = SPATIAL_TYPE
    elif wl.head_types == "random":
        perm = np.random.default_rng(1000 + seed).permutation(wl.H)
        t[perm[: wl.H // 2]] = SPATIAL_TYPE
    else:
        raise ValueError(wl.head_types)
    return t


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def generate(wl: Workload, seed: Optional[int] = None,
             types_seed: Optional[int] = None, heads: Optional[range] = None):
    """Draw q, k, v for one workload.

    Returns ``(q, k, v, types)``.  For bf16 workloads q/k/v are uint16 bf16
    bit patterns; for fp32 workloads they are float32.  All are [B, H, N, d]
    row-major.  ``types_seed`` fixes the head-type draw independently of the
    data seed (the calibrated workload keeps the types of its first input).

    u [H, F, d] and w [H, P, d] come from default_rng(seed) in that order; the
    (N, d) slab of tensor t (0 = q, 1 = k, 2 = v) for (b, h) comes from
    default_rng((seed, t, b, h)), is biased and rounded on its own, and the
    slabs are filled by a thread pool.  ``heads`` (a range of head indices)
    draws only those heads' slabs: the result equals the same slice of the
    whole layer, and ``types`` stays the whole layer's."""
    seed = wl.seed if seed is None else seed
    tseed = seed if types_seed is None else types_seed
    B, H, N, d, F, P = wl.B, wl.H, wl.N, wl.d, wl.F, wl.P
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((H, F, d), dtype=np.float32)
    wv = rng.standard_normal((H, P, d), dtype=np.float32)
    types = head_types(wl, tseed)
    bf16 = wl.dtype == "bf16"
    out_dtype = np.uint16 if bf16 else np.float32
    two = np.float32(2.0)
    heads = range(H) if heads is None else heads
    if len(heads) and (heads.start < 0 or heads.stop > H or heads.step != 1):
        raise ValueError(f"heads {heads} outside 0..{H}")
    outs = [np.empty((B, len(heads), N, d), dtype=out_dtype) for _ in range(3)]

    def slab(job):
        t, b, hl = job
        h = heads[hl]
        z = np.random.default_rng((seed, t, b, h)).standard_normal((N, d), dtype=np.float32)
        z = z.reshape(F, P, d)
        if types[h] == SPATIAL_TYPE:
            z += two * u[h][:, None, :]
        else:
            z += two * wv[h][None, :, :]
        z = z.reshape(N, d)
        outs[t][b, hl] = to_bf16_bits(z) if bf16 else z

    jobs = [(t, b, hl) for t in range(3) for b in range(B) for hl in range(len(heads))]
    with ThreadPoolExecutor(max_workers=_threads()) as ex:
        list(ex.map(slab, jobs))
    return outs[0], outs[1], outs[2], types


def as_float64(x: np.ndarray) -> np.ndarray:
    """Decode a generated tensor (bf16 bits or float32) to float64."""
    if x.dtype == np.uint16:
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def qk_norm_weights(wl: Workload, seed: Optional[int] = None):
    """Per-channel QK-Norm weights gamma_q, gamma_k (float32 [d]): 1 + 0.25 z
    with z ~ N(0, 1) from default_rng(2000 + seed), q's then k's.  Synthetic
    stand-ins for a model's learned weights."""
    seed = wl.seed if seed is None else seed
    rng = np.random.default_rng(2000 + seed)
    g = np.float32(1.0) + np.float32(0.25) * rng.standard_normal((2, wl.d), dtype=np.float32)
    return np.ascontiguousarray(g[0]), np.ascontiguousarray(g[1])


def rope_tables(wl: Workload, theta: float = 10000.0):
    """3D rotary-position tables cos, sin (float32 [N, d / 2]) for frame-major
    tokens n = f * P + y * pw + x.  The d / 2 channel pairs are split over the
    three axes as (d / 8, 3 d / 16, 3 d / 16) pairs for (f, y, x); pair i of
    an axis with n_a pairs turns at frequency theta^(-i / n_a), so the angle
    is the token's coordinate on that axis times that frequency.  These are
    inputs (a model computes them from its own positional scheme); both sides
    read the same float32 tables."""
    d, F, ph, pw = wl.d, wl.F, wl.ph, wl.pw
    n_t = d // 8
    n_y = (d // 2 - n_t) // 2
    n_x = d // 2 - n_t - n_y
    n = np.arange(wl.N)
    coords = (n // (ph * pw), (n // pw) % ph, n % pw)
    parts = []
    for c, n_a in zip(coords, (n_t, n_y, n_x)):
        freq = theta ** (-np.arange(n_a, dtype=np.float64) / n_a)
        parts.append(c[:, None].astype(np.float64) * freq[None, :])
    ang = np.concatenate(parts, axis=1)
    return (np.ascontiguousarray(np.cos(ang).astype(np.float32)),
            np.ascontiguousarray(np.sin(ang).astype(np.float32)))


def sample_queries(wl: Workload, seed: Optional[int] = None) -> np.ndarray:
    """Profiling sample: S distinct frame-major token indices drawn by
    default_rng(seed).choice, sorted ascending, shared by every (batch, head)."""
    seed = wl.seed if seed is None else seed
    idx = np.random.default_rng(seed).choice(wl.N, size=wl.S, replace=False)
    return np.sort(idx).astype(np.int32)
