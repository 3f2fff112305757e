"""Seeded synthetic inputs shaped like video-DiT attention layers.

This module draws random numbers only: it holds none of the method's
arithmetic and is the one module that both the CUDA path's tests/benchmark
and the CPU oracle's tests consume.

Recipe (stands in for Wan2.1 / HunyuanVideo 720p video tokens, whose
prompts and weights are not available): for each (b, h), from
``numpy.random.default_rng([seed, b, h])``,

* omega_i ~ N(0, diag(lt^-2, ls^-2, ls^-2)), i < 64, and phase_i ~ U[0, 2pi);
* f_i(p) = cos(omega_i . p + phase_i) with p = (t, y, x) in grid units and
  token n = (t*Hg + y)*Wg + x (original order, no permutation);
* W in R^{d x 64} with N(0, 1/64) entries, shared by q and k so that
  attention is local in space and time;
* q = W f(p) + 0.5 eps_q, k = W f(p) + 0.5 eps_k, v ~ N(0, 1).

Values are generated in fp64 and rounded to bf16 (fp64 -> fp32 -> bf16,
each round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int
    Hg: int
    Wg: int
    budget: int          # expected KV blocks per query block (n)
    lt: float            # Fourier lengthscale in time (grid units)
    ls: float            # Fourier lengthscale in space
    seed: int

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def nqb(self) -> int:
        return (self.N + 127) // 128

    @property
    def nkb(self) -> int:
        return (self.N + 3) // 4

    @property
    def last_valid(self) -> int:
        return self.N - 128 * (self.nqb - 1)


def budget_blocks(fraction: float, nkb: int) -> int:
    """Budget in blocks for a density fraction: round-half-up(fraction * nkb)."""
    return min(nkb, int(math.floor(fraction * nkb + 0.5)))


# The five workloads.  Budgets: toy 13 blocks; 10% of 8190 = 819; 8% of
# 18900 = 1512; 8% of 29700 = 2376.
TOY = Workload("toy_4x8x16", 1, 2, 64, 4, 8, 16, 13, 3.0, 3.0, 0)
WAN480 = Workload("wan2.1_480p_21x30x52", 1, 40, 128, 21, 30, 52, 819, 3.0, 4.0, 0)
WAN720 = Workload("wan2.1_720p_21x45x80", 1, 40, 128, 21, 45, 80, 1512, 3.0, 4.0, 1)
HUNYUAN720 = Workload("hunyuan_720p_33x45x80", 1, 24, 128, 33, 45, 80, 2376, 2.0, 4.0, 2)
SWEEP_FRACTIONS = (0.01, 0.02, 0.05, 0.10, 0.25, 1.00)

WORKLOADS = {w.name: w for w in (TOY, WAN480, WAN720, HUNYUAN720)}


def with_budget(w: Workload, budget: int) -> Workload:
    return dataclasses.replace(w, budget=int(budget))


def grid_coords(T: int, Hg: int, Wg: int) -> np.ndarray:
    """[N, 3] (t, y, x) of token n = (t*Hg + y)*Wg + x."""
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    return np.stack([t.reshape(-1), y.reshape(-1), x.reshape(-1)], axis=1).astype(np.float64)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 -> fp32 -> bf16 (each to nearest even); return uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    bias = (u >> np.uint32(16)) & np.uint32(1)
    bias += np.uint32(0x7FFF)
    bias += u                      # no overflow for finite values
    out = (bias >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def head_qkv(w: Workload, b: int, h: int, coords: np.ndarray | None = None):
    """q, k, v of one (b, h) as fp64 [N, d] arrays."""
    rng = np.random.default_rng([w.seed, b, h])
    if coords is None:
        coords = grid_coords(w.T, w.Hg, w.Wg)
    omega = rng.standard_normal((64, 3)) / np.array([w.lt, w.ls, w.ls])
    phase = rng.uniform(0.0, 2.0 * math.pi, 64)
    W = rng.standard_normal((w.d, 64)) / 8.0
    feats = np.cos(coords @ omega.T + phase)
    base = feats @ W.T
    q = base + 0.5 * rng.standard_normal((w.N, w.d))
    k = base + 0.5 * rng.standard_normal((w.N, w.d))
    v = rng.standard_normal((w.N, w.d))
    return q, k, v


def layer_qkv_bits(w: Workload, heads: range | None = None, threads: int | None = None):
    """bf16 bit patterns of q, k, v: uint16 arrays [B, len(heads), N, d].

    Heads are generated independently (each from its own seeded stream), in a
    thread pool when there are several.
    """
    import concurrent.futures
    import os

    heads = range(w.H) if heads is None else heads
    coords = grid_coords(w.T, w.Hg, w.Wg)
    shape = (w.B, len(heads), w.N, w.d)
    q = np.empty(shape, np.uint16)
    k = np.empty(shape, np.uint16)
    v = np.empty(shape, np.uint16)

    def one(job):
        b, i, h = job
        qh, kh, vh = head_qkv(w, b, h, coords)
        q[b, i] = to_bf16_bits(qh)
        k[b, i] = to_bf16_bits(kh)
        v[b, i] = to_bf16_bits(vh)

    jobs = [(b, i, h) for b in range(w.B) for i, h in enumerate(heads)]
    n = threads or min(len(jobs), os.cpu_count() or 1, 16)
    if n <= 1:
        for job in jobs:
            one(job)
    else:
        with concurrent.futures.ThreadPoolExecutor(n) as ex:
            list(ex.map(one, jobs))
    return q, k, v


def perturbation_bits(w: Workload, step: int, base_q: np.ndarray, base_k: np.ndarray,
                      sigma: float = 0.05):
    """Denoising-step drift for the plan-reuse workload: q, k += sigma * N(0,1).

    base_q/base_k are fp32 arrays of the previous step; the drift is a
    cumulative random walk with fresh noise per step from rng([seed, 1000+step]).
    Returns the new fp32 arrays (the caller rounds them to bf16).
    """
    rng = np.random.default_rng([w.seed, 1000 + step])
    q = base_q + sigma * rng.standard_normal(base_q.shape, dtype=np.float32)
    k = base_k + sigma * rng.standard_normal(base_k.shape, dtype=np.float32)
    return q, k


def random_scores(rows: int, nkb: int, seed: int, concentration: float = 3.0) -> np.ndarray:
    """A seeded fp32 score array [rows, nkb] of non-negative rows summing to ~1.

    Heavy-tailed (log-normal) so that some blocks cap at pi = 1; used to feed
    the sampler alone.
    """
    rng = np.random.default_rng([seed, 77])
    x = np.exp(concentration * rng.standard_normal((rows, nkb)))
    x /= x.sum(axis=1, keepdims=True)
    return x.astype(np.float32)
