"""Seeded synthetic inputs for the DLRMv1 sparse/interaction stage.

This module only draws inputs: it holds none of the stage's arithmetic, so both
the CUDA path and the CPU oracle can be fed from it. Nothing in the product's
compute path depends on it.

Recipe (the pages' workloads are synthetic dials, and the sizes here are the
benchmark configurations of this library):

* tables: ``F`` tables of ``N x D`` f32 drawn N(0, 0.1), table ``k`` from a
  torch generator seeded ``1000 + k`` on the device that will hold it;
* indices: ``(F, B*L)`` int32, table ``k`` from numpy ``PCG64(2000 + k)``;
  either uniform on ``[0, N)`` or a bounded Zipf law ``P(rank r) ~ r^-alpha``
  over ranks ``1..N``, where rank ``r`` maps to a row through a fixed random
  permutation of the table (``PCG64(4000 + k)``), so hot rows are scattered;
* offsets: ``(F, B)`` int32, fixed stride, ``offsets[k, b] = b * L``;
* dense: ``(B, D)`` f32 N(0, 1), torch generator seeded ``3000``.
"""
from __future__ import annotations

import dataclasses
import functools
from typing import Iterator, List, Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """One shape of the stage: batch ``B``, ``F`` tables of ``N x D``, bag ``L``."""

    name: str
    B: int
    F: int
    N: int
    D: int
    L: int
    dist: str = "uniform"  # "uniform" | "zipf"
    alpha: float = 0.0
    concat_dense: bool = False

    @property
    def P(self) -> int:
        """Dots per sample over the F+1 features: (F+1)F/2."""
        return (self.F + 1) * self.F // 2

    @property
    def table_bytes(self) -> int:
        return self.F * self.N * self.D * 4

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The configurations of the stage this library is measured and checked on.
TINY = Workload("tiny_b16_f2_n1000_d16_l4", B=16, F=2, N=1000, D=16, L=4)
C2_CONCAT = Workload("b2048_f8_n100k_d64_l32_uniform_concat", B=2048, F=8, N=100_000, D=64,
                     L=32, concat_dense=True)
C3_ZIPF = Workload("b2048_f32_n1m_d64_l16_zipf1.05", B=2048, F=32, N=1_000_000, D=64, L=16,
                   dist="zipf", alpha=1.05)
C3_UNIFORM = C3_ZIPF.scaled(name="b2048_f32_n1m_d64_l16_uniform", dist="uniform", alpha=0.0)
C5_ZIPF = Workload("b65536_f26_n4m_d128_l20_zipf1.2", B=65536, F=26, N=4_000_000, D=128, L=20,
                   dist="zipf", alpha=1.2)

SWEEP_BATCHES = tuple(2 ** i for i in range(11))  # 1 .. 1024
SWEEP_TABLES = (1, 4, 8, 16, 32)

CONFIGS = {
    "tiny": TINY,
    "c2": C2_CONCAT,
    "c3": C3_ZIPF,
    "c3u": C3_UNIFORM,
    "c5": C5_ZIPF,
}


def sweep() -> Iterator[Workload]:
    """The 11 x 5 batch x table-count sweep: 100000 x 64 tables, L = 8, uniform."""
    for F in SWEEP_TABLES:
        for B in SWEEP_BATCHES:
            yield Workload(f"sweep_b{B}_f{F}_n100k_d64_l8", B=B, F=F, N=100_000, D=64, L=8)


@functools.lru_cache(maxsize=4)
def _zipf_cdf(N: int, alpha: float) -> np.ndarray:
    ranks = np.arange(1, N + 1, dtype=np.float64)
    pmf = ranks ** (-alpha)
    cdf = np.cumsum(pmf)
    cdf /= cdf[-1]
    return cdf


def zipf_ranks(rng: np.random.Generator, n: int, N: int, alpha: float) -> np.ndarray:
    """``n`` draws of a 0-based rank in ``[0, N)`` with ``P(r) ~ (r+1)^-alpha``."""
    cdf = _zipf_cdf(N, alpha)
    u = rng.random(n)
    r = np.searchsorted(cdf, u, side="right")
    np.minimum(r, N - 1, out=r)
    return r


def table_indices(w: Workload, k: int, n: Optional[int] = None, replica: int = 0) -> np.ndarray:
    """Index stream of table ``k`` (``n`` entries, default ``B*L``), int32.

    ``replica`` selects an independent batch for another data-parallel replica
    (seed ``2000 + k + 100003 * replica``); replica 0 is the standard stream.
    """
    n = w.B * w.L if n is None else n
    rng = np.random.Generator(np.random.PCG64(2000 + k + 100003 * replica))
    if w.dist == "uniform":
        return rng.integers(0, w.N, size=n, dtype=np.int64).astype(np.int32)
    if w.dist == "zipf":
        ranks = zipf_ranks(rng, n, w.N, w.alpha)
        perm = np.random.Generator(np.random.PCG64(4000 + k)).permutation(w.N)
        return perm[ranks].astype(np.int32)
    raise ValueError(f"unknown index distribution {w.dist!r}")


def make_indices(w: Workload, replica: int = 0) -> np.ndarray:
    """``(F, B*L)`` int32 index matrix, table-major."""
    out = np.empty((w.F, w.B * w.L), dtype=np.int32)
    for k in range(w.F):
        out[k] = table_indices(w, k, replica=replica)
    return out


def make_offsets(w: Workload) -> np.ndarray:
    """``(F, B)`` int32 fixed-stride offsets ``b * L``."""
    row = np.arange(w.B, dtype=np.int64) * w.L
    return np.broadcast_to(row.astype(np.int32), (w.F, w.B)).copy()


def make_weights(w: Workload, device="cpu") -> List["torch.Tensor"]:
    """F tables ``(N, D)`` f32 ~ N(0, 0.1), table k seeded ``1000 + k``."""
    import torch

    tables = []
    for k in range(w.F):
        g = torch.Generator(device=device)
        g.manual_seed(1000 + k)
        t = torch.empty((w.N, w.D), dtype=torch.float32, device=device)
        t.normal_(0.0, 0.1, generator=g)
        tables.append(t)
    return tables


def make_dense(w: Workload, device="cpu") -> "torch.Tensor":
    """Dense features ``(B, D)`` f32 ~ N(0, 1), seeded ``3000``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(3000)
    t = torch.empty((w.B, w.D), dtype=torch.float32, device=device)
    t.normal_(0.0, 1.0, generator=g)
    return t


# DLRMv1 MLPs around the stage. The pages give no layer widths for their DLRMv1
# sweep; these follow the DLRM reference architecture for 13 dense features
# and D = 64: bottom 13-512-256-D, top (D+P)-512-256-1.
DENSE_FEATURES = 13
BOTTOM_HIDDEN = (512, 256)
TOP_HIDDEN = (512, 256)


def make_mlp_layers(in_features: int, widths, seed: int, device="cpu", last: str = "relu"):
    """Seeded layers ``(w, bias, act)`` of an MLP ``in_features -> widths...``.

    ``w`` is ``(N, K)`` bf16 (round-to-nearest-even of N(0, sqrt(2/(N+K))) f32
    draws) stored with a row pitch rounded up to 8 elements; ``bias`` is
    ``(N,)`` f32 N(0, sqrt(1/N)); hidden layers use ReLU, the last ``last``.
    Layer ``i`` draws from a torch generator seeded ``seed * 100 + i``.
    """
    import torch

    layers = []
    k = in_features
    for i, n in enumerate(widths):
        g = torch.Generator(device=device)
        g.manual_seed(seed * 100 + i)
        w32 = torch.empty((n, k), device=device).normal_(0.0, (2.0 / (n + k)) ** 0.5,
                                                          generator=g)
        b = torch.empty(n, device=device).normal_(0.0, (1.0 / n) ** 0.5, generator=g)
        w = torch.empty((n, (k + 7) // 8 * 8), dtype=torch.bfloat16, device=device)[:, :k]
        w.copy_(w32.to(torch.bfloat16))
        act = last if i == len(widths) - 1 else "relu"
        layers.append((w, b, act))
        k = n
    return layers


def make_dense_features(B: int, device="cpu", seed: int = 5000):
    """``(B, 13)`` bf16 dense input features (log-normal-like, as Criteo's
    log(1 + count) features): |N(0, 1)| rounded to bf16, pitch 16."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.empty((B, DENSE_FEATURES), device=device).normal_(0.0, 1.0, generator=g).abs_()
    out = torch.empty((B, 16), dtype=torch.bfloat16, device=device)[:, :DENSE_FEATURES]
    out.copy_(x.to(torch.bfloat16))
    return out


def make_ragged_offsets(w: Workload) -> np.ndarray:
    """``(F, B)`` int32 offsets of ragged bags over the same ``B*L`` entries per
    table: bag starts are sorted uniform draws on ``[0, B*L]`` with the first at 0
    (mean length L, lengths from 0 upward), table ``k`` from ``PCG64(6000 + k)``."""
    T = w.B * w.L
    off = np.empty((w.F, w.B), dtype=np.int32)
    for k in range(w.F):
        rng = np.random.Generator(np.random.PCG64(6000 + k))
        cuts = np.sort(rng.integers(0, T + 1, size=w.B - 1))
        off[k, 0] = 0
        off[k, 1:] = cuts
    return off


def make_sample_weights(w: Workload) -> np.ndarray:
    """``(F, B*L)`` f32 per-sample weights, uniform on [0, 1), ``PCG64(7000 + k)``."""
    out = np.empty((w.F, w.B * w.L), dtype=np.float32)
    for k in range(w.F):
        out[k] = np.random.Generator(np.random.PCG64(7000 + k)).random(w.B * w.L,
                                                                        dtype=np.float32)
    return out
