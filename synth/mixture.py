"""Seeded Gaussian-mixture generator and seeded initial-centroid choice.

Recipe (every draw comes from torch.Generator objects seeded from `seed`, one
independent stream per purpose, so changing one draw leaves the others unchanged):

  centers   n_comp x d, iid U[-1, 1] ("uniform") or iid N(0, 1) ("normal");
  component per point, iid categorical: equal weights, or Zipf weights w_j ~ j^-s
            (rank j = 1..n_comp), drawn by inverse CDF of a uniform;
  point     = center[component] + sigma * N(0, I), computed in fp32, then stored as
            fp32 or rounded (nearest even) to bf16;
  init      = the first K entries of a seeded random permutation of [0, N): K distinct
            point indices; the initial centroids are those points.

Generation on a CUDA device uses the device generator (fast for the 10^8-point case);
generation on the CPU uses the CPU generator.  The two give different (but equally
distributed) data; any comparison between the oracle and the GPU uses one generated
array, copied to wherever it is needed.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

# Stream ids for the independent generators derived from one seed.
_S_CENTERS, _S_COMP, _S_NOISE, _S_INIT = 11, 23, 37, 41
_S_QCOMP, _S_QNOISE = 53, 67  # query draws (offset by 1000 * query stream)
_S_ADV = 71  # adversarial rounding rows


@dataclass(frozen=True)
class MixtureSpec:
    name: str
    n: int
    d: int
    k: int                 # number of clusters (centroids) and of mixture components
    dtype: str             # "f32" or "bf16": storage type of X (and the MMA operand)
    centers: str           # "uniform" in [-1,1]^d or "normal" N(0, I)
    sigma: float
    weights: str           # "equal" or "zipf"
    zipf_s: float = 1.2
    metric: str = "l2"     # "l2" or "cosine"
    niter: int = 5
    seed: int = 0


# The workloads: shapes, distributions and iteration counts, keyed by name.
_SPECS = [
    MixtureSpec("tiny_65536x128_k256_f32", 65_536, 128, 256, "f32", "uniform", 0.1,
                "equal", niter=5),
    MixtureSpec("ivf_1000000x768_k4096_f32_cosine", 1_000_000, 768, 4096, "f32",
                "normal", 0.3, "equal", metric="cosine", niter=20),
    MixtureSpec("mid_10000000x128_k1024_f32", 10_000_000, 128, 1024, "f32",
                "uniform", 0.2, "equal", niter=10),
    MixtureSpec("zipf_16000000x128_k65536_f32", 16_000_000, 128, 65_536, "f32",
                "normal", 0.15, "zipf", zipf_s=1.2, niter=5),
    MixtureSpec("large_100000000x128_k32768_bf16", 100_000_000, 128, 32_768, "bf16",
                "normal", 0.25, "equal", niter=3),
]
CONFIGS = {s.name: s for s in _SPECS}
TINY, IVF, MID, ZIPF, LARGE = (s.name for s in _SPECS)


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + stream)
    return g


def _torch_dtype(dtype: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def gaussian_mixture(n: int, d: int, n_comp: int, *, centers: str = "normal",
                     sigma: float = 0.1, weights: str = "equal", zipf_s: float = 1.2,
                     dtype: str = "f32", seed: int = 0, device="cpu",
                     chunk_rows: int = 1 << 22, shard: int = 0):
    """Return (X [n, d] fp32 or bf16, comp [n] int32 component ids, centers [n_comp, d]
    fp32), all on `device`.  `shard` selects independent component and noise draws from
    the same mixture (same centers): the points of one data-parallel rank; shard 0 is the
    plain draw."""
    device = torch.device(device)
    cen = _centers(d, n_comp, centers, seed, device)

    X, comp = _draw_points(n, d, cen, sigma, weights, zipf_s, dtype,
                           _gen(device, seed, _S_COMP + 1000 * shard),
                           _gen(device, seed, _S_NOISE + 1000 * shard), device, chunk_rows)
    return X, comp, cen


def _centers(d: int, n_comp: int, centers: str, seed: int, device) -> torch.Tensor:
    gc = _gen(device, seed, _S_CENTERS)
    if centers == "uniform":
        return torch.rand(n_comp, d, generator=gc, device=device) * 2.0 - 1.0
    if centers == "normal":
        return torch.randn(n_comp, d, generator=gc, device=device)
    raise ValueError(centers)


def _draw_points(n, d, cen, sigma, weights, zipf_s, dtype, gk, gn, device, chunk_rows):
    n_comp = cen.shape[0]
    if weights == "equal":
        comp = torch.randint(0, n_comp, (n,), generator=gk, device=device,
                             dtype=torch.int64)
    elif weights == "zipf":
        w = torch.arange(1, n_comp + 1, device=device, dtype=torch.float64) ** (-zipf_s)
        cdf = torch.cumsum(w / w.sum(), 0)
        cdf[-1] = 1.0
        u = torch.rand(n, generator=gk, device=device, dtype=torch.float64)
        comp = torch.searchsorted(cdf, u, right=True).clamp_(max=n_comp - 1)
    else:
        raise ValueError(weights)
    X = torch.empty(n, d, dtype=_torch_dtype(dtype), device=device)
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        noise = torch.randn(r1 - r0, d, generator=gn, device=device)
        X[r0:r1] = (cen[comp[r0:r1]] + sigma * noise).to(X.dtype)
        del noise
    return X, comp.to(torch.int32)


def mixture_queries(nq: int, d: int, n_comp: int, *, centers: str = "normal",
                    sigma: float = 0.1, weights: str = "equal", zipf_s: float = 1.2,
                    seed: int = 0, stream: int = 0, device="cpu") -> torch.Tensor:
    """nq fp32 queries from the same mixture as gaussian_mixture(..., seed=seed) (same
    centers, fresh component and noise draws); `stream` selects independent query sets."""
    device = torch.device(device)
    cen = _centers(d, n_comp, centers, seed, device)
    Q, _ = _draw_points(nq, d, cen, sigma, weights, zipf_s, "f32",
                        _gen(device, seed, _S_QCOMP + 1000 * stream),
                        _gen(device, seed, _S_QNOISE + 1000 * stream), device, 1 << 22)
    return Q


def adversarial_rows(n: int, d: int, seed: int = 0) -> torch.Tensor:
    """n x d fp32 rows built to stress bf16 rounding: every coordinate positive and just
    under half a bf16 unit above a power of two (2^-2 .. 2^2, drawn per coordinate), with a
    small seeded jitter that keeps it there (1 + (0.49 +- 0.005) 2^-7 times the power).
    Rounding such operands to bf16 shrinks each by nearly the same relative amount and
    every partial sum of their products grows, so roundings pile up one way."""
    g = torch.Generator().manual_seed(seed * 1_000_003 + _S_ADV)
    e = torch.randint(-2, 3, (n, d), generator=g).double()
    jit = (torch.rand(n, d, generator=g, dtype=torch.float64) - 0.5) * 0.01
    m = 1.0 + (0.49 + jit) * 2.0 ** -7
    return (m * torch.pow(2.0, e)).float()


def init_indices(n: int, k: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """First k entries of a seeded random permutation of [0, n): k distinct indices."""
    if k > n:
        raise ValueError("k > n")
    g = _gen(torch.device(device), seed, _S_INIT)
    return torch.randperm(n, generator=g, device=device)[:k]


def make_config(cfg, device="cpu", n: int | None = None, **overrides):
    """Materialise a workload: returns (spec, X, C0 fp32, comp, centers).

    `cfg` is a workload name (a key of CONFIGS) or a MixtureSpec; `n` (and any MixtureSpec field given in
    `overrides`) shrinks or alters the spec for small test cases."""
    spec = CONFIGS[cfg] if not isinstance(cfg, MixtureSpec) else cfg
    if n is not None:
        overrides["n"] = n
    if overrides:
        spec = replace(spec, **overrides)
    X, comp, cen = gaussian_mixture(spec.n, spec.d, spec.k, centers=spec.centers,
                                    sigma=spec.sigma, weights=spec.weights,
                                    zipf_s=spec.zipf_s, dtype=spec.dtype, seed=spec.seed,
                                    device=device)
    idx = init_indices(spec.n, spec.k, spec.seed, device=device)
    C0 = X[idx].float().contiguous()
    return spec, X, C0, comp, cen
