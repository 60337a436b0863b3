"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This package makes data only: Gaussian-mixture points and initial centroids.  It holds
none of the clustering arithmetic (no distances, no means, no normalisation), so the
oracle and the CUDA path can both draw their inputs from it without sharing any of the
method.

The workloads follow the pages: synthetic mixture-of-Gaussians corpora (LEANN FlashLib
guide, section "诚实的局限说明": the benchmark corpus is a synthetic Gaussian mixture with
more components than nlist), with the 1M x 768, nlist 4096 coarse-quantizer shape of that
guide's "性能对比" section, and the d=128, K=32768 shape of the Flash-KMeans article's
headline run scaled to one GPU.
"""
from .mixture import (CONFIGS, IVF, LARGE, MID, TINY, ZIPF, MixtureSpec, adversarial_rows,
                      gaussian_mixture, init_indices, make_config, mixture_queries)

__all__ = ["CONFIGS", "TINY", "IVF", "MID", "ZIPF", "LARGE", "MixtureSpec", "make_config",
           "gaussian_mixture", "init_indices", "mixture_queries", "adversarial_rows"]
