"""Oracle: the vecset encoder (point cloud -> vecset), in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pages say only that the VDM encoder compresses the input point cloud into
a fixed-size vecset with cross-attention (FlashVDM, aipaper.cc summary,
section 3 "Foundational Concepts: encoder"), and that the decoder is the same
kind of block in the other direction.  The plainest reading, written out here:

* the N latent tokens sit at N of the cloud's points (the query points, chosen
  by the caller: a uniform random subset in the workloads);
* every point of the cloud is embedded with the decoder's Fourier features and
  projected to the model width, ``u = W_in pe(p) + b_in``; LayerNorm and two
  projections give the keys and values, ``K, V = LN(u) Wk^T + bk, LN(u) Wv^T + bv``
  (the decoder's K/V path with the point features in the place of the latents);
* each latent token runs the decoder's block from its query point:
  ``q = Wq pe(x) + bq``, multi-head attention over the cloud, ``x1 = q + Wo a + bo``,
  ``x2 = x1 + W2 GELU(W1 LN1(x1) + b1) + b2``; the token is ``x2`` (no head).

The vecset does not depend on the order of the cloud's points (a pin), and a
decoder can consume it directly (its own LayerNorm and K/V projection).
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from . import decoder as D


def point_features(points: np.ndarray, w_in: np.ndarray, b_in: np.ndarray) -> np.ndarray:
    """``u = W_in pe(p) + b_in`` for the cloud's points: ``[M, C]``."""
    return D.linear(D.fourier_embed(points), w_in, b_in)


def encode(points: np.ndarray, queries: np.ndarray, w_in: np.ndarray, b_in: np.ndarray,
           w: Dict[str, np.ndarray], query_ln: bool = True) -> np.ndarray:
    """Vecset ``[N, C]`` of one cloud ``points[M,3]`` with latent tokens at
    ``queries[N,3]``; ``w`` holds the block's parameters (decoder layout, the
    head unused)."""
    K, V = D.precompute_kv(point_features(points, w_in, b_in), w)
    return D.decode_points(queries, K, V, w, query_ln, return_features=True)[1]
