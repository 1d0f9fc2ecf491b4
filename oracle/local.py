"""Oracle: the local (MSVS-style) vecset decoder query, in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The MSVS-VAE article (kwkr.cn) replaces the global cross-attention of vecset
decoding by a local operator and queries several scales of latents:

* AVS-Conv (§1.1): for a query point, only its K nearest support features (by
  Euclidean distance) take part; dynamic weights generated from the relative
  coordinates by a small MLP weight the features, and a mean-pooling residual
  branch is added;
* multi-scale query decoding, MSQ (§1.3): AVS-Conv queries every scale of the
  latent hierarchy; the results are concatenated and fused by a light network
  that outputs the SDF.

The latent hierarchy itself (its point-shuffle upsampling, §1.2) is an input
here: per scale s, anchor positions ``a[s][n_s,3]`` and features
``F[s][n_s,C_s]``.  Readings taken where the article gives no formula:

* neighbours: the K anchors of the scale with the smallest squared distance
  ``((a_x - x)^2 + (a_y - y)^2) + (a_z - z)^2`` evaluated in float32 (this
  decides an index set, so both sides take it in the kernel's precision), ties
  to the smaller anchor index;
* dynamic weights of neighbour j: ``w_j = W2_s GELU(W1_s (a_j - x) + b1_s) + b2_s``
  (one weight per channel, hidden width given by ``W1_s``);
* AVS-Conv: ``f_s(x) = (1/K) sum_j w_j * F_j + (1/K) sum_j F_j`` (elementwise
  product; the second term is the mean-pooling residual);
* MSQ: ``sdf = w_o . GELU(Wf [f_0, f_1, ...] + bf) + b_o``.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np

from . import decoder as D


def knn(x: np.ndarray, anchors: np.ndarray, K: int) -> np.ndarray:
    """Indices ``[M, K]`` of the K anchors nearest to each point of ``x[M,3]``
    (float32 squared distances, summed x, y then z; ties to the smaller index),
    nearest first."""
    x = np.asarray(x, np.float32)
    a = np.asarray(anchors, np.float32)
    out = np.empty((x.shape[0], K), np.int64)
    idx = np.arange(a.shape[0])
    for m in range(x.shape[0]):
        d = a - x[m]
        d2 = (d[:, 0] * d[:, 0] + d[:, 1] * d[:, 1]) + d[:, 2] * d[:, 2]   # float32, this order
        out[m] = np.lexsort((idx, d2))[:K]
    return out


def avs_conv(x: np.ndarray, anchors: np.ndarray, feats: np.ndarray, w: Dict[str, np.ndarray],
             K: int) -> np.ndarray:
    """AVS-Conv of one scale at points ``x[M,3]``: ``[M, C_s]``."""
    x = np.asarray(x, np.float64)
    a = np.asarray(anchors, np.float64)
    F = np.asarray(feats, np.float64)
    nb = knn(x, anchors, K)
    rel = a[nb] - x[:, None, :]                                     # [M, K, 3]
    hid = D.gelu(rel @ np.asarray(w["W1"], np.float64).T + np.asarray(w["b1"], np.float64))
    wts = hid @ np.asarray(w["W2"], np.float64).T + np.asarray(w["b2"], np.float64)   # [M, K, C]
    Fj = F[nb]                                                      # [M, K, C]
    return (wts * Fj).sum(axis=1) / K + Fj.sum(axis=1) / K


def decode_local(x: np.ndarray, anchors: List[np.ndarray], feats: List[np.ndarray],
                 scale_w: List[Dict[str, np.ndarray]], fuse: Dict[str, np.ndarray], K: int) -> np.ndarray:
    """SDF ``[M]`` at points ``x[M,3]`` from the multi-scale anchors."""
    f = np.concatenate([avs_conv(x, a, F, w, K) for a, F, w in zip(anchors, feats, scale_w)], axis=1)
    h = D.gelu(f @ np.asarray(fuse["Wf"], np.float64).T + np.asarray(fuse["bf"], np.float64))
    return h @ np.asarray(fuse["wo"], np.float64) + float(fuse["bo"][0])
