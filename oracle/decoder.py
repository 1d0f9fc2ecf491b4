"""Oracle: the vecset decoder evaluated per query point in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The pages describe the decoder as cross-attention from query points to the
unordered latent token set, followed by the SDF at each point (FlashVDM
summary, section 3 "Vecset Diffusion Model: decoder").  The concrete network
below is the plainest reading of that description plus the workload
definitions (Fourier features with 8 octaves, one cross-attention block with
heads of 64, output projection with residual, LayerNorm + GELU MLP with
residual, LayerNorm + linear SDF head):

    pe  = [x, y, z, sin(2^k pi x_a), cos(2^k pi x_a)]        (51 values, + 13 zero pads)
    q   = Wq pe + bq
    K,V = LN_kv(z) Wk^T + bk,  LN_kv(z) Wv^T + bv               (split into H heads of 64)
    a_h = softmax(q_h K_h^T / sqrt(64)) V_h                     (dense, or over a token subset)
    x1  = q + Wo a + bo
    x2  = x1 + W2 GELU(W1 LN1(x1) + b1) + b2                    (LN1 dropped without query LN)
    dec = w_head . LN2(x2) + b_head                             (LN2 dropped without query LN)

Readings taken where the pages are silent: LayerNorm uses epsilon 1e-5 and the
biased variance; GELU is the exact erf form; the attention scale is 1/8; the
"efficient decoder" (section 4.1 item 3, "remove part of the LayerNorm
layers") drops the two query-side LayerNorms and keeps LN_kv.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
from scipy.special import erf

HEAD_DIM = 64
PE_DIM = 51
PE_PAD = 64
N_FREQ = 8
LN_EPS = 1e-5


def grid_points(R: int, idx: Optional[np.ndarray] = None) -> np.ndarray:
    """Cell-centred coordinates of an R^3 grid over [-1, 1]^3.

    Voxel (i, j, k) sits at ``-1 + (2 i + 1) / R`` on each axis; its linear
    index is ``(i R + j) R + k`` (x slowest, z fastest).  Cell centring makes
    a voxel's 2^3 children at resolution 2R nest exactly inside it, which the
    coarse-to-fine subdivision of the hierarchical decoder needs (section 4.1
    item 1, step 3: "subdivide the selected voxels").
    """
    if idx is None:
        idx = np.arange(R ** 3, dtype=np.int64)
    idx = np.asarray(idx, dtype=np.int64)
    i, rem = np.divmod(idx, R * R)
    j, k = np.divmod(rem, R)
    ijk = np.stack([i, j, k], axis=1).astype(np.float64)
    return -1.0 + (2.0 * ijk + 1.0) / R


def fourier_embed(p: np.ndarray) -> np.ndarray:
    """``[M,3] -> [M,64]``: raw xyz, then sin for axes x,y,z and octaves
    k = 0..7 at lane ``3 + 8 a + k``, then cos at lane ``27 + 8 a + k``; lanes
    51..63 are zero."""
    p = np.asarray(p, dtype=np.float64)
    M = p.shape[0]
    out = np.zeros((M, PE_PAD), dtype=np.float64)
    out[:, 0:3] = p
    for a in range(3):
        for k in range(N_FREQ):
            arg = (2.0 ** k) * math.pi * p[:, a]
            out[:, 3 + 8 * a + k] = np.sin(arg)
            out[:, 27 + 8 * a + k] = np.cos(arg)
    return out


def layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray) -> np.ndarray:
    """LayerNorm over the last axis: biased variance, epsilon 1e-5."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + LN_EPS) * np.asarray(g, np.float64) + np.asarray(b, np.float64)


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: ``x * Phi(x)`` with the standard normal CDF written via erf."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def linear(x: np.ndarray, W: np.ndarray, b: Optional[np.ndarray]) -> np.ndarray:
    """``y = x W^T + b`` with ``W[out][in]``."""
    y = np.asarray(x, np.float64) @ np.asarray(W, np.float64).T
    if b is not None:
        y = y + np.asarray(b, np.float64)
    return y


def precompute_kv(z: np.ndarray, w: Dict[str, np.ndarray]) -> tuple:
    """Keys and values of one shape's vecset: ``z[N,C] -> K, V [H,N,64]``."""
    zn = layer_norm(z, w["ln_kv_g"], w["ln_kv_b"])
    K = linear(zn, w["Wk"], w["bk"])
    V = linear(zn, w["Wv"], w["bv"])
    N, C = K.shape
    H = C // HEAD_DIM
    K = K.reshape(N, H, HEAD_DIM).transpose(1, 0, 2).copy()
    V = V.reshape(N, H, HEAD_DIM).transpose(1, 0, 2).copy()
    return K, V


def attention_probs(q: np.ndarray, K: np.ndarray, sel: Optional[np.ndarray] = None) -> np.ndarray:
    """Per-head softmax weights ``[H, M, n]`` of queries ``q[M,C]`` over the
    tokens ``sel`` (all tokens if None), scale 1/sqrt(64)."""
    H = K.shape[0]
    M = q.shape[0]
    Ks = K if sel is None else K[:, sel, :]
    q = np.asarray(q, np.float64)
    out = np.empty((H, M, Ks.shape[1]), np.float64)
    for h in range(H):
        s = q[:, h * HEAD_DIM:(h + 1) * HEAD_DIM] @ Ks[h].T / math.sqrt(HEAD_DIM)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        out[h] = e / e.sum(axis=1, keepdims=True)
    return out


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray,
              sel: Optional[np.ndarray] = None) -> np.ndarray:
    """Multi-head cross-attention output ``[M,C]`` (heads concatenated)."""
    H = K.shape[0]
    M = q.shape[0]
    P = attention_probs(q, K, sel)
    Vs = V if sel is None else V[:, sel, :]
    return np.concatenate([P[h] @ Vs[h] for h in range(H)], axis=1)


def decode_points(p: np.ndarray, K: np.ndarray, V: np.ndarray, w: Dict[str, np.ndarray],
                  query_ln: bool = True, sel: Optional[np.ndarray] = None,
                  chunk: int = 512, return_attn: bool = False, return_tsdf: bool = False,
                  return_features: bool = False):
    """Raw decoder output ``dec`` at points ``p[M,3]`` (float64 ``[M]``).

    ``sel`` restricts attention to a subset of token indices (adaptive KV
    selection, section 4.1 item 2 step 5).  With ``return_attn`` the
    attention output ``a[M,C]`` is returned too.  With ``return_tsdf`` the
    raw truncated-SDF head is returned too: a second linear head on the same
    final features, ``t = w_tsdf . LN2(x2) + b_tsdf`` (the pages' VAE is
    trained to output a tSDF beside the SDF, aipaper.cc summary section 4.1
    item 1, "key details" 1).  With ``return_features`` the block output
    ``x2[M,C]`` (before the head's LayerNorm) is returned last.
    """
    p = np.asarray(p, np.float64).reshape(-1, 3)
    M = p.shape[0]
    out = np.empty(M, np.float64)
    attn = np.empty((M, K.shape[0] * HEAD_DIM)) if return_attn else None
    tsdf = np.empty(M, np.float64) if return_tsdf else None
    feats = np.empty((M, K.shape[0] * HEAD_DIM)) if return_features else None
    for s in range(0, M, chunk):
        pe = fourier_embed(p[s:s + chunk])
        q = linear(pe, w["Wq"], w["bq"])
        a = attention(q, K, V, sel)
        if return_attn:
            attn[s:s + chunk] = a
        x1 = q + linear(a, w["Wo"], w["bo"])
        h_in = layer_norm(x1, w["ln1_g"], w["ln1_b"]) if query_ln else x1
        x2 = x1 + linear(gelu(linear(h_in, w["W1"], w["b1"])), w["W2"], w["b2"])
        if return_features:
            feats[s:s + chunk] = x2
        y = layer_norm(x2, w["ln2_g"], w["ln2_b"]) if query_ln else x2
        out[s:s + chunk] = y @ np.asarray(w["w_head"], np.float64) + float(w["b_head"][0])
        if return_tsdf:
            tsdf[s:s + chunk] = y @ np.asarray(w["w_tsdf"], np.float64) + float(w["b_tsdf"][0])
    res = (out,) + ((attn,) if return_attn else ()) + ((tsdf,) if return_tsdf else ()) + \
        ((feats,) if return_features else ())
    return res if len(res) > 1 else out


def sphere_sdf(p: np.ndarray, spheres: np.ndarray) -> np.ndarray:
    """Exact signed distance to a union of spheres ``[S,4] = (c, r)``:
    ``min_s |p - c_s| - r_s`` (negative inside)."""
    p = np.asarray(p, np.float64).reshape(-1, 3)
    sp = np.asarray(spheres, np.float64)
    d = np.sqrt(((p[:, None, :] - sp[None, :, :3]) ** 2).sum(axis=2)) - sp[None, :, 3]
    return d.min(axis=1)


def tsdf_field(p: np.ndarray, t: np.ndarray, spheres: Optional[np.ndarray], dec_scale: float,
               trunc: float) -> np.ndarray:
    """Synthetic truncated SDF: ``clip((sphere SDF + dec_scale tanh(t)) / trunc,
    -1, 1)`` with ``t`` the raw tSDF head; the raw head itself without
    spheres.  (A tSDF saturates at +-1 beyond the truncation distance and
    measures closeness to the surface inside it.)"""
    t = np.asarray(t, np.float64)
    if spheres is None:
        return t
    return np.clip((sphere_sdf(p, spheres) + float(dec_scale) * np.tanh(t)) / float(trunc), -1.0, 1.0)


def field(p: np.ndarray, dec: np.ndarray, spheres: Optional[np.ndarray],
          dec_scale: float) -> np.ndarray:
    """Synthetic SDF field: sphere-union SDF plus ``dec_scale * tanh(dec)``;
    the raw decoder output when no spheres are given."""
    dec = np.asarray(dec, np.float64)
    if spheres is None:
        return dec
    return sphere_sdf(p, spheres) + float(dec_scale) * np.tanh(dec)
