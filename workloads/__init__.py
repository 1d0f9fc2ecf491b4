"""Seeded synthetic workloads for the vecset SDF decoder.

This module only *draws* inputs: latent vecsets, decoder weights, unions of
spheres and query points.  It holds none of the decoder's arithmetic, so both
the CPU oracle (``oracle/``) and the CUDA path's tests and benchmark can use it
without sharing any computation.

Sizes follow the five workloads of the lightning vecset decoder study
("Unleashing Vecset Diffusion Model for Fast Shape Generation", FlashVDM,
section 4.1: hierarchical volume decoding, adaptive KV selection, efficient
decoder; section 6, Tables 1 and 3 use a 3072-token vecset decoded to 384^3).
Real latents and trained weights are not available, so every array is drawn
from a seeded generator:

* latents ``z ~ N(0, 1)``;
* weight matrices ``~ N(0, 0.02^2)``, biases zero, LayerNorm gamma one / beta
  zero (all still passed explicitly);
* sphere centres ``U[-0.6, 0.6]^3``, radii ``U[0.05, 0.3]``.

Each array has its own generator ``PCG64(SeedSequence([seed, key, array_id]))``
so that arrays do not depend on each other's sizes.  For bf16 workloads the
weight matrices are rounded to bf16 (round to nearest even) here, so both sides
consume identical values.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, Optional

import numpy as np

PE_DIM = 51       # 3 raw coordinates + 2 (sin, cos) x 3 axes x 8 frequencies
PE_PAD = 64       # the embedding is zero-padded to 64 lanes
HEAD_DIM = 64     # every attention head is 64 wide
N_FREQ = 8

# array ids for the per-array seed sequences
_A_Z, _A_WQ, _A_WK, _A_WV, _A_WO, _A_W1, _A_W2, _A_WH = range(8)
_A_CENTRE, _A_RADIUS, _A_POINTS = 8, 9, 10
_A_CLOUD, _A_QUERY, _A_WIN = 11, 12, 13
_A_LOCAL = 30
_A_STRESS = 20
_A_WT = 21


@dataclass(frozen=True)
class DecoderSpec:
    """Shape of one vecset decoder (cross-attention block + MLP + SDF head)."""
    C: int            # model width
    H: int            # heads (C == H * 64)
    F: int            # MLP hidden width
    N: int            # latent tokens per shape
    query_ln: bool    # LayerNorm before the MLP and before the head
    dtype: str        # 'f32' or 'bf16' (storage type of matrices and K/V)

    def __post_init__(self):
        assert self.C == self.H * HEAD_DIM, "C must equal H * 64"


@dataclass(frozen=True)
class Config:
    cid: int
    name: str
    dec: DecoderSpec
    B: int = 1                 # shapes in the batch
    mode: str = "dense"        # 'dense' (one grid) or 'hier' (coarse to fine)
    grid_R: int = 32           # dense mode: grid resolution per axis
    r0: int = 0                # hier mode: coarse resolution
    n_levels: int = 1          # hier mode: number of levels (r0 * 2^(L-1) final)
    adaptive: bool = False     # adaptive KV selection on fine levels
    tile: int = 8              # sub-volume edge (fine voxels)
    n_probe: int = 64          # probe queries per sub-volume
    top_k: int = 1024          # kept latent tokens per sub-volume
    n_spheres: int = 0         # analytic term: spheres per shape (0 = none)
    dec_scale: float = 0.0     # field = sphere SDF + dec_scale * tanh(dec)
    seed_key: int = 0          # key for the latents and decoder weights
    sphere_key: int = 0        # key for the spheres

    @property
    def r_final(self) -> int:
        return self.r0 << (self.n_levels - 1) if self.mode == "hier" else self.grid_R

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


_DEC_TINY = DecoderSpec(C=64, H=1, F=256, N=256, query_ln=True, dtype="f32")
_DEC_FULL = DecoderSpec(C=512, H=8, F=2048, N=3072, query_ln=True, dtype="bf16")
_DEC_SLIM = DecoderSpec(C=256, H=4, F=512, N=4096, query_ln=False, dtype="bf16")
# the efficient decoder at a quarter of the full width: narrower, smaller MLP ratio, no
# query-side LayerNorm (techwalker article, section 5; aipaper.cc summary, section 4.1 item 3)
_DEC_QUARTER = DecoderSpec(C=128, H=2, F=256, N=3072, query_ln=False, dtype="bf16")

CONFIGS: Dict[int, Config] = {
    1: Config(1, "tiny dense fp32, 32^3", _DEC_TINY, grid_R=32, seed_key=1),
    2: Config(2, "dense bf16, 128^3", _DEC_FULL, grid_R=128, seed_key=2),
    3: Config(3, "hierarchical bf16, 96->192->384", _DEC_FULL, mode="hier", r0=96,
              n_levels=3, n_spheres=16, dec_scale=0.01, seed_key=2, sphere_key=3),
    4: Config(4, "hierarchical + adaptive KV bf16, 96->192->384", _DEC_FULL,
              mode="hier", r0=96, n_levels=3, adaptive=True, n_spheres=16,
              dec_scale=0.01, seed_key=2, sphere_key=3),
    5: Config(5, "batched slim decoder, 4 shapes, 128->256->512, adaptive KV",
              _DEC_SLIM, B=4, mode="hier", r0=128, n_levels=3, adaptive=True,
              n_spheres=24, dec_scale=0.01, seed_key=5, sphere_key=5),
    6: Config(6, "quarter-width efficient decoder, hierarchical + adaptive KV bf16, 96->192->384",
              _DEC_QUARTER, mode="hier", r0=96, n_levels=3, adaptive=True, n_spheres=16,
              dec_scale=0.01, seed_key=6, sphere_key=3),
}


def _rng(seed: int, key: int, array_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, key, array_id])))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).reshape(a.shape)


def make_decoder(spec: DecoderSpec, seed: int = 0, key: int = 0, B: int = 1,
                 stress: bool = False, tsdf: bool = False) -> Dict[str, np.ndarray]:
    """Latents ``z[B,N,C]`` (float32) and decoder parameters (float32 arrays).

    Matrices follow the ``y = x W^T + b`` convention with ``W[out][in]``.
    ``Wq`` is ``[C, 64]``; columns 51..63 face the zero pad lanes of the
    embedding and are zero.  With ``stress`` the query/key projections get
    std 0.2 (attention logits of order 5 instead of nearly uniform weights)
    and biases, LayerNorm affines and a non-zero-mean value bias are drawn
    too, so that an error in any of them shows in the output.  With ``tsdf``
    a second head ``w_tsdf`` (N(0, 0.02^2), stress: 0.2) and ``b_tsdf`` (0)
    are drawn for the truncated-SDF output channel.
    """
    C, F, N = spec.C, spec.F, spec.N
    std = 0.02
    qk_std = 0.2 if stress else std

    def mat(aid, shape, s):
        return (_rng(seed, key, aid).standard_normal(shape) * s).astype(np.float32)

    w = {}
    wq = np.zeros((C, PE_PAD), np.float32)
    wq[:, :PE_DIM] = mat(_A_WQ, (C, PE_DIM), qk_std)
    w["Wq"] = wq
    w["Wk"] = mat(_A_WK, (C, C), qk_std)
    w["Wv"] = mat(_A_WV, (C, C), std)
    w["Wo"] = mat(_A_WO, (C, C), std)
    w["W1"] = mat(_A_W1, (F, C), std)
    w["W2"] = mat(_A_W2, (C, F), std)
    w["w_head"] = mat(_A_WH, (C,), std)
    if spec.dtype == "bf16":
        for k in ("Wq", "Wk", "Wv", "Wo", "W1", "W2"):
            w[k] = round_bf16(w[k])

    zeros = lambda n: np.zeros((n,), np.float32)
    ones = lambda n: np.ones((n,), np.float32)
    w.update(bq=zeros(C), bk=zeros(C), bv=zeros(C), bo=zeros(C), b1=zeros(F), b2=zeros(C),
             ln_kv_g=ones(C), ln_kv_b=zeros(C), ln1_g=ones(C), ln1_b=zeros(C),
             ln2_g=ones(C), ln2_b=zeros(C), b_head=zeros(1))
    if stress:
        r = _rng(seed, key, _A_STRESS)
        for k, n in (("bq", C), ("bk", C), ("bo", C), ("b1", F), ("b2", C)):
            w[k] = (r.standard_normal(n) * 0.05).astype(np.float32)
        w["bv"] = (0.3 + r.standard_normal(C) * 0.1).astype(np.float32)
        for k in ("ln_kv_g", "ln1_g", "ln2_g"):
            w[k] = (1.0 + r.standard_normal(C) * 0.1).astype(np.float32)
        for k in ("ln_kv_b", "ln1_b", "ln2_b"):
            w[k] = (r.standard_normal(C) * 0.1).astype(np.float32)
        w["b_head"] = np.array([0.05], np.float32)

    if tsdf:
        w["w_tsdf"] = mat(_A_WT, (C,), 0.2 if stress else std)
        w["b_tsdf"] = np.zeros((1,), np.float32)
    z = _rng(seed, key, _A_Z).standard_normal((B, N, C)).astype(np.float32)
    return {"z": z, "weights": w}


def make_spheres(n_spheres: int, seed: int = 0, key: int = 0, B: int = 1) -> np.ndarray:
    """``[B, S, 4]`` float32 rows ``(cx, cy, cz, r)``."""
    c = _rng(seed, key, _A_CENTRE).uniform(-0.6, 0.6, (B, n_spheres, 3))
    r = _rng(seed, key, _A_RADIUS).uniform(0.05, 0.3, (B, n_spheres, 1))
    return np.concatenate([c, r], axis=2).astype(np.float32)


def make_points(M: int, seed: int = 0, key: int = 0, B: int = 1) -> np.ndarray:
    """``[B, M, 3]`` float32 query points uniform in [-1, 1]^3."""
    return _rng(seed, key, _A_POINTS).uniform(-1.0, 1.0, (B, M, 3)).astype(np.float32)


def make_point_cloud(spheres: np.ndarray, n_points: int, n_queries: int, seed: int = 0,
                     key: int = 0) -> Dict[str, np.ndarray]:
    """A point cloud on the surface of a union of spheres ``[S,4]`` and the
    encoder's latent query points, a uniform random subset of it.

    Points are drawn on the spheres in proportion to their areas (uniform
    directions); points inside another sphere are not on the union's surface
    and are drawn again.  Returns ``points [n_points, 3]`` and
    ``queries [n_queries, 3]`` (float32)."""
    rng = _rng(seed, key, _A_CLOUD)
    sp = np.asarray(spheres, np.float64)
    area = sp[:, 3] ** 2
    out = []
    while sum(len(x) for x in out) < n_points:
        s_idx = rng.choice(len(sp), n_points, p=area / area.sum())
        d = rng.standard_normal((n_points, 3))
        d /= np.linalg.norm(d, axis=1, keepdims=True)
        pts = sp[s_idx, :3] + d * sp[s_idx, 3:4]
        dist = np.sqrt(((pts[:, None, :] - sp[None, :, :3]) ** 2).sum(axis=2)) - sp[None, :, 3]
        inside_other = (dist < -1e-6).any(axis=1)
        out.append(pts[~inside_other])
    pts = np.concatenate(out)[:n_points].astype(np.float32)
    q = _rng(seed, key, _A_QUERY).permutation(n_points)[:n_queries]
    return {"points": pts, "queries": pts[np.sort(q)]}


def make_encoder_input_proj(C: int, seed: int = 0, key: int = 0, dtype: str = "bf16") -> Dict[str, np.ndarray]:
    """The encoder's point-feature projection ``W_in [C,64]`` (columns 51..63
    face the zero pad lanes) ~ N(0, 0.02^2), rounded to bf16 for bf16 blocks,
    and ``b_in = 0``."""
    w = np.zeros((C, PE_PAD), np.float32)
    w[:, :PE_DIM] = (_rng(seed, key, _A_WIN).standard_normal((C, PE_DIM)) * 0.02).astype(np.float32)
    if dtype == "bf16":
        w = round_bf16(w)
    return {"W_in": w, "b_in": np.zeros((C,), np.float32)}


def make_local_decoder(spheres: np.ndarray, n_anchors=(4096, 16384), channels=(64, 32), hidden: int = 16,
                       fuse_hidden: int = 64, seed: int = 0, key: int = 0) -> Dict:
    """A two-scale latent hierarchy for the local (MSVS-style) decoder query and
    its weights: per scale s, anchors on the surface of a union of spheres
    (``n_anchors[s]`` points, as point-shuffle upsampling would place them near
    the surface), features ``~ N(0, 1)`` with ``channels[s]`` channels (halving
    from scale to scale), dynamic-weight MLP ``W1 [hidden,3] ~ N(0, 4^2)``
    (relative offsets are a few hundredths), ``b1 ~ N(0, 0.5^2)``,
    ``W2 [C,hidden] ~ N(0, 0.25^2)``, ``b2 = 0``; fusion ``Wf [fuse_hidden, sum C]
    ~ N(0, 0.1^2)``, ``bf = 0``, ``wo ~ N(0, 0.1^2)``, ``bo = 0`` (float32)."""
    out = {"anchors": [], "feats": [], "scales": []}
    for s, (n, C) in enumerate(zip(n_anchors, channels)):
        out["anchors"].append(make_point_cloud(spheres, n, 1, seed, key * 16 + s)["points"])
        r = _rng(seed, key * 16 + s, _A_LOCAL)
        out["feats"].append(r.standard_normal((n, C)).astype(np.float32))
        out["scales"].append({"W1": (r.standard_normal((hidden, 3)) * 4.0).astype(np.float32),
                              "b1": (r.standard_normal(hidden) * 0.5).astype(np.float32),
                              "W2": (r.standard_normal((C, hidden)) * 0.25).astype(np.float32),
                              "b2": np.zeros(C, np.float32)})
    r = _rng(seed, key, _A_LOCAL + 1)
    cs = int(sum(channels))
    out["fuse"] = {"Wf": (r.standard_normal((fuse_hidden, cs)) * 0.1).astype(np.float32),
                   "bf": np.zeros(fuse_hidden, np.float32),
                   "wo": (r.standard_normal(fuse_hidden) * 0.1).astype(np.float32),
                   "bo": np.zeros(1, np.float32)}
    return out


def make_inputs(cfg: Config, seed: int = 0, stress: bool = False) -> Dict[str, np.ndarray]:
    """All inputs of one workload: ``z``, ``weights`` and (if any) ``spheres``."""
    d = make_decoder(cfg.dec, seed=seed, key=cfg.seed_key, B=cfg.B, stress=stress)
    d["spheres"] = (make_spheres(cfg.n_spheres, seed, cfg.sphere_key, cfg.B)
                    if cfg.n_spheres else None)
    return d


def small_variant(cfg: Config, N: Optional[int] = None, R: Optional[int] = None,
                  r0: Optional[int] = None, top_k: Optional[int] = None,
                  n_probe: Optional[int] = None) -> Config:
    """Same structure as ``cfg`` at sizes a CPU oracle finishes in seconds."""
    dec = cfg.dec
    if N is not None:
        dec = replace(dec, N=N)
    kw = {"dec": dec}
    if R is not None:
        kw["grid_R"] = R
    if r0 is not None:
        kw["r0"] = r0
    if top_k is not None:
        kw["top_k"] = top_k
    if n_probe is not None:
        kw["n_probe"] = n_probe
    return replace(cfg, **kw)
