"""Python binding of the B200 vecset SDF decoder library (``libvdm.so``).

Argument marshalling only: every step of the decoder runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  The
functions carry the C names declared in ``include/vdm.h``:

    vdm_precompute_kv, vdm_decode_dense, vdm_select_kv,
    vdm_hierarchical_workspace_size, vdm_decode_hierarchical

Importing this package loads ``libvdm.so``; if the library is missing the
import fails (there is no fallback implementation).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvdm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m neural_sdf_volume_b200.build` "
        "(the CUDA library is required; there is no CPU path)")
_lib = C.CDLL(LIB_PATH)

MAX_LEVELS = 6
VDM_F32, VDM_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "workspace", 4: "cuda",
          5: "timeout", 6: "internal"}

EXPORTS = ("vdm_precompute_kv", "vdm_decode_dense", "vdm_select_kv",
           "vdm_hierarchical_workspace_size", "vdm_decode_hierarchical",
           "vdm_decode_hierarchical_noalloc", "vdm_compare_volumes",
           "vdm_surface_workspace_size", "vdm_extract_surface", "vdm_surface_case_table",
           "vdm_refine_workspace_size", "vdm_refine_level",
           "vdm_encode_workspace_size", "vdm_encode", "vdm_local_workspace_size", "vdm_decode_local",
           "vdm_debug_inject", "vdm_debug_exp2", "vdm_debug_gelu", "vdm_set_cta_pairs",
           "vdm_profile_begin", "vdm_profile_end",
           "vdm_status_string", "vdm_last_error", "vdm_abi_version")
PROF_CLASSES = ("kv", "decode", "select", "mark", "scan", "list", "fill", "probe")


class VdmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"vdm status {status} ({STATUS.get(status, '?')}): {msg}")
        self.status = status


class CDecoder(C.Structure):
    _fields_ = [("C", C.c_int32), ("H", C.c_int32), ("F", C.c_int32), ("query_ln", C.c_int32),
                ("dtype", C.c_int32),
                ("Wq", C.c_void_p), ("Wk", C.c_void_p), ("Wv", C.c_void_p), ("Wo", C.c_void_p),
                ("W1", C.c_void_p), ("W2", C.c_void_p),
                ("bq", C.c_void_p), ("bk", C.c_void_p), ("bv", C.c_void_p), ("bo", C.c_void_p),
                ("b1", C.c_void_p), ("b2", C.c_void_p),
                ("ln_kv_g", C.c_void_p), ("ln_kv_b", C.c_void_p),
                ("ln1_g", C.c_void_p), ("ln1_b", C.c_void_p), ("ln2_g", C.c_void_p), ("ln2_b", C.c_void_p),
                ("w_head", C.c_void_p), ("b_head", C.c_void_p),
                ("w_tsdf", C.c_void_p), ("b_tsdf", C.c_void_p)]


class CAnalytic(C.Structure):
    _fields_ = [("spheres", C.c_void_p), ("n_spheres", C.c_int32), ("dec_scale", C.c_float),
                ("tsdf_trunc", C.c_float)]


class CHierParams(C.Structure):
    _fields_ = [("r0", C.c_int32), ("n_levels", C.c_int32), ("adaptive", C.c_int32),
                ("tile", C.c_int32), ("n_probe", C.c_int32), ("top_k", C.c_int32),
                ("seed", C.c_uint64), ("tsdf_threshold", C.c_float)]


class CHierStats(C.Structure):
    _fields_ = [(n, C.c_int64 * MAX_LEVELS) for n in
                ("resolution", "decoded", "active_parents", "tiles", "selected_tiles", "probes")]


class CHierDebug(C.Structure):
    _fields_ = [("grid", C.c_void_p * MAX_LEVELS), ("active", C.c_void_p * MAX_LEVELS),
                ("dec", C.c_void_p * MAX_LEVELS), ("tile_ids", C.c_void_p * MAX_LEVELS),
                ("sel", C.c_void_p * MAX_LEVELS), ("max_tiles", C.c_int64),
                ("probes", C.c_void_p * MAX_LEVELS), ("scores", C.c_void_p * MAX_LEVELS),
                ("attn", C.c_void_p * MAX_LEVELS), ("attn_stride", C.c_int64),
                ("tsdf", C.c_void_p * MAX_LEVELS)]

DEBUG_ARRAYS = ("grid", "active", "dec", "tile_ids", "sel", "probes", "scores", "attn", "tsdf")


LOCAL_MAX_SCALES = 4


class CLocalDecoder(C.Structure):
    _fields_ = [("n_scales", C.c_int32), ("K", C.c_int32), ("hidden", C.c_int32), ("fuse_hidden", C.c_int32),
                ("n_anchors", C.c_int32 * LOCAL_MAX_SCALES), ("channels", C.c_int32 * LOCAL_MAX_SCALES)] + \
        [(n, C.c_void_p * LOCAL_MAX_SCALES) for n in ("anchors", "feats", "W1", "b1", "W2", "b2")] + \
        [(n, C.c_void_p) for n in ("Wf", "bf", "wo", "bo")]


class CProfile(C.Structure):
    _fields_ = [("launches", C.c_int64 * 8), ("ms", C.c_double * 8)]


_vp, _i32, _i64 = C.c_void_p, C.c_int32, C.c_int64
_lib.vdm_precompute_kv.argtypes = [C.POINTER(CDecoder), _vp, _i32, _i32, _vp, _vp, _vp]
_lib.vdm_decode_dense.argtypes = [C.POINTER(CDecoder), _vp, _vp, _i32, _i32, _vp, _i64, _i32,
                                  C.POINTER(CAnalytic), _vp, _vp]
_lib.vdm_select_kv.argtypes = [C.POINTER(CDecoder), _vp, _vp, _i32, _vp, _vp, _i32, _i64, _i32,
                               _vp, _vp, _vp, _vp]
_lib.vdm_hierarchical_workspace_size.argtypes = [C.POINTER(CDecoder), C.POINTER(CHierParams), _i32,
                                                 C.POINTER(C.c_size_t)]
_lib.vdm_decode_hierarchical.argtypes = [C.POINTER(CDecoder), _vp, _vp, _i32, _i32,
                                         C.POINTER(CHierParams), C.POINTER(CAnalytic), _vp, _vp,
                                         C.c_size_t, C.POINTER(CHierStats), C.POINTER(CHierDebug), _vp]
_lib.vdm_decode_hierarchical_noalloc.argtypes = [C.POINTER(CDecoder), _vp, _vp, _i32, _i32,
                                                 C.POINTER(CHierParams), C.POINTER(CAnalytic), _vp,
                                                 C.POINTER(CHierStats), C.POINTER(CHierDebug), _vp]
_lib.vdm_compare_volumes.argtypes = [_vp, _vp, _i64, _vp, _vp]
_lib.vdm_surface_workspace_size.argtypes = [_i32, C.POINTER(C.c_size_t)]
_lib.vdm_extract_surface.argtypes = [_vp, _i32, _vp, _i64, _vp, _i64, C.POINTER(C.c_int64),
                                     C.POINTER(C.c_int64), _vp, C.c_size_t, _vp]
_lib.vdm_surface_case_table.argtypes = [_vp, _vp]
_lib.vdm_refine_workspace_size.argtypes = [_i32, C.POINTER(C.c_size_t)]
_lib.vdm_refine_level.argtypes = [_vp, _i32, _vp, _vp, _vp, _vp, _vp, C.c_size_t, _vp]
_lib.vdm_encode_workspace_size.argtypes = [C.POINTER(CDecoder), _i32, C.POINTER(C.c_size_t)]
_lib.vdm_local_workspace_size.argtypes = [C.POINTER(CLocalDecoder), C.POINTER(C.c_size_t)]
_lib.vdm_decode_local.argtypes = [C.POINTER(CLocalDecoder), _vp, _i64, _vp, _vp, _vp, C.c_size_t, _vp]
_lib.vdm_encode.argtypes = [C.POINTER(CDecoder), _vp, _vp, _vp, _i32, _i32, _vp, _i32, _vp, _vp, C.c_size_t, _vp]
_lib.vdm_debug_inject.argtypes = [_i32, _i64]
_lib.vdm_debug_inject.restype = C.c_int
_lib.vdm_debug_exp2.argtypes = [C.c_void_p, C.c_void_p, _i64, C.c_void_p]
_lib.vdm_debug_exp2.restype = C.c_int
_lib.vdm_debug_gelu.argtypes = [C.c_void_p, C.c_void_p, _i64, C.c_void_p]
_lib.vdm_debug_gelu.restype = C.c_int
_lib.vdm_set_cta_pairs.argtypes = [_i32]
_lib.vdm_set_cta_pairs.restype = C.c_int
_lib.vdm_profile_begin.argtypes = []
_lib.vdm_profile_end.argtypes = [C.POINTER(CProfile)]
for _f in ("vdm_precompute_kv", "vdm_decode_dense", "vdm_select_kv",
           "vdm_hierarchical_workspace_size", "vdm_decode_hierarchical",
           "vdm_decode_hierarchical_noalloc", "vdm_compare_volumes", "vdm_profile_begin",
           "vdm_profile_end", "vdm_surface_workspace_size", "vdm_extract_surface",
           "vdm_surface_case_table", "vdm_refine_workspace_size", "vdm_refine_level",
           "vdm_encode_workspace_size", "vdm_encode", "vdm_local_workspace_size", "vdm_decode_local"):
    getattr(_lib, _f).restype = C.c_int
_lib.vdm_status_string.argtypes = [C.c_int]
_lib.vdm_status_string.restype = C.c_char_p
_lib.vdm_last_error.restype = C.c_char_p
_lib.vdm_abi_version.restype = C.c_int32


def _check(status: int):
    if status != 0:
        raise VdmError(status, _lib.vdm_last_error().decode(errors="replace"))


def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ----------------------------------------------------------------- decoder parameters
_MATS = ("Wq", "Wk", "Wv", "Wo", "W1", "W2")
_VECS = ("bq", "bk", "bv", "bo", "b1", "b2", "ln_kv_g", "ln_kv_b", "ln1_g", "ln1_b",
         "ln2_g", "ln2_b", "w_head", "b_head")


@dataclass
class Decoder:
    """Device-resident decoder parameters plus the C struct pointing at them."""
    C: int
    H: int
    F: int
    query_ln: bool
    dtype: str
    tensors: Dict[str, "object"]

    @staticmethod
    def from_numpy(weights: Dict[str, np.ndarray], C: int, H: int, F: int, query_ln: bool,
                   dtype: str, device="cuda") -> "Decoder":
        torch = _torch()
        tdt = torch.float32 if dtype == "f32" else torch.bfloat16
        t = {}
        for k in _MATS:
            t[k] = torch.from_numpy(np.ascontiguousarray(weights[k], np.float32)).to(device=device, dtype=tdt)
        for k in _VECS + (("w_tsdf", "b_tsdf") if "w_tsdf" in weights else ()):
            t[k] = torch.from_numpy(np.ascontiguousarray(weights[k], np.float32).reshape(-1)).to(device)
        return Decoder(C, H, F, bool(query_ln), dtype, t)

    @property
    def torch_dtype(self):
        torch = _torch()
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def cstruct(self) -> CDecoder:
        d = CDecoder()
        d.C, d.H, d.F, d.query_ln = self.C, self.H, self.F, int(self.query_ln)
        d.dtype = VDM_F32 if self.dtype == "f32" else VDM_BF16
        for k in _MATS + _VECS:
            setattr(d, k, self.tensors[k].data_ptr())
        if "w_tsdf" in self.tensors:   # optional truncated-SDF head
            d.w_tsdf = self.tensors["w_tsdf"].data_ptr()
            d.b_tsdf = self.tensors["b_tsdf"].data_ptr()
        return d


def _analytic(spheres, dec_scale: float, tsdf_trunc: float = 0.0):
    if spheres is None:
        return None
    a = CAnalytic()
    a.spheres = spheres.data_ptr()
    a.n_spheres = int(spheres.shape[1])
    a.dec_scale = float(dec_scale)
    a.tsdf_trunc = float(tsdf_trunc)
    return a


# ----------------------------------------------------------------- entry points
def vdm_precompute_kv(dec: Decoder, z, stream=None):
    """``z[B,N,C]`` float32 (device) -> ``K, V [B,H,N,64]`` in the decoder dtype."""
    torch = _torch()
    B, N, Cw = z.shape
    K = torch.empty((B, dec.H, N, 64), device=z.device, dtype=dec.torch_dtype)
    V = torch.empty_like(K)
    cd = dec.cstruct()
    _check(_lib.vdm_precompute_kv(C.byref(cd), z.data_ptr(), B, N, K.data_ptr(), V.data_ptr(),
                                  _stream(stream)))
    return K, V


def vdm_decode_dense(dec: Decoder, K, V, xyz=None, grid_R: int = 0, spheres=None,
                     dec_scale: float = 0.0, out=None, stream=None):
    """Decoder output at ``xyz[B,M,3]`` or at the voxels of the ``grid_R^3`` grid."""
    torch = _torch()
    B, H, N, _ = K.shape
    M = xyz.shape[1] if xyz is not None else grid_R ** 3
    if out is None:
        out = torch.empty((B, M), device=K.device, dtype=torch.float32)
    cd = dec.cstruct()
    an = _analytic(spheres, dec_scale)
    _check(_lib.vdm_decode_dense(C.byref(cd), K.data_ptr(), V.data_ptr(), B, N, _ptr(xyz), M,
                                 grid_R, C.byref(an) if an else None, out.data_ptr(), _stream(stream)))
    return out


def vdm_select_kv(dec: Decoder, K, V, probe_xyz, tile_off, top_k: int, want_scores: bool = False,
                  stream=None, want_probe_dec: bool = False):
    """Per sub-volume Top-K token ids ``[T, top_k]``, then (when asked) scores
    ``[T, N]`` and the probes' raw decoder output ``[P]``, in that order."""
    torch = _torch()
    N = K.shape[-2]
    T = int(tile_off.numel()) - 1
    P = int(probe_xyz.shape[0]) if probe_xyz is not None else 0
    sel = torch.empty((max(T, 0), top_k), device=K.device, dtype=torch.int32)
    score = torch.empty((max(T, 0), N), device=K.device, dtype=torch.float32) if want_scores else None
    pdec = torch.empty((P,), device=K.device, dtype=torch.float32) if want_probe_dec else None
    cd = dec.cstruct()
    _check(_lib.vdm_select_kv(C.byref(cd), K.data_ptr(), V.data_ptr(), N, _ptr(probe_xyz),
                              tile_off.data_ptr(), T, P, top_k, sel.data_ptr(), _ptr(score), _ptr(pdec),
                              _stream(stream)))
    out = (sel,)
    if want_scores:
        out += (score,)
    if want_probe_dec:
        out += (pdec,)
    return out if len(out) > 1 else sel


def hier_params(r0: int, n_levels: int, adaptive: bool = False, tile: int = 8, n_probe: int = 64,
                top_k: int = 1024, seed: int = 0, tsdf_threshold: float = 0.95) -> CHierParams:
    p = CHierParams()
    p.r0, p.n_levels, p.adaptive, p.tile = r0, n_levels, int(adaptive), tile
    p.n_probe, p.top_k, p.seed = n_probe, top_k, seed
    p.tsdf_threshold = tsdf_threshold
    return p


def vdm_hierarchical_workspace_size(dec: Decoder, params: CHierParams, N: int) -> int:
    n = C.c_size_t(0)
    cd = dec.cstruct()
    _check(_lib.vdm_hierarchical_workspace_size(C.byref(cd), C.byref(params), N, C.byref(n)))
    return int(n.value)


def vdm_decode_hierarchical(dec: Decoder, K, V, params: CHierParams, spheres=None,
                            dec_scale: float = 0.0, workspace=None, out=None, debug=None,
                            stream=None, tsdf_trunc: float = 0.0):
    """Coarse-to-fine decoding of B shapes -> (grid ``[B,Rf,Rf,Rf]``, per-shape stats).

    ``debug`` is an optional dict of device tensors keyed like ``vdm_hier_debug``
    (``grid``, ``active``, ``dec``, ``tile_ids``, ``sel``, ``probes``, ``scores``,
    ``attn``: lists indexed by level, plus ``max_tiles`` and ``attn_stride``)."""
    torch = _torch()
    B, H, N, _ = K.shape
    Rf = params.r0 << (params.n_levels - 1)
    if out is None:
        out = torch.empty((B, Rf, Rf, Rf), device=K.device, dtype=torch.float32)
    if workspace is None:
        nbytes = vdm_hierarchical_workspace_size(dec, params, N)
        workspace = torch.empty((nbytes,), device=K.device, dtype=torch.uint8)
    stats = (CHierStats * B)()
    dbg = None
    if debug is not None:
        dbg = CHierDebug()
        for key in DEBUG_ARRAYS:
            arr = getattr(dbg, key)
            for l, t in enumerate(debug.get(key, [])):
                arr[l] = _ptr(t) or 0
        dbg.max_tiles = int(debug.get("max_tiles", 0))
        dbg.attn_stride = int(debug.get("attn_stride", 0))
    cd = dec.cstruct()
    an = _analytic(spheres, dec_scale, tsdf_trunc)
    _check(_lib.vdm_decode_hierarchical(C.byref(cd), K.data_ptr(), V.data_ptr(), B, N,
                                        C.byref(params), C.byref(an) if an else None,
                                        out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                        stats, C.byref(dbg) if dbg else None, _stream(stream)))
    st = [{k: list(getattr(stats[b], k)) for k in ("resolution", "decoded", "active_parents",
                                                    "tiles", "selected_tiles", "probes")}
          for b in range(B)]
    return out, st


def vdm_decode_hierarchical_noalloc(dec: Decoder, K, V, params: CHierParams, spheres=None,
                                    dec_scale: float = 0.0, out=None, stream=None):
    """``vdm_decode_hierarchical`` with the library's built-in 32 MiB scratch
    instead of a caller workspace (for callers that may not allocate device
    memory).  Only the output grid is passed in."""
    torch = _torch()
    B, H, N, _ = K.shape
    Rf = params.r0 << (params.n_levels - 1)
    if out is None:
        out = torch.empty((B, Rf, Rf, Rf), device=K.device, dtype=torch.float32)
    stats = (CHierStats * B)()
    cd = dec.cstruct()
    an = _analytic(spheres, dec_scale)
    _check(_lib.vdm_decode_hierarchical_noalloc(C.byref(cd), K.data_ptr(), V.data_ptr(), B, N,
                                                C.byref(params), C.byref(an) if an else None,
                                                out.data_ptr(), stats, None, _stream(stream)))
    return out


def vdm_compare_volumes(a, b, stream=None) -> Dict[str, float]:
    """Counts of two same-shaped float32 device volumes: inside each (f < 0),
    inside both, same sign, and the largest |a - b|; plus V-IoU and sign
    agreement derived from them."""
    torch = _torch()
    assert a.shape == b.shape and a.dtype == torch.float32 and b.dtype == torch.float32
    a = a.contiguous()
    b = b.contiguous()
    out = torch.empty((5,), device=a.device, dtype=torch.int64)
    _check(_lib.vdm_compare_volumes(a.data_ptr(), b.data_ptr(), a.numel(), out.data_ptr(),
                                    _stream(stream)))
    c = out.cpu().numpy().astype(np.uint64)
    n = int(a.numel())
    in_a, in_b, both, same = (int(x) for x in c[:4])
    union = in_a + in_b - both
    dmax = float(np.array([int(c[4]) & 0xFFFFFFFF], np.uint32).view(np.float32)[0])
    return {"n": n, "inside_a": in_a, "inside_b": in_b, "inside_both": both, "same_sign": same,
            "v_iou": both / union if union else 1.0, "sign_agreement": same / n if n else 1.0,
            "max_abs_diff": dmax}


def vdm_encode(block: Decoder, W_in, b_in, points, queries, stream=None):
    """Vecsets ``[B, N, C]`` (float32) of point clouds ``points[B, M, 3]`` with
    latent tokens at ``queries[B, N, 3]``; ``block`` holds the cross-attention
    block (decoder layout), ``W_in [C, 64]`` (block dtype) and ``b_in [C]`` the
    point-feature projection."""
    torch = _torch()
    B, M, _ = points.shape
    N = queries.shape[1]
    cd = block.cstruct()
    n = C.c_size_t(0)
    _check(_lib.vdm_encode_workspace_size(C.byref(cd), M, C.byref(n)))
    ws = torch.empty((n.value,), device=points.device, dtype=torch.uint8)
    z = torch.empty((B, N, block.C), device=points.device, dtype=torch.float32)
    _check(_lib.vdm_encode(C.byref(cd), W_in.data_ptr(), b_in.data_ptr(), points.contiguous().data_ptr(), B, M,
                           queries.contiguous().data_ptr(), N, z.data_ptr(), ws.data_ptr(), ws.numel(),
                           _stream(stream)))
    return z


@dataclass
class LocalDecoder:
    """Device-resident multi-scale anchors and weights of the local decoder."""
    K: int
    tensors: Dict[str, "object"]
    cs: "object" = None

    @staticmethod
    def from_numpy(d: Dict, K: int, device="cuda") -> "LocalDecoder":
        torch = _torch()
        t = {}
        for s, (a, f, w) in enumerate(zip(d["anchors"], d["feats"], d["scales"])):
            t[f"anchors{s}"] = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)
            t[f"feats{s}"] = torch.from_numpy(np.ascontiguousarray(f, np.float32)).to(device)
            for k in ("W1", "b1", "W2", "b2"):
                t[f"{k}{s}"] = torch.from_numpy(np.ascontiguousarray(w[k], np.float32)).to(device)
        for k in ("Wf", "bf", "wo", "bo"):
            t[k] = torch.from_numpy(np.ascontiguousarray(d["fuse"][k], np.float32)).to(device)
        ld = LocalDecoder(K, t)
        c = CLocalDecoder()
        c.n_scales = len(d["anchors"])
        c.K = K
        c.hidden = int(d["scales"][0]["W1"].shape[0])
        c.fuse_hidden = int(d["fuse"]["Wf"].shape[0])
        for s in range(c.n_scales):
            c.n_anchors[s] = int(d["anchors"][s].shape[0])
            c.channels[s] = int(d["feats"][s].shape[1])
            c.anchors[s] = t[f"anchors{s}"].data_ptr()
            c.feats[s] = t[f"feats{s}"].data_ptr()
            for k in ("W1", "b1", "W2", "b2"):
                getattr(c, k)[s] = t[f"{k}{s}"].data_ptr()
        for k in ("Wf", "bf", "wo", "bo"):
            setattr(c, k, t[k].data_ptr())
        ld.cs = c
        return ld


def vdm_decode_local(ld: LocalDecoder, xyz, want_knn: bool = False, workspace=None, stream=None):
    """SDF of the local decoder at ``xyz[M, 3]`` (float32, device); with
    ``want_knn`` also the neighbour indices ``[M, n_scales, K]``."""
    torch = _torch()
    M = int(xyz.shape[0])
    out = torch.empty((M,), device=xyz.device, dtype=torch.float32)
    knn = (torch.empty((M, ld.cs.n_scales, ld.K), device=xyz.device, dtype=torch.int32) if want_knn else None)
    if workspace is None:
        n = C.c_size_t(0)
        _check(_lib.vdm_local_workspace_size(C.byref(ld.cs), C.byref(n)))
        workspace = torch.empty((n.value,), device=xyz.device, dtype=torch.uint8)
    _check(_lib.vdm_decode_local(C.byref(ld.cs), xyz.contiguous().data_ptr(), M, out.data_ptr(), _ptr(knn),
                                 workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return (out, knn) if want_knn else out


def vdm_refine_workspace_size(R: int) -> int:
    n = C.c_size_t(0)
    _check(_lib.vdm_refine_workspace_size(R, C.byref(n)))
    return int(n.value)


def vdm_refine_level(f, fine=None, parents=None, workspace=None, stream=None):
    """One level step without the decoder: ``f[R,R,R]`` -> (refine mask words
    ``[(R/4)^3]`` int64 view of uint64, device counts ``[2]``); fills ``fine``
    ``[2R,2R,2R]`` with parent values and ``parents`` ``[R^3]`` when given."""
    torch = _torch()
    R = int(f.shape[-1])
    if workspace is None:
        workspace = torch.empty((vdm_refine_workspace_size(R),), device=f.device, dtype=torch.uint8)
    mask = torch.empty(((R // 4) ** 3,), device=f.device, dtype=torch.int64)
    counts = torch.zeros((2,), device=f.device, dtype=torch.int32)
    _check(_lib.vdm_refine_level(f.data_ptr(), R, _ptr(fine), mask.data_ptr(), _ptr(parents),
                                 counts.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                 _stream(stream)))
    return mask, counts


def vdm_surface_workspace_size(R: int) -> int:
    n = C.c_size_t(0)
    _check(_lib.vdm_surface_workspace_size(R, C.byref(n)))
    return int(n.value)


def vdm_extract_surface(f, workspace=None, stream=None):
    """Marching-cubes mesh of a float32 device volume ``f[R,R,R]``:
    ``(vertices [V,3] float32, triangles [T,3] int32)`` on the device."""
    torch = _torch()
    R = int(f.shape[-1])
    f = f.contiguous()
    if workspace is None:
        workspace = torch.empty((vdm_surface_workspace_size(R),), device=f.device, dtype=torch.uint8)
    nv, nt = C.c_int64(0), C.c_int64(0)
    st = _lib.vdm_extract_surface(f.data_ptr(), R, None, 0, None, 0, C.byref(nv), C.byref(nt),
                                  workspace.data_ptr(), workspace.numel(), _stream(stream))
    if st not in (0, 3):
        _check(st)
    verts = torch.empty((nv.value, 3), device=f.device, dtype=torch.float32)
    tris = torch.empty((nt.value, 3), device=f.device, dtype=torch.int32)
    if nv.value or nt.value:
        _check(_lib.vdm_extract_surface(f.data_ptr(), R, verts.data_ptr(), nv.value, tris.data_ptr(),
                                        nt.value, C.byref(nv), C.byref(nt), workspace.data_ptr(),
                                        workspace.numel(), _stream(stream)))
    return verts, tris


def vdm_surface_case_table():
    """The library's generated marching-cubes case table: ``(ntri[256], tri[256,5,3])``."""
    ntri = np.zeros(256, np.uint8)
    tri = np.zeros((256, 5, 3), np.uint8)
    _check(_lib.vdm_surface_case_table(ntri.ctypes.data, tri.ctypes.data))
    return ntri, tri


def vdm_debug_inject(mode: int, timeout_cycles: int = 0):
    """Test hook: mode 1 withholds one completion signal in the next
    tensor-core decode launch (its bounded waits then report a timeout)."""
    _check(_lib.vdm_debug_inject(mode, timeout_cycles))


def vdm_debug_exp2(x, stream=None):
    """Test hook: 2^x (float32 CUDA tensor) by the decoder softmax's polynomial form."""
    import torch

    x = x.contiguous()
    if x.dtype != torch.float32 or not x.is_cuda:
        raise ValueError("x must be a float32 CUDA tensor")
    y = torch.empty_like(x)
    _check(_lib.vdm_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), _stream(stream)))
    return y


def vdm_debug_gelu(x, stream=None):
    """Test hook: the decoder's GELU of x (float32 CUDA tensor) as ``(bf16 pair form, float32 scalar form)``."""
    import torch

    x = x.contiguous()
    if x.dtype != torch.float32 or not x.is_cuda:
        raise ValueError("x must be a float32 CUDA tensor")
    y = torch.empty(2 * x.numel(), dtype=torch.float32, device=x.device)
    _check(_lib.vdm_debug_gelu(x.data_ptr(), y.data_ptr(), x.numel(), _stream(stream)))
    return y[: x.numel()].view_as(x), y[x.numel():].view_as(x)


def vdm_set_cta_pairs(enable: bool):
    """Run tensor-core decoding on CTA pairs (True) or one CTA per MMA (False, the default)."""
    _check(_lib.vdm_set_cta_pairs(1 if enable else 0))


def vdm_profile_begin():
    """Start bracketing this thread's kernel launches with CUDA events."""
    _check(_lib.vdm_profile_begin())


def vdm_profile_end() -> Dict[str, Dict[str, float]]:
    """Wait for the recorded events; per kernel class: launches and device ms."""
    p = CProfile()
    _check(_lib.vdm_profile_end(C.byref(p)))
    return {n: {"launches": int(p.launches[i]), "ms": float(p.ms[i])}
            for i, n in enumerate(PROF_CLASSES)}


def abi_version() -> int:
    return int(_lib.vdm_abi_version())
