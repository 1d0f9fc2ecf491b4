"""The C-ABI library loads and exports every entry point of include/vdm.h, and
argument errors come back as status codes before any device work (no GPU)."""
import ctypes as C
import os
import re

import pytest

import neural_sdf_volume_b200 as vdm
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "vdm.h")).read()
    return sorted(set(re.findall(r"VDM_API\s+[\w\s\*]+?\b(vdm_\w+)\s*\(", src)))


def test_every_declared_function_is_exported():
    names = _header_functions()
    assert len(names) == len(vdm.EXPORTS), names
    for n in names:
        assert hasattr(vdm._lib, n), n
    assert set(names) == set(vdm.EXPORTS)


def test_status_strings_and_version():
    assert vdm.abi_version() == 3
    assert vdm._lib.vdm_status_string(0) == b"ok"
    assert vdm._lib.vdm_status_string(3) == b"workspace too small"


def _fake_decoder(C_=512, H=8, F=2048, dtype=vdm.VDM_BF16):
    d = vdm.CDecoder()
    d.C, d.H, d.F, d.query_ln, d.dtype = C_, H, F, 1, dtype
    addr = 0x10000
    for name, _ in vdm.CDecoder._fields_[5:]:
        setattr(d, name, addr)
        addr += 0x10000
    return d


def _ws(d, p, N):
    n = C.c_size_t(0)
    st = vdm._lib.vdm_hierarchical_workspace_size(C.byref(d), C.byref(p), N, C.byref(n))
    return st, n.value


def test_shape_limits_are_reported():
    p = vdm.hier_params(96, 3)
    assert _ws(_fake_decoder(C_=500, H=8), p, 3072)[0] == 2          # C != 64 H
    assert _ws(_fake_decoder(C_=1024, H=16), p, 3072)[0] == 2        # C too wide
    assert _ws(_fake_decoder(F=100), p, 3072)[0] == 2                 # F not a multiple of 64
    assert _ws(_fake_decoder(), p, 9000)[0] == 2                      # N too large
    assert _ws(_fake_decoder(), vdm.hier_params(90, 3), 3072)[0] == 2   # r0 % 4
    assert _ws(_fake_decoder(), vdm.hier_params(96, 3, adaptive=True, tile=16), 3072)[0] == 2
    assert b"r0" in vdm._lib.vdm_last_error() or b"edge" in vdm._lib.vdm_last_error()


def test_null_arguments_are_rejected():
    d = _fake_decoder()
    d.W1 = 0
    st = vdm._lib.vdm_decode_dense(C.byref(d), 0x1000, 0x2000, 1, 16, None, 8, 2, None, 0x3000, None)
    assert st == 1 and b"W1" in vdm._lib.vdm_last_error()
    assert vdm._lib.vdm_decode_dense(None, 0x1000, 0x2000, 1, 16, None, 8, 2, None, 0x3000, None) == 1
    d = _fake_decoder()
    # grid mode needs M == R^3
    assert vdm._lib.vdm_decode_dense(C.byref(d), 0x1000, 0x2000, 1, 16, None, 9, 2, None, 0x3000, None) == 1
    # misaligned matrix
    d.Wo = 0x10002
    assert vdm._lib.vdm_decode_dense(C.byref(d), 0x1000, 0x2000, 1, 16, None, 8, 2, None, 0x3000, None) == 1
    # M == 0 is a no-op
    d = _fake_decoder()
    assert vdm._lib.vdm_decode_dense(C.byref(d), 0x1000, 0x2000, 1, 16, None, 0, 0, None, 0x3000, None) == 0


def test_select_rejects_bad_top_k():
    d = _fake_decoder()
    st = vdm._lib.vdm_select_kv(C.byref(d), 0x1000, 0x2000, 64, 0x3000, 0x4000, 2, 10, 65, 0x5000, None, None, None)
    assert st == 1


@pytest.mark.parametrize("cid", [3, 4, 5])
def test_workspace_sizes_and_too_small_workspace(cid):
    cfg = W.CONFIGS[cid]
    d = _fake_decoder(cfg.dec.C, cfg.dec.H, cfg.dec.F)
    p = vdm.hier_params(cfg.r0, cfg.n_levels, cfg.adaptive, cfg.tile, cfg.n_probe, cfg.top_k)
    st, n = _ws(d, p, cfg.dec.N)
    assert st == 0
    R1 = cfg.r0 * 2
    assert n >= 4 * (cfg.r0 ** 3 + R1 ** 3)          # intermediate grids at least
    assert n < 4 << 30
    stats = (vdm.CHierStats * 1)()
    st = vdm._lib.vdm_decode_hierarchical(C.byref(d), 0x1000, 0x2000, 1, cfg.dec.N, C.byref(p), None,
                                          0x3000, 0x4000, n - 1024, stats, None, None)
    assert st == 3 and b"workspace" in vdm._lib.vdm_last_error()


def test_compare_volumes_argument_errors():
    lib = vdm._lib
    assert lib.vdm_compare_volumes(None, None, -1, 0x1000, None) == 1        # negative size
    assert lib.vdm_compare_volumes(None, None, 10, 0x1000, None) == 1        # null inputs
    assert lib.vdm_compare_volumes(0x1000, 0x2000, 10, 0x1004, None) == 1    # misaligned out


def test_surface_case_table_equals_the_oracle_rules():
    """Host logic, no GPU: the library generates its marching-cubes table from the
    stated face and fan rules; every one of the 256 sign patterns gives exactly
    the oracle's triangles (edge ids, order)."""
    from oracle import surface as OS
    ntri, tri = vdm.vdm_surface_case_table()
    for cfg in range(256):
        want = OS.cube_triangles(cfg)
        assert ntri[cfg] == len(want), cfg
        assert [tuple(int(x) for x in t) for t in tri[cfg, :ntri[cfg]]] == [tuple(t) for t in want], cfg


def test_surface_workspace_and_argument_errors():
    n = C.c_size_t(0)
    assert vdm._lib.vdm_surface_workspace_size(12, C.byref(n)) == 2       # R % 8
    assert vdm._lib.vdm_surface_workspace_size(2048, C.byref(n)) == 2     # too large
    assert vdm._lib.vdm_surface_workspace_size(64, C.byref(n)) == 0 and n.value > 64 ** 3
    nv, nt = C.c_int64(0), C.c_int64(0)
    assert vdm._lib.vdm_extract_surface(None, 64, None, 0, None, 0, C.byref(nv), C.byref(nt),
                                        0x1000, n.value, None) == 1
