"""Pins of the adaptive-KV oracle: published SplitMix64 outputs, brute-force
ranking and Top-K, closed forms (identical keys/values) and the k = N
identity with dense decoding (no GPU)."""
import os

import numpy as np
import pytest

import workloads as W
from oracle import adaptive as A
from oracle import decoder as D
from oracle import hierarchy as HV
from oracle import volume as VOL

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_stream():
    for line in open(os.path.join(GOLD, "splitmix64_state0.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        _, state, out = line.split()
        assert int(A.splitmix64(np.uint64(int(state, 16)))) == int(out, 16)


def test_probe_choice_is_smallest_keys_brute_force():
    rng = np.random.default_rng(0)
    idx = np.sort(rng.choice(10 ** 6, 300, replace=False))
    m = A.choose_probes(idx, 64, seed=5, level=2)
    assert m.sum() == 64
    salt = int(A.splitmix64(np.uint64(5) ^ (np.uint64(2) << np.uint64(32))))
    keys = [(int(A.splitmix64(np.uint64(int(i) ^ salt))), int(i)) for i in idx]
    want = set(i for _, i in sorted(keys)[:64])
    assert set(idx[m].tolist()) == want
    # at most n_probe queries: all are probes
    assert A.choose_probes(idx[:64], 64, 5, 2).all()
    # different level -> different sample
    assert set(idx[A.choose_probes(idx, 64, 5, 1)].tolist()) != want


def test_top_k_brute_force_with_ties():
    rng = np.random.default_rng(1)
    s = rng.integers(0, 20, 200).astype(np.float64)     # many ties
    for k in (1, 7, 64, 199, 200, 500):
        want = sorted(sorted(range(200), key=lambda j: (-s[j], j))[:k])
        np.testing.assert_array_equal(A.top_k(s, k), want)


def test_tile_binning():
    R, t = 16, 8
    idx = np.arange(R ** 3)
    tid = A.tile_of(idx, R, t)
    assert tid.max() == 7 and np.bincount(tid).tolist() == [512] * 8
    i, rem = np.divmod(idx, R * R); j, k = np.divmod(rem, R)
    np.testing.assert_array_equal(tid, ((i // 8) * 2 + j // 8) * 2 + k // 8)


def _small_setup(key=3, stress=False, N=48):
    spec = W.DecoderSpec(C=128, H=2, F=128, N=N, query_ln=True, dtype="f32")
    d = W.make_decoder(spec, seed=0, key=key, stress=stress)
    K, V = D.precompute_kv(d["z"][0], d["weights"])
    sp = W.make_spheres(4, 0, key)[0]
    return d["weights"], K, V, sp


def test_identical_keys_give_equal_scores_and_first_k_tokens():
    w, K, V, sp = _small_setup()
    Kc = np.repeat(K[:, :1], K.shape[1], axis=1)
    q = A.query_vectors(D.grid_points(16, np.arange(10)), w)
    sc = A.token_scores(q, Kc)
    np.testing.assert_allclose(sc, 10 * 2 / K.shape[1], rtol=1e-12)
    np.testing.assert_array_equal(A.top_k(sc, 5), np.arange(5))


def test_scores_sum_to_probes_times_heads():
    w, K, V, sp = _small_setup(stress=True)
    q = A.query_vectors(D.grid_points(16, np.arange(0, 4096, 97)), w)
    assert A.token_scores(q, K).sum() == pytest.approx(q.shape[0] * 2, rel=1e-12)


def test_adaptive_with_k_equal_n_is_dense():
    w, K, V, sp = _small_setup(stress=True)
    R = 16
    kids = np.arange(0, R ** 3, 3)
    ad = A.adaptive_level(1, R, kids, K, V, w, True, sp, 0.01, seed=0, n_probe=8, k=K.shape[1])
    dense = D.decode_points(D.grid_points(R, kids), K, V, w, True)
    np.testing.assert_allclose(ad["dec"], dense, atol=1e-12)


def test_adaptive_identical_values_closed_form():
    # identical V rows: the attention output is that row for any subset, so
    # adaptive decoding equals dense decoding at every query
    w, K, V, sp = _small_setup(stress=True)
    Vc = np.repeat(V[:, 5:6], V.shape[1], axis=1)
    R = 16
    kids = np.arange(0, R ** 3, 2)
    ad = A.adaptive_level(1, R, kids, K, Vc, w, True, sp, 0.01, seed=0, n_probe=8, k=4,
                          keep_tiles=True)
    dense = D.decode_points(D.grid_points(R, kids), K, Vc, w, True)
    np.testing.assert_allclose(ad["dec"], dense, atol=1e-12)
    assert any("sel" in t and t["sel"].size == 4 for t in ad["tiles"].values())


def test_adaptive_small_tiles_are_dense_and_probes_exact():
    w, K, V, sp = _small_setup(stress=True)
    R = 16
    kids = np.arange(0, R ** 3, 37)          # few queries per tile
    ad = A.adaptive_level(2, R, kids, K, V, w, True, sp, 0.01, seed=1, n_probe=8, k=6,
                          keep_tiles=True)
    dense = D.decode_points(D.grid_points(R, kids), K, V, w, True)
    pos = {int(v): n for n, v in enumerate(kids)}
    for t in ad["tiles"].values():
        rows = [pos[int(v)] for v in t["idx"][t["probe"]]]
        np.testing.assert_allclose(ad["dec"][rows], dense[rows], atol=1e-12)
        if t["idx"].size <= 8:
            assert t["probe"].all() and "sel" not in t


def test_hierarchical_adaptive_runs_and_counts():
    w, K, V, sp = _small_setup(stress=False)
    res = VOL.hierarchical_volume(K, V, w, 8, 3, True, sp, 0.01, adaptive=True, seed=0,
                                  n_probe=16, top_k=24, keep_tiles=True)
    lv = res["levels"]
    assert lv[2]["R"] == 32 and res["grid"].shape == (32, 32, 32)
    for L in (1, 2):
        assert lv[L]["children"].size == 8 * lv[L - 1]["parents"].size
        # every decoded child belongs to a tile record
        n = sum(t["idx"].size for t in lv[L]["tiles"].values())
        assert n == lv[L]["children"].size


def _unxorshift(z: int, s: int) -> int:
    # inverse of z ^= z >> s on 64-bit words
    x = z
    for _ in range(64 // s + 1):
        x = z ^ (x >> s)
    return x & (2 ** 64 - 1)


def test_probe_keys_are_distinct_for_distinct_voxels():
    """splitmix64 is a bijection of 64-bit words (an added constant, xor-shifts and
    multiplications by odd constants are each invertible), and so is the xor with one
    salt: distinct voxel indices get distinct probe keys, so the smaller-index tie-break
    of the probe rule never decides anything.  Checked by inverting the mix on random
    words, and by the keys of a million consecutive indices being distinct."""
    mask = 2 ** 64 - 1
    m1, m2, golden = int(A._M1), int(A._M2), int(A._GOLDEN)
    inv1, inv2 = pow(m1, -1, 2 ** 64), pow(m2, -1, 2 ** 64)
    rng = np.random.default_rng(3)
    for x in rng.integers(0, 2 ** 63, 200, dtype=np.int64).tolist() + [0, 1, mask]:
        z = int(A.splitmix64(np.uint64(x)))
        z = _unxorshift(z, 31)
        z = _unxorshift((z * inv2) & mask, 27)
        z = _unxorshift((z * inv1) & mask, 30)
        assert (z - golden) & mask == x
    keys = A.probe_key(0, 2, np.arange(2 ** 20, dtype=np.int64))
    assert np.unique(keys).size == keys.size
