"""Pins of the oracle's Philox generator and block Hadamard transforms."""
import json
import os

import numpy as np
import scipy.linalg
import scipy.stats

from oracle import hadamard as hd
from oracle import philox

KAT = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")))


def test_philox_known_answers():
    for v in KAT["vectors"]:
        c = [int(h, 16) for h in v["ctr"]]
        k = [int(h, 16) for h in v["key"]]
        out = philox.philox4x32_10(*c, *k)
        assert ["%08x" % int(o) for o in out] == v["out"]


def test_philox_stream_layout():
    # word idx&3 of the block for counter (idx>>2, 0, tag, tensor_tag), key = seed
    seed = 0x123456789ABCDEF0
    idx = np.arange(64, dtype=np.uint64)
    w = philox.words(seed, idx, 5, 9)
    for i in (0, 1, 2, 3, 4, 37, 63):
        blk = philox.philox4x32_10(i >> 2, 0, 5, 9, seed & 0xFFFFFFFF, seed >> 32)
        assert int(w[i]) == int(blk[i & 3])
    # high index bits land in counter word 1
    big = np.array([(1 << 34) + 5], dtype=np.uint64)
    blk = philox.philox4x32_10((1 << 32) + 1 & 0xFFFFFFFF, 1, 5, 9, seed & 0xFFFFFFFF, seed >> 32)
    assert int(philox.words(seed, big, 5, 9)[0]) == int(blk[1])


def test_philox_uniformity():
    u = philox.uniform(7, np.arange(1 << 18, dtype=np.uint64), philox.TAG_SR_ELEM, 1)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert scipy.stats.kstest(u, "uniform").pvalue > 1e-3
    # streams with different tags / tensor tags / seeds are unrelated
    v = philox.uniform(7, np.arange(1 << 18, dtype=np.uint64), philox.TAG_SR_ELEM, 2)
    assert abs(np.corrcoef(u, v)[0, 1]) < 0.01
    s = philox.rht_signs(3, 0, 1 << 16)
    assert abs(s.mean()) < 0.02 and set(np.unique(s)) == {-1.0, 1.0}


def test_sylvester_matches_scipy_and_is_orthogonal():
    for g in (2, 16, 32, 64, 128, 256):
        h = hd.sylvester(g)
        np.testing.assert_array_equal(h, scipy.linalg.hadamard(g))
        hn = h / np.sqrt(g)
        np.testing.assert_allclose(hn @ hn.T, np.eye(g), atol=1e-14)
        np.testing.assert_array_equal(h, h.T)          # symmetric, so H^-1 = H


def test_fwht_of_basis_vectors_is_exact():
    for g in (16, 32, 64, 128, 256):
        e = np.eye(g, dtype=np.float32)
        y = hd.fwht_f32(e, g)
        want = (scipy.linalg.hadamard(g) * np.float64(hd.hadamard_scale(g))).astype(np.float32)
        np.testing.assert_array_equal(y, want.T)
    assert hd.hadamard_scale(16) == np.float32(0.25)
    assert hd.hadamard_scale(32).view(np.uint32) == 0x3E3504F3
    assert hd.hadamard_scale(128).view(np.uint32) == 0x3DB504F3


def test_fwht_f32_close_to_exact_transform():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    for g in (16, 32, 64, 128, 256):
        for rz in (False, True):
            y = hd.block_transform(x, g, rz, seed=11, sign_tag=3).astype(np.float64)
            ref = hd.block_transform_f64(x, g, rz, seed=11, sign_tag=3)
            scale = np.abs(x).reshape(64, -1, g).sum(-1).repeat(g, -1) / np.sqrt(g)
            assert np.all(np.abs(y - ref) <= 8 * 2.0 ** -24 * scale + 1e-30)


def test_rotation_cancels_on_inner_dimension():
    """<RHT a, RHT b> = <a, b> for operands rotated with the same signs
    (Quartet II page, computation graph step 5)."""
    rng = np.random.default_rng(1)
    a = rng.standard_normal((32, 256)).astype(np.float32)
    b = rng.standard_normal((48, 256)).astype(np.float32)
    ra = hd.block_transform(a, 128, True, seed=5, sign_tag=0).astype(np.float64)
    rb = hd.block_transform(b, 128, True, seed=5, sign_tag=0).astype(np.float64)
    ref = a.astype(np.float64) @ b.astype(np.float64).T
    bound = np.abs(a).astype(np.float64) @ np.abs(b).astype(np.float64).T
    assert np.all(np.abs(ra @ rb.T - ref) <= 1e-5 * bound)
    # different signs do not cancel
    rc = hd.block_transform(b, 128, True, seed=6, sign_tag=0).astype(np.float64)
    assert np.abs(ra @ rc.T - ref).max() > 1.0


def test_inverse_h_roundtrip():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((8, 96))
    y = hd.block_transform_f64(x, 32, False)
    np.testing.assert_allclose(hd.inverse_block_h_f64(y, 32), x, atol=1e-12)
