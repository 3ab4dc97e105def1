"""Pins the oracle's Philox4x32-10 and dropout contract.

cuRAND's host-side PHILOX4_32_10 generator is an implementation independent
of the oracle's (and runs without a GPU).  Its output block i, for offset 0,
is Philox((i div 65536, 0, i mod 65536, 0), key = (seed lo, seed hi)); a
generator offset of o*4*65536 words adds o to the 64-bit (c0, c1) pair.
"""
import ctypes
import glob
import os

import numpy as np
import pytest

from oracle import dropout_keep, dropout_threshold, philox4x32_10
from oracle.layer import dropout_lanes


def _curand():
    import torch  # noqa: F401  (locates the bundled nvidia wheels)
    cands = []
    for p in __import__("sys").path:
        cands += glob.glob(os.path.join(p, "nvidia", "curand", "lib", "libcurand.so*"))
    cands += glob.glob("/usr/local/cuda/lib64/libcurand.so*")
    for c in cands:
        try:
            return ctypes.CDLL(c)
        except OSError:
            continue
    return None


LIB = _curand()
PHILOX = 161  # CURAND_RNG_PSEUDO_PHILOX4_32_10


def _curand_words(seed, offset, n):
    gen = ctypes.c_void_p()
    assert LIB.curandCreateGeneratorHost(ctypes.byref(gen), PHILOX) == 0
    try:
        assert LIB.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert LIB.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
        out = np.zeros(n, dtype=np.uint32)
        assert LIB.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(n)) == 0
        return out.reshape(-1, 4)
    finally:
        LIB.curandDestroyGenerator(gen)


@pytest.mark.skipif(LIB is None, reason="libcurand not found")
@pytest.mark.parametrize("seed", [0, 1234, 0xDEADBEEFCAFEF00D])
@pytest.mark.parametrize("base", [0, 3, 1 << 32, (1 << 32) + 5])
def test_philox_matches_curand_host(seed, base):
    nblk = 65536 * 2 + 64
    ref = _curand_words(seed, base * 4 * 65536, 4 * nblk)
    i = np.arange(nblk, dtype=np.uint64)
    c01 = np.uint64(base) + i // np.uint64(65536)
    c2 = i % np.uint64(65536)
    w = philox4x32_10(c01 & np.uint64(0xFFFFFFFF), c01 >> np.uint64(32), c2, 0,
                      seed & 0xFFFFFFFF, seed >> 32)
    mine = np.stack(w, axis=1).astype(np.uint32)
    assert np.array_equal(mine, ref)


def test_lane_layout():
    # lane k of group g is the 16-bit half (k & 1) of word (k >> 1), low half first
    w = philox4x32_10(5, 0, 2, 7, 1234, 0)
    lanes = dropout_lanes(40, 8, 2, 7, 1234)
    want = [(int(w[k >> 1]) >> (16 * (k & 1))) & 0xFFFF for k in range(8)]
    assert lanes.tolist() == want


def test_threshold():
    assert dropout_threshold(0.0) == 0
    assert dropout_threshold(0.1) == 6553
    assert dropout_threshold(np.float32(0.1)) == 6553
    assert dropout_threshold(0.5) == 32768


def test_p_zero_keeps_everything():
    assert dropout_keep(0, 1 << 16, 0, 0, 1234, 0.0).all()


@pytest.mark.parametrize("site", [0, 1, 2])
def test_kept_fraction(site):
    n = 1 << 20
    p = 0.1
    keep = dropout_keep(8 * 12345, n, site, 3, 1234, p)
    frac = keep.mean()
    assert abs(frac - (1 - p)) <= 5 * np.sqrt(p * (1 - p) / n)


def test_sites_and_offsets_are_distinct_streams():
    a = dropout_lanes(0, 4096, 0, 0, 1234)
    assert not np.array_equal(a, dropout_lanes(0, 4096, 1, 0, 1234))
    assert not np.array_equal(a, dropout_lanes(0, 4096, 0, 1, 1234))
    assert not np.array_equal(a, dropout_lanes(0, 4096, 0, 0, 1235))
