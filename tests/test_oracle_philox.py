"""Pins for the oracle's Philox4x32-10 against cuRAND's host-side generator.

cuRAND's host Philox4_32_10 generator (a library routine, run on the CPU)
emits, for seed s, 4-word blocks n = x * 65536 + z equal to
Philox4x32-10(counter = (x lo, x hi, z, 0), key = (s lo, s hi)); its offset
skips 32-bit outputs.  Matching it on many blocks pins the oracle's rounds,
multipliers, Weyl key schedule, key words and counter words 0-2.  Counter
word 3 (the batch index b in the SIP draw) is pinned on the GPU against
cuRAND's device function.
"""
import ctypes
import os

import numpy as np
import pytest

import oracle

_CURAND = None


def _curand():
    global _CURAND
    if _CURAND is None:
        for p in ("/usr/local/cuda/lib64/libcurand.so", "libcurand.so", "libcurand.so.10"):
            try:
                _CURAND = ctypes.CDLL(p)
                break
            except OSError:
                continue
    if _CURAND is None:
        pytest.skip("libcurand not found")
    return _CURAND


def curand_host_philox(seed: int, offset: int, n: int) -> np.ndarray:
    cr = _curand()
    g = ctypes.c_void_p()
    CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161
    assert cr.curandCreateGeneratorHost(ctypes.byref(g), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert cr.curandSetPseudoRandomGeneratorSeed(g, ctypes.c_ulonglong(seed)) == 0
        assert cr.curandSetGeneratorOffset(g, ctypes.c_ulonglong(offset)) == 0
        out = np.zeros(n, np.uint32)
        assert cr.curandGenerate(g, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(n)) == 0
    finally:
        cr.curandDestroyGenerator(g)
    return out


def _key(seed):
    return [seed & 0xFFFFFFFF, seed >> 32]


@pytest.mark.parametrize("seed", [0, 42, 0x123456789ABCDEF0, 0xFFFFFFFFFFFFFFFF])
def test_philox_matches_curand_counter_word2(seed):
    out = curand_host_philox(seed, 0, 4 * 300)
    for n in range(300):
        ref = out[4 * n: 4 * n + 4]
        got = oracle.philox4x32_10([0, 0, n, 0], _key(seed))
        assert (got == ref).all(), (seed, n)


@pytest.mark.parametrize("blk", [65536, 65536 * 7 + 3, 2**32 + 11, 2**48 + 5 * 65536 + 17,
                                 3 * 2**48 + 2**40 + 123, 2**61 - 1])
def test_philox_matches_curand_counter_words01(blk):
    seed = 0xFEDCBA9876543210
    out = curand_host_philox(seed, 4 * blk, 4)
    x, z = divmod(blk, 65536)
    got = oracle.philox4x32_10([x & 0xFFFFFFFF, x >> 32, z, 0], _key(seed))
    assert (got == out).all()


def test_philox_uniformity_chi_square():
    # 2^14 calls -> 2^16 words; 256 bins of the top byte; chi-square with 255 dof
    # has mean 255 and sd ~22.6: accept below mean + 6 sd.
    words = np.concatenate([oracle.philox4x32_10([j, 7, 0, 0], [42, 0]) for j in range(1 << 14)])
    hist = np.bincount(words >> 24, minlength=256)
    exp = len(words) / 256.0
    chi2 = float(((hist - exp) ** 2 / exp).sum())
    assert chi2 < 255 + 6 * 22.6
