"""Pins for the oracle's primitives: Philox4x32-10, the E4M3 codec and the
query quantisation.  Each is checked against something other than the oracle
itself: a library implementation (cuRAND's host generator, torch's float8
conversion), a closed form, or brute force."""
import ctypes
import glob
import math
import os

import numpy as np
import pytest
import torch


def _curand():
    cands = glob.glob("/usr/local/cuda/lib64/libcurand.so*")
    import site
    for sp in site.getsitepackages():
        cands += glob.glob(os.path.join(sp, "nvidia", "curand", "lib", "libcurand.so*"))
    for c in cands:
        try:
            return ctypes.CDLL(c)
        except OSError:
            continue
    pytest.skip("libcurand not found")


def _curand_host_philox(seed: int, n_blocks: int) -> np.ndarray:
    """cuRAND's host-side PHILOX4_32_10 generator (runs on the CPU)."""
    lib = _curand()
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0  # CURAND_RNG_PSEUDO_PHILOX4_32_10
    assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
    out = np.zeros(4 * n_blocks, np.uint32)
    assert lib.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(out.size)) == 0
    lib.curandDestroyGenerator(gen)
    return out.reshape(n_blocks, 4)


@pytest.mark.parametrize("seed", [0, 1, 0x0123456789ABCDEF, 2**64 - 1, 977])
def test_philox_matches_curand_host_generator(oracle_lib, seed):
    # cuRAND's host Philox emits, for its first blocks, Philox4x32-10 of the
    # counter (0, 0, i, 0) under the key (seed low word, seed high word).
    ref = _curand_host_philox(seed, 300)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for i in list(range(0, 300, 7)) + [299]:
        got = oracle_lib.philox4x32_10([0, 0, i, 0], key)
        assert list(got) == list(ref[i]), (seed, i)


def test_explore_key_is_word_j_mod_4_of_counter_j_div_4_req_layer_step(oracle_lib):
    seed = 0xDEADBEEF12345678
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for j in (0, 5, 6, 7, 8, 4099):
        got = oracle_lib.explore_key(seed, j, 7, 3, (1 << 32) + 9)
        ref = oracle_lib.philox4x32_10([j // 4, 7, 3, 9], key)[j % 4]
        assert got == ref, j


def test_explore_keys_uniform_chi_square(oracle_lib):
    # Keys over blocks x steps: the top 6 bits must look uniform.
    keys = np.array([oracle_lib.explore_key(2, j, 3, 0, t) for j in range(512) for t in range(64)],
                    np.uint64)
    counts = np.bincount((keys >> 26).astype(np.int64), minlength=64)
    expected = keys.size / 64
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    # 63 degrees of freedom: mean 63, sd ~11.2; 140 is far in the tail.
    assert chi2 < 140, chi2


def test_e4m3_decode_all_codes_vs_torch(oracle_lib):
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle_lib.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c] and math.copysign(1, got) == math.copysign(1, ref[c]), c


def test_e4m3_encode_vs_torch_rne(oracle_lib):
    vals = sorted({oracle_lib.e4m3_decode(c) for c in range(0x7F)})
    xs = [0.0, -0.0, 1e-30, -1e-30]
    for a, b in zip(vals[:-1], vals[1:]):
        mid = 0.5 * (a + b)                     # exact tie: must go to the even code
        xs += [a, b, mid, np.nextafter(mid, 0.0), np.nextafter(mid, 1e9)]
    xs += list(np.random.default_rng(0).uniform(-460, 460, 4000))
    xs = np.array(xs, np.float64)
    xs = np.concatenate([xs, -xs])
    xs = xs[np.abs(xs) < 464.0]                 # torch overflows to NaN beyond the last tie
    # torch converts from fp32; keep inputs exactly representable in fp32.
    xs = xs[xs.astype(np.float32).astype(np.float64) == xs]
    ref = torch.from_numpy(xs.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_lib.e4m3_encode(x) for x in xs], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(xs[i], got[i], ref[i]) for i in bad[:5]]


def test_e4m3_encode_saturates(oracle_lib):
    for x in [448.0, 463.9, 464.0, 480.0, 1e6, float("inf")]:
        assert oracle_lib.e4m3_encode(x) == 0x7E
        assert oracle_lib.e4m3_encode(-x) == 0xFE
    assert oracle_lib.e4m3_encode(float("nan")) & 0x7F == 0x7F


def test_q_exponent_closed_form(oracle_lib):
    rng = np.random.default_rng(1)
    amaxes = list(np.exp(rng.uniform(-40, 40, 2000))) + [448.0, 448.0 * 2 ** 5, 448.0 * 2 ** -7,
                                                        np.nextafter(448.0, 1e9), 1.0, 1.75, 1.7500001]
    for a in amaxes:
        e = oracle_lib.q_exponent(a)
        # smallest e with a <= 448 * 2^e
        assert a <= 448.0 * 2.0 ** e and a > 448.0 * 2.0 ** (e - 1), (a, e)
        # agrees with ceil(log2(a / 448)) away from exact powers of two
        f = math.log2(a / 448.0)
        if abs(f - round(f)) > 1e-9:
            assert e == math.ceil(f)
    assert oracle_lib.q_exponent(0.0) == 0


def test_quantize_q_vs_torch_and_error_bound(oracle_lib):
    rng = np.random.default_rng(2)
    rows, H, d = 3, 5, 64
    q = rng.standard_normal((rows, H, d)) * np.exp(rng.uniform(-6, 6, (rows, H, 1)))
    q = torch.from_numpy(q).to(torch.bfloat16).double().numpy()   # bf16-valued input
    q[1, 2] = 0.0                                                  # all-zero head: e = 0
    w = rng.uniform(0, 1, (rows, H)).astype(np.float32)
    q8, wq, e = oracle_lib.quantize_q(q, w)
    assert e[1, 2] == 0 and np.all(q8[1, 2] == 0)
    scaled = q * np.ldexp(1.0, -e)[..., None]
    ref = torch.from_numpy(scaled.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q8, ref)
    assert np.array_equal(wq, (w.astype(np.float64) * np.ldexp(1.0, e)).astype(np.float32))
    deq = np.vectorize(oracle_lib.e4m3_decode)(q8) * np.ldexp(1.0, e)[..., None]
    # RNE error of E4M3 is at most half an ulp: 2^-4 relative for normals,
    # 2^-10 * 2^e absolute in the subnormal range.
    bound = np.maximum(np.abs(q) * 2.0 ** -4, np.ldexp(1.0, e - 10)[..., None])
    assert np.all(np.abs(deq - q) <= bound)
    # The scale is tight: each nonzero head's largest code is at least 224.
    amax_codes = np.abs(np.vectorize(oracle_lib.e4m3_decode)(q8)).max(-1)
    assert np.all((amax_codes >= 224.0) | (np.abs(q).max(-1) == 0))
