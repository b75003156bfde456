"""Pins of the oracle's tables (RNG, fp16 rounding, Lloyd-Max codebook, Hadamard rotation,
bit packing) against published values, closed forms and library routines."""
import math

import numpy as np
import pytest
import scipy.linalg
from scipy import stats

import oracle as O
from conftest import read_golden


# ---------------------------------------------------------------- SplitMix64
def test_splitmix64_reference_outputs():
    for seed, idx, val in read_golden("splitmix64.txt"):
        seed, idx, val = int(seed), int(idx), int(val)
        assert O.splitmix64(seed, idx + 1)[idx] == val


def test_stream_seeds_differ_and_signs_are_balanced():
    a = O.random_signs(7, O.TAG_ROT_SIGNS, 4096)
    b = O.random_signs(7, O.TAG_OUT_SIGNS, 4096)
    assert set(np.unique(a)) == {-1.0, 1.0}
    assert not np.array_equal(a, b)
    # fair coin: |mean| within 4 standard errors
    assert abs(a.mean()) < 4.0 / math.sqrt(4096)
    # the sign is bit 63 of the draw
    z = O.splitmix64(O.stream_seed(7, O.TAG_ROT_SIGNS), 16)
    assert np.array_equal(a[:16], np.array([-1.0 if v >> 63 else 1.0 for v in z]))


def test_gaussian_projection_is_standard_normal_and_fp16_exact():
    s = O.gaussian_fp16_matrix(3, 128, 128)
    assert s.shape == (128, 128)
    assert np.array_equal(O.fp16_rn(s), s)
    v = s.ravel()
    n = v.size
    assert abs(v.mean()) < 4.0 / math.sqrt(n)
    assert abs(v.var() - 1.0) < 4.0 * math.sqrt(2.0 / n)
    # Kolmogorov-Smirnov against N(0,1) (scipy): fp16 rounding is far below KS resolution
    assert stats.kstest(v, "norm").pvalue > 1e-4
    # Box-Muller of the first pair, written from the definition
    a, b = O.splitmix64(O.stream_seed(3, O.TAG_QJL_GAUSS), 2)
    u1 = ((a >> 11) + 1) * 2.0 ** -53
    u2 = (b >> 11) * 2.0 ** -53
    z = math.sqrt(-2.0 * math.log(u1)) * math.cos(2.0 * math.pi * u2)
    assert s[0, 0] == float(np.float16(z))


# ---------------------------------------------------------------- fp16 rounding
@pytest.mark.parametrize("x,expected", [
    (1.0 + 2.0 ** -11, 1.0),                   # exact tie -> even mantissa
    (1.0 + 3 * 2.0 ** -11, 1.0 + 2.0 ** -9),   # tie -> even (rounds up)
    (1.0 + 2.0 ** -11 + 2.0 ** -30, 1.0 + 2.0 ** -10),
    (65504.0, 65504.0),                        # largest finite
    (65519.0, 65504.0),
    (65520.0, math.inf),                       # halfway to 2^16 rounds to infinity
    (2.0 ** -24, 2.0 ** -24),                  # smallest subnormal
    (2.0 ** -25, 0.0),                         # tie to even (zero)
    (3 * 2.0 ** -26, 2.0 ** -24),
    (-2.5, -2.5),
    (1.0 / 3.0, 0.333251953125),
])
def test_fp16_round_nearest_even(x, expected):
    assert O.fp16_rn(x) == expected


def test_fp16_bits_roundtrip():
    v = np.array([0.0, 1.0, -2.0, 65504.0, 2.0 ** -24])
    assert list(O.fp16_bits(v)) == [0x0000, 0x3C00, 0xC000, 0x7BFF, 0x0001]
    assert np.array_equal(O.fp16_from_bits(O.fp16_bits(v)), v)


def test_bf16_round_nearest_even():
    assert O.bf16_rn(1.0 + 2.0 ** -8) == 1.0          # tie -> even
    assert O.bf16_rn(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert O.bf16_rn(-3.0) == -3.0


# ---------------------------------------------------------------- Lloyd-Max codebook
def test_codebook_one_bit_closed_form():
    c, t = O.lloyd_max_gaussian(1)
    assert np.allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-14)
    assert t.tolist() == [0.0]
    assert abs(O.gaussian_distortion(c, t) - (1 - 2 / math.pi)) < 1e-14


def test_codebook_matches_max_1960_table():
    for row in read_golden("lloyd_max_gaussian.txt"):
        bits, mse, levels = int(row[0]), float(row[1]), [float(v) for v in row[2:]]
        c, t = O.lloyd_max_gaussian(bits)
        half = c[len(c) // 2:]
        assert np.allclose(half, levels, atol=1.5e-4), (bits, half)
        assert abs(O.gaussian_distortion(c, t) - mse) < 1e-5 + 1e-3 * mse


def test_codebook_structure():
    for bits in range(1, 5):
        c, t = O.lloyd_max_gaussian(bits)
        assert c.shape == (1 << bits,) and t.shape == ((1 << bits) - 1,)
        assert np.all(np.diff(c) > 0) and np.all(np.diff(t) > 0)
        assert np.array_equal(c, -c[::-1])                         # symmetric
        assert t[len(t) // 2] == 0.0                               # middle threshold
        assert np.allclose(t, 0.5 * (c[:-1] + c[1:]), atol=1e-15)  # midpoints
        # centroid condition: each level is the conditional mean of its cell (scipy)
        edges = np.concatenate([[-np.inf], t, [np.inf]])
        for k in range(len(c)):
            a, b = edges[k], edges[k + 1]
            mass = stats.norm.cdf(b) - stats.norm.cdf(a)
            mean = (stats.norm.pdf(a) - stats.norm.pdf(b)) / mass
            assert abs(mean - c[k]) < 1e-9


def test_codebook_distortion_matches_monte_carlo():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(2_000_000)
    for bits in range(1, 5):
        c, t = O.lloyd_max_gaussian(bits)
        cell = np.searchsorted(t, x)                 # brute-force nearest cell (scipy-free)
        mc = np.mean((x - c[cell]) ** 2)
        assert abs(mc - O.gaussian_distortion(c, t)) < 5e-3 * O.gaussian_distortion(c, t) + 2e-4


def test_codebook_mse_matches_table1_window():
    """validate_paper.py test_mse_codebook_table1: total MSE / Table-1 value in [0.85, 1.20]."""
    for bits, value in read_golden("table1_mse.txt"):
        bits, value = int(bits), float(value)
        c, t = O.lloyd_max_gaussian(bits)
        ratio = O.gaussian_distortion(c, t) / value
        assert 0.85 <= ratio <= 1.20, (bits, ratio)


# ---------------------------------------------------------------- rotation
@pytest.mark.parametrize("d", [8, 16, 128])
def test_hadamard_is_sylvester(d):
    assert np.array_equal(O.sylvester_hadamard(d), scipy.linalg.hadamard(d))


def test_rotation_orthonormal_and_sign_order():
    s = O.random_signs(11, O.TAG_ROT_SIGNS, 16)
    P = O.rotation_matrix(s)
    assert np.allclose(P.T @ P, np.eye(16), atol=1e-12)
    # signs are applied first: column j of Pi is s_j times column j of H / sqrt(d)
    H = scipy.linalg.hadamard(16)
    assert np.allclose(P, H * s[None, :] / 4.0, atol=1e-15)
    B = O.block_rotation_matrix(O.random_signs(2, O.TAG_NORM_SIGNS, 96), 32)
    assert np.allclose(B.T @ B, np.eye(96), atol=1e-12)
    assert np.allclose(B[:32, 32:], 0.0)


# ---------------------------------------------------------------- packing
def test_packing_matches_page_layouts():
    for row in read_golden("packing_layout.txt"):
        if row[0] == "ledger":
            continue
        width = int(row[0])
        arrow = row.index("->")
        vals = [int(v) for v in row[1:arrow]]
        expected = int(row[arrow + 1])
        packed = O.pack_bits(np.array([vals]), width)
        assert packed.tolist() == [[expected]], (row, packed)


@pytest.mark.parametrize("width", [1, 2, 4])
def test_pack_unpack_roundtrip(width):
    rng = np.random.default_rng(width)
    codes = rng.integers(0, 1 << width, size=(50, 128))
    packed = O.pack_bits(codes, width)
    assert packed.shape == (50, 128 * width // 8)
    assert np.array_equal(O.unpack_bits(packed, width, 128), codes)


def test_storage_ledger_52_bytes():
    led = next(r for r in read_golden("packing_layout.txt") if r[0] == "ledger")
    f = dict(zip(led[1::2], map(int, led[2::2])))
    q = O.build_quantizer(128, 3, "prod", 0)
    lay = O.key_layout(q)
    assert lay["idx_bytes"] == f["idx"]
    assert lay["sign_bytes"] == f["signs"]
    assert 2 * lay["n_norms"] == f["norms"]
    assert lay["bytes_per_key"] == f["total"]
    assert 128 * 2 == f["fp16"]


@pytest.mark.parametrize("mode,bits,nbytes", [
    ("mse", 1, 18), ("mse", 2, 34), ("mse", 3, 66), ("mse", 4, 66),
    ("prod", 2, 36), ("prod", 3, 52), ("prod", 4, 84),
    ("grouped", 1, 24), ("grouped", 2, 44), ("grouped", 3, 68),
])
def test_bytes_per_key_each_mode(mode, bits, nbytes):
    outl = np.arange(0, 128, 4)
    q = O.build_quantizer(128, bits, mode, 0, outl)
    assert O.key_layout(q)["bytes_per_key"] == nbytes


def test_compression_ratio_window():
    """validate_paper.py test_compression_ratio: H_kv=8, N=4096, 3-bit K + 2-bit V;
    ratio fp16 / packed must lie in (2, 8)."""
    q = O.build_quantizer(128, 3, "prod", 0)
    key_b = O.key_layout(q)["bytes_per_key"]
    val = O.quantize_values(np.zeros((1, 128)), 2, 32)
    val_b = val["q"].shape[1] + val["params"].size * 2
    n, h = 4096, 8
    ratio = (n * h * 128 * 2 * 2) / (n * h * (key_b + val_b))
    assert 2.0 < ratio < 8.0
    assert abs(ratio - 5.12) < 1e-12
