"""Pins for the float64 oracle, each against something other than the oracle itself:
published values, library routines (scipy, torch), brute force on tiny inputs, closed
forms and invariants.  CPU only."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

from kv_cache_tiering_b200 import synth
from oracle import akv_oracle as ora
from oracle import lloyd_max as lm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# ----------------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------------


def test_bf16_decode_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x7F80, 0x3E80, 0x0001], dtype=np.uint16)
    got = ora.bf16_bits_to_f64(bits)
    want = [1.0, -2.0, 0.0, -0.0, math.inf, 0.25, 2.0 ** -133]
    assert got.tolist() == want


def _all_finite_f16():
    bits = np.arange(0, 0x7C00, dtype=np.uint16)  # +0 .. max finite
    return bits, bits.view(np.float16).astype(np.float64)


def _nearest_f16_bruteforce(x: float) -> int:
    """Round-to-nearest-even to binary16 by exhaustive search over all positive finite values."""
    bits, vals = _all_finite_f16()
    fx = Fraction(x)
    best, best_err = None, None
    for b, v in zip(bits.tolist(), vals.tolist()):
        err = abs(Fraction(v) - fx)
        if best_err is None or err < best_err or (err == best_err and b % 2 == 0):
            best, best_err = b, err
    return best


def test_f64_to_f16_is_single_rne_rounding():
    gen = np.random.default_rng(1)
    xs = list(gen.uniform(1e-3, 60000, 40))
    # exact ties and near-ties: midpoints between neighbouring binary16 values
    for base in (1.0, 0.12841797, 1024.0, 2.73242188):
        b16 = np.float16(base).view(np.uint16)
        lo = float(np.uint16(b16).view(np.float16))
        hi = float(np.uint16(b16 + 1).view(np.float16))
        mid = (lo + hi) / 2
        xs += [mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf)]
    for x in xs:
        assert int(ora.f64_to_f16_bits(x)) == _nearest_f16_bruteforce(float(x)), x


# ----------------------------------------------------------------------------------
# Hadamard rotation
# ----------------------------------------------------------------------------------


@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128])
def test_fwht_equals_scipy_hadamard(d):
    gen = np.random.default_rng(d)
    x = gen.integers(-1000, 1000, size=(5, d)).astype(np.float64)
    h = scipy.linalg.hadamard(d).astype(np.float64)  # Sylvester construction
    assert np.array_equal(ora.fwht(x), x @ h.T)


@pytest.mark.parametrize("d", [2, 8, 64, 128])
def test_fwht_orthogonality_and_self_inverse(d):
    eye = np.eye(d)
    h = ora.fwht(eye)  # rows are H e_i
    assert np.array_equal(h @ h.T, d * eye)
    gen = np.random.default_rng(7)
    x = gen.standard_normal((3, d))
    assert np.allclose(ora.fwht(ora.fwht(x)) / d, x, atol=1e-12)


def test_rotation_preserves_dot_products():
    gen = np.random.default_rng(3)
    q, k = gen.standard_normal((2, 128))
    qr = ora.fwht(q) / math.sqrt(128)
    kr = ora.fwht(k) / math.sqrt(128)
    assert abs(qr @ kr - q @ k) < 1e-12


# ----------------------------------------------------------------------------------
# scale
# ----------------------------------------------------------------------------------


def test_pairwise_sum_order_hand_computed():
    # squares [2^54, 1, 1, 1, 1, 1, 1, 1]: pairwise halving gives 2^54 + 4
    # ((2^54 + 1) -> 2^54, (1 + 1) = 2, 2^54 + 2 -> 2^54 (tie to even), then + 4).
    # A sequential sum gives 2^54 and the exact sum rounds to 2^54 + 8.
    x = np.array([2.0 ** 27] + [1.0] * 7)
    assert ora.pairwise_sum_of_squares(x) == 2.0 ** 54 + 4


def test_scale_equals_rounded_exact_norm():
    gen = np.random.default_rng(11)
    x_bits = synth.normal_bf16(gen, (64, 128))
    s_bits = ora.scale_f16_bits(ora.bf16_bits_to_f64(x_bits))
    for row, sb in zip(ora.bf16_bits_to_f64(x_bits), s_bits):
        norm = math.sqrt(math.fsum(v * v for v in row))
        assert int(sb) == _nearest_f16_bruteforce(norm)


def test_scale_special_cases():
    zero = np.zeros((1, 128), dtype=np.uint16)
    enc = ora.encode(zero)
    assert enc.scale_bits[0] == 0 and np.all(enc.codes == 7)
    big = _bf16(np.full((1, 128), 6000.0))  # norm ~ 67882 > 65504 -> binary16 inf
    enc = ora.encode(big)
    assert enc.overflow[0] and enc.scale_bits[0] == 0 and np.all(enc.codes == 7)
    bad = _bf16(np.r_[np.ones(127), np.nan][None, :])
    enc = ora.encode(bad)
    assert enc.nonfinite[0] and enc.scale_bits[0] == 0


# ----------------------------------------------------------------------------------
# centroid table
# ----------------------------------------------------------------------------------


def _max1960():
    levels, thresholds, dist = {}, {}, None
    with open(os.path.join(GOLDEN, "max1960_n16.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kind, idx, val = line.split()
            if kind == "level":
                levels[int(idx)] = float(val)
            elif kind == "threshold":
                thresholds[int(idx)] = float(val)
            else:
                dist = float(val)
    return levels, thresholds, dist


def test_centroids_match_max_1960_table():
    # The 1960 table was computed by hand-era numerics: its printed values agree with
    # the exact optimum to within one unit in the last printed place (0.3881 for
    # 0.388048...), so that is the tolerance.
    levels, thresholds, dist = _max1960()
    c = np.array(lm.lloyd_max_normal_f64())
    for i, v in levels.items():
        decimals = len(str(v).split(".")[1])
        assert abs(c[i] - v) <= 10 ** -decimals + 1e-12, (i, c[i], v)
        assert abs(c[15 - i] + v) <= 10 ** -decimals + 1e-12
    b = lm.boundaries(c)
    for i, v in thresholds.items():
        decimals = len(str(v).split(".")[1])
        assert abs(b[i - 1] - v) <= 10 ** -decimals + 1e-12, (i, b[i - 1], v)
    # the printed distortion 0.009497 is 0.04% below the exact optimum 0.0095010
    assert abs(lm.quantiser_mse(c) / dist - 1.0) < 1e-3


def test_quantiser_mse_equals_numerical_integration():
    from scipy.integrate import quad
    c = np.array(lm.lloyd_max_normal_f64())
    e = [-np.inf, *lm.boundaries(c).tolist(), np.inf]
    pdf = lambda x: math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    ref = sum(quad(lambda x, j=j: (x - c[j]) ** 2 * pdf(x), e[j], e[j + 1], epsabs=1e-15, epsrel=1e-13)[0]
              for j in range(16))
    assert abs(lm.quantiser_mse(c) - ref) < 1e-12


def test_centroid_fixed_point_and_f16_rounding():
    c = np.array(lm.lloyd_max_normal_f64())
    assert np.max(np.abs(lm.lloyd_step(c) - c)) < 1e-13
    assert np.all(np.diff(c) > 0) and np.array_equal(c, -c[::-1])
    bits = lm.centroids_f16_bits()
    for v, b in zip(c, bits):
        if v > 0:
            assert int(b) == _nearest_f16_bruteforce(float(v))
    assert np.array_equal(lm.centroids_f16(), -lm.centroids_f16()[::-1])


# ----------------------------------------------------------------------------------
# codes, packing, dequantisation
# ----------------------------------------------------------------------------------


def test_codes_equal_bruteforce_nearest_centroid():
    gen = np.random.default_rng(5)
    x_bits = synth.normal_bf16(gen, (200, 128))
    enc = ora.encode(x_bits)
    x = ora.bf16_bits_to_f64(x_bits)
    z = x @ scipy.linalg.hadamard(128).T.astype(np.float64)
    s = ora.f16_bits_to_f64(enc.scale_bits)
    c = lm.centroids_f16()
    u = z / s[:, None]
    nearest = np.argmin(np.abs(u[..., None] - c[None, None, :]), axis=-1)  # lowest index on ties
    assert np.array_equal(enc.codes, nearest.astype(np.uint8))


def test_codes_round_trip_a_centroid_vector():
    # Quantisation sees u = sqrt(d) * (rotated x) / ||x||, a vector of norm sqrt(d).
    # Take codes of a Gaussian draw, scale their centroids to norm sqrt(d) (a factor
    # within 8% of 1; every level is at least 12% away from its cell's edges), and build x with
    # H x = 3 u: every coordinate then sits at its centroid and must get its code back.
    gen = np.random.default_rng(9)
    c = lm.centroids_f16()
    for d in (64, 128):
        want = np.argmin(np.abs(gen.standard_normal(d)[:, None] - c[None, :]), axis=1)
        factor = math.sqrt(d) / np.linalg.norm(c[want])
        assert abs(factor - 1.0) < 0.08
        u = c[want] * factor
        x = 3.0 * scipy.linalg.hadamard(d).astype(np.float64) @ u / d
        enc = ora.encode(_bf16(x[None, :]))
        assert np.array_equal(enc.codes[0], want)


def test_pack_and_block_layout_by_hand():
    assert ora.pack_codes(np.array([1, 2, 3, 4, 15, 0])).tolist() == [0x21, 0x43, 0x0F]
    assert np.array_equal(ora.unpack_codes(np.array([0x21, 0x43, 0x0F])), [1, 2, 3, 4, 15, 0])
    d = 4
    codes = np.arange(17 * d).reshape(17, d) % 16
    scales = np.arange(1, 18, dtype=np.uint16) * 0x0101
    blocks = ora.pack_blocks(codes, scales)
    assert blocks.shape == (2, ora.block_bytes(d)) == (2, 64)
    # token 1 of block 0: codes 4,5,6,7 -> bytes 0x54, 0x76 at offset 1*(d/2)
    assert blocks[0, 2:4].tolist() == [0x54, 0x76]
    # scale of token 1 at 16*(d/2) + 2, little-endian
    assert blocks[0, 32 + 2:32 + 4].tolist() == [0x02, 0x02]
    # token 16 is the first row of block 1; the rest of block 1 is the zero-vector encoding
    assert blocks[1, 0:2].tolist() == [0x10 | 0x01 << 4 if False else (codes[16, 0] | codes[16, 1] << 4), codes[16, 2] | codes[16, 3] << 4]
    assert np.all(blocks[1, 2:32] == 0x77) and np.all(blocks[1, 34:] == 0)
    c2, s2 = ora.unpack_blocks(blocks, 17, d)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)


def test_value_block_layout_by_hand():
    # codes chosen so every (token, dim) is recognisable: code = (7 * t + 3 * dim) mod 16
    def codes_for(n, d):
        t = np.arange(n)[:, None]
        dim = np.arange(d)[None, :]
        return ((7 * t + 3 * dim) % 16).astype(np.uint8)
    # d = 64: pair row r at byte 64 r, units of 8 bytes, unit u at position u ^ w(r)
    d = 64
    c = codes_for(17, d)
    sc = (np.arange(17, dtype=np.uint16) + 1) * 0x0102
    vb = ora.pack_value_blocks(c, sc)
    assert vb.shape == (2, 544)
    # tokens 0, 1 dim 0: pair row 0, w = 0 -> byte 0
    assert vb[0, 0] == c[0, 0] | c[1, 0] << 4 == 0x70
    # tokens 4, 5 dim 0: pair row 2, w = 4 -> unit 0 at position 4 -> byte 128 + 32 = 160
    assert vb[0, 160] == c[4, 0] | c[5, 0] << 4 == 0x3C
    # tokens 6, 7 dim 9: pair row 3, w = 4 -> unit 1 at position 5 -> byte 192 + 40 + 1 = 233
    assert vb[0, 233] == c[6, 9] | c[7, 9] << 4 == 0xC5
    # tokens 2, 3 dim 9: pair row 1, w = 0 -> byte 64 + 9 = 73
    assert vb[0, 73] == c[2, 9] | c[3, 9] << 4 == 0x09
    # scales as for keys: token 5 at 16 * 32 + 10, little-endian
    assert vb[0, 522:524].tolist() == [0x0C, 0x06]
    # token 16 heads block 1 (paired with a padding token of code 7), the rest is padding
    assert vb[1, 0] == c[16, 0] | 7 << 4
    assert np.all(vb[1, 64:512] == 0x77) and np.all(vb[1, 514:] == 0)
    c2, s2 = ora.unpack_value_blocks(vb, 17, d)
    assert np.array_equal(c2, c) and np.array_equal(s2, sc)
    # d = 128: units of 16 bytes, w(r) = 2 (r mod 4)
    d = 128
    c = codes_for(16, d)
    vb = ora.pack_value_blocks(c, np.zeros(16, np.uint16))
    # tokens 2, 3 dim 17: pair row 1, w = 2 -> unit 1 at position 3 -> byte 128 + 48 + 1 = 177
    assert vb[0, 177] == c[2, 17] | c[3, 17] << 4 == 0x81
    # tokens 14, 15 dim 127: pair row 7, w = 6 -> unit 7 at position 1 -> byte 896 + 16 + 15 = 927
    assert vb[0, 927] == c[14, 127] | c[15, 127] << 4 == 0x6F
    c2, _ = ora.unpack_value_blocks(vb, 16, d)
    assert np.array_equal(c2, c)


def test_dequantize_reproduces_table():
    # d = 64 and s = 8 = sqrt(64): y_i = s * c[code_i] / sqrt(d) = c[code_i] exactly
    codes = np.tile(np.arange(16, dtype=np.uint8), 4)[None, :]
    s = ora.f64_to_f16_bits(np.array([8.0]))
    y = ora.dequantize_rotated(codes, s)
    assert np.array_equal(y[0], lm.centroids_f16()[codes[0]])
    x = ora.dequantize(codes, s)
    assert np.allclose(scipy.linalg.hadamard(64) @ x[0] / 8.0, y[0], atol=1e-13)


def test_round_trip_mse_matches_quantiser_distortion():
    gen = np.random.default_rng(21)
    x_bits = synth.normal_bf16(gen, (4000, 128))
    enc = ora.encode(x_bits)
    x = ora.bf16_bits_to_f64(x_bits)
    xh = ora.dequantize(enc.codes, enc.scale_bits)
    rel = np.sum((x - xh) ** 2, axis=1) / np.sum(x * x, axis=1)
    assert abs(np.mean(rel) / 0.009497 - 1.0) < 0.10


# ----------------------------------------------------------------------------------
# attention, splits, merge
# ----------------------------------------------------------------------------------


def _attend_fsum(q, k, v, scale):
    s = [scale * math.fsum(a * b for a, b in zip(q, kt)) for kt in k]
    m = max(s)
    w = [math.exp(x - m) for x in s]
    ell = math.fsum(w)
    o = [math.fsum(wt * vt[i] for wt, vt in zip(w, v)) / ell for i in range(len(v[0]))]
    return np.array(o), m + math.log(ell)


def test_attend_bruteforce_tiny():
    gen = np.random.default_rng(2)
    for t in (1, 2, 5, 8):
        q, k, v = gen.standard_normal(6), gen.standard_normal((t, 6)), gen.standard_normal((t, 6))
        o, lse = ora.attend(q, k, v, 0.7)
        o2, lse2 = _attend_fsum(q, k, v, 0.7)
        assert np.allclose(o, o2, atol=1e-14) and abs(lse - lse2) < 1e-14


def test_attend_matches_torch_sdpa_gqa_f64():
    gen = np.random.default_rng(4)
    hq, hkv, t, d = 8, 2, 37, 16
    q = gen.standard_normal((hq, d))
    k = gen.standard_normal((hkv, t, d))
    v = gen.standard_normal((hkv, t, d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, :, None, :], torch.tensor(k)[None], torch.tensor(v)[None],
        scale=0.3, enable_gqa=True)[0, :, 0, :].numpy()
    for h in range(hq):
        o, _ = ora.attend(q[h], k[ora.gqa_kv_head(h, hq, hkv)], v[ora.gqa_kv_head(h, hq, hkv)], 0.3)
        assert np.allclose(o, ref[h], atol=1e-13)


def test_attend_closed_forms():
    gen = np.random.default_rng(6)
    q, k, v = gen.standard_normal(8), gen.standard_normal((1, 8)), gen.standard_normal((1, 8))
    o, lse = ora.attend(q, k, v, 0.5)
    assert np.array_equal(o, v[0]) and lse == 0.5 * float(k[0] @ q)
    kk = np.repeat(k, 5, axis=0)
    vv = gen.standard_normal((5, 8))
    o, lse = ora.attend(q, kk, vv, 0.5)
    assert np.allclose(o, vv.mean(axis=0), atol=1e-14)
    assert abs(lse - (0.5 * float(k[0] @ q) + math.log(5))) < 1e-13
    o0, l0 = ora.attend(np.zeros(8), np.zeros((0, 8)), np.zeros((0, 8)), 1.0)
    assert np.all(o0 == 0) and l0 == -math.inf


def test_split_ranges():
    assert ora.split_ranges(0, 64) == []
    assert ora.split_ranges(256, 64) == [(0, 64), (64, 128), (128, 192), (192, 256)]
    assert ora.split_ranges(130, 64) == [(0, 64), (64, 128), (128, 130)]


def test_merge_any_partition_equals_unsplit():
    gen = np.random.default_rng(8)
    q, k, v = gen.standard_normal(16), gen.standard_normal((50, 16)) * 2, gen.standard_normal((50, 16))
    o_ref, l_ref = ora.attend(q, k, v, 0.4)
    for trial in range(20):
        cuts = np.sort(gen.choice(np.arange(1, 50), size=gen.integers(0, 10), replace=False))
        edges = [0, *cuts.tolist(), 50]
        parts = [ora.attend(q, k[a:b], v[a:b], 0.4) for a, b in zip(edges[:-1], edges[1:])]
        parts.append(ora.attend(q, k[:0], v[:0], 0.4))  # an empty split
        order = gen.permutation(len(parts))  # the merge is commutative
        o, l = ora.merge_lse(np.stack([parts[i][0] for i in order]), np.array([parts[i][1] for i in order]))
        assert np.allclose(o, o_ref, atol=1e-12) and abs(l - l_ref) < 1e-12
    o, l = ora.merge_lse(np.zeros((3, 16)), np.full(3, -np.inf))
    assert np.all(o == 0) and l == -math.inf
    o, l = ora.merge_lse(np.zeros((0, 16)), np.zeros(0))
    assert np.all(o == 0) and l == -math.inf


def test_rotated_domain_attention_equals_dequantised_attention():
    """The identity the compact tier relies on: q . x_hat = (H q / sqrt d) . y."""
    gen = np.random.default_rng(12)
    d, t = 128, 40
    x_bits = synth.normal_bf16(gen, (t, d))
    enc = ora.encode(x_bits)
    q = gen.standard_normal(d)
    xh = ora.dequantize(enc.codes, enc.scale_bits)
    y = ora.dequantize_rotated(enc.codes, enc.scale_bits)
    qr = ora.fwht(q) / math.sqrt(d)
    assert np.allclose(xh @ q, y @ qr, atol=1e-12)
    v_bits = synth.normal_bf16(gen, (t, d))
    encv = ora.encode(v_bits)
    vh = ora.dequantize(encv.codes, encv.scale_bits)
    vy = ora.dequantize_rotated(encv.codes, encv.scale_bits)
    o, lse = ora.attend(q, xh, vh, 0.1)
    o_rot, lse_rot = ora.attend(qr, y, vy, 0.1)
    assert np.allclose(ora.fwht(o_rot) / math.sqrt(d), o, atol=1e-12) and abs(lse - lse_rot) < 1e-12


def test_decode_sequence_merge_equals_direct():
    gen = np.random.default_rng(13)
    hq, hkv, d = 8, 2, 32
    q = gen.standard_normal((hq, d))
    tiers = [(gen.standard_normal((hkv, 70, d)), gen.standard_normal((hkv, 70, d))),
             (gen.standard_normal((hkv, 33, d)), gen.standard_normal((hkv, 33, d)))]
    partials, (mo, ml), (do, dl) = ora.decode_sequence(q, tiers, 0.2, 16)
    assert [p[0].shape[0] for p in partials] == [5, 3]
    assert np.allclose(mo, do, atol=1e-12) and np.allclose(ml, dl, atol=1e-12)


def test_rotation_signs_by_hand_and_by_property():
    # d = 2: H = [[1, 1], [1, -1]]; bit 1 set negates coordinate 1 before the transform
    assert ora.rotate(np.array([3.0, 5.0]), 0b10).tolist() == [-2.0, 8.0]
    assert ora.rotate(np.array([3.0, 5.0]), 0b01).tolist() == [2.0, -8.0]
    assert ora.rotate(np.array([3.0, 5.0]), 0).tolist() == [8.0, -2.0]
    d = 128
    gen = np.random.default_rng(5)
    bits = int(gen.integers(0, 2**62)) | (int(gen.integers(0, 2**62)) << 64)
    x = _bf16(gen.standard_normal((6, d)))
    # encoding with signs = encoding the sign-flipped input (bf16 sign flips are exact)
    flip = np.array([(bits >> i) & 1 for i in range(d)], dtype=np.uint16) << 15
    enc_s = ora.encode(x, bits)
    enc_f = ora.encode(x ^ flip)
    assert np.array_equal(enc_s.codes, enc_f.codes) and np.array_equal(enc_s.scale_bits, enc_f.scale_bits)
    # (H S) (H S)^T = d I, so rotated queries keep dot products
    M = np.stack([ora.rotate(e, bits) for e in np.eye(d)])
    assert np.allclose(M @ M.T, d * np.eye(d), atol=0, rtol=0)
    # the inverse applies the signs after the transform: the round trip stays within the
    # quantiser's error, while the wrong order would not
    xf = ora.bf16_bits_to_f64(x)
    xh = ora.dequantize(enc_s.codes, enc_s.scale_bits, bits)
    rel = np.sum((xh - xf) ** 2, axis=1) / np.sum(xf ** 2, axis=1)
    assert np.all(rel < 0.02)
    wrong = ora.fwht(ora.sign_vector(bits, d) * ora.dequantize_rotated(enc_s.codes, enc_s.scale_bits)) / np.sqrt(d)
    assert np.all(np.sum((wrong - xf) ** 2, axis=1) / np.sum(xf ** 2, axis=1) > 0.5)
    # no bits: the plain transform
    assert np.array_equal(ora.encode(x, 0).codes, ora.encode(x).codes)
