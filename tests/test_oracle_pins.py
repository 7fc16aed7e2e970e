"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here re-types the oracle's formulas to compare them with themselves:
each check is a library routine (numpy's float16 cast, ml_dtypes' E2M1 and
e8m0 casts, numpy float64 matmul, scikit-learn's Lloyd k-means), a closed
form written out by hand (tests/golden), an exhaustive/brute-force search,
an invariant, or a figure printed by the pages (soft band).
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def _rows(name):
    out = []
    for line in open(os.path.join(GOLD, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            out.append(line.split())
    return out


def _f(tok):
    return float.fromhex(tok) if "0x" in tok else float(tok)


# --------------------------------------------------------------------------
# IEEE binary16 conversion (library: numpy's float16 cast is RNE)
# --------------------------------------------------------------------------

def test_f16_from_f32_matches_numpy(orc):
    specials = [0.0, -0.0, 1.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e9, 2.0 ** -14, 2.0 ** -24,
                2.0 ** -25, 1.5 * 2.0 ** -25, 2.0 ** -26, 3.0 * 2.0 ** -26, 0.1, 1.0 / 3, -2.5e-7,
                1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2048.0 + 1.0, 2048.0 + 3.0, float("inf")]
    vals = np.array(specials + list(RNG.standard_normal(4000) * 10.0 ** RNG.uniform(-9, 5, 4000)), np.float32)
    # ties: values exactly halfway between fp16 neighbours
    ties = (np.arange(1, 2000, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -10)
    vals = np.concatenate([vals, ties, -ties])
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([orc.f32_to_f16_bits(float(v)) for v in vals], np.uint16)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, [(float(vals[i]), hex(ref[i]), hex(got[i])) for i in bad[:5]]


def test_f16_to_f32_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([orc.f16_bits_to_f32(int(b)) for b in bits], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(ref[~nan].view(np.uint32), got[~nan].view(np.uint32))


# --------------------------------------------------------------------------
# FP4 E2M1 + e8m0 (library: ml_dtypes float4_e2m1fn / float8_e8m0fnu)
# --------------------------------------------------------------------------

def test_e2m1_value_set_golden():
    rows = _rows("e2m1_values.txt")
    codes = np.array([int(r[0]) for r in rows], np.uint8)
    vals = np.array([_f(r[1]) for r in rows], np.float32)
    lib_vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    assert np.array_equal(lib_vals.view(np.uint32), vals.view(np.uint32))


def test_e2m1_rounding_matches_library_near_every_threshold(orc):
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    cuts = [(a + b) / 2 for a, b in zip(grid, grid[1:])] + grid + [7.0, 8.0, 100.0]
    vals = []
    for c in cuts:
        v = np.float32(c)
        lo, hi = v, v
        vals.append(v)
        for _ in range(4):  # 4 ulps on each side of every tie and grid point
            lo = np.nextafter(lo, np.float32(-1), dtype=np.float32)
            hi = np.nextafter(hi, np.float32(100), dtype=np.float32)
            vals += [lo, hi]
    vals += list(RNG.uniform(0, 9, 3000).astype(np.float32))
    vals = np.array(vals, np.float32)
    vals = np.concatenate([vals, -vals, np.array([0.0, -0.0, 1e-30, -1e-30], np.float32)])
    ref = vals.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    got = np.array([orc.e2m1_code(float(v)) for v in vals], np.uint8)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, [(float(vals[i]), int(ref[i]), int(got[i])) for i in bad[:5]]


def test_e8m0_closed_form_golden(orc):
    for amax_s, byte_s, *_ in _rows("e8m0_scale_cases.txt"):
        amax = float(np.float32(_f(amax_s)))
        assert orc.e8m0_byte(amax) == int(byte_s), amax_s


def test_e8m0_scale_is_library_e8m0_of_the_power_of_two(orc):
    # the byte is the e8m0 encoding (per ml_dtypes) of 2^(floor(log2 amax) - 2)
    amax = (np.abs(RNG.standard_normal(3000)) * 10.0 ** RNG.uniform(-30, 30, 3000)).astype(np.float32)
    for a in amax:
        b = orc.e8m0_byte(float(a))
        ref = np.array([2.0 ** (b - 127)], np.float32).astype(ml_dtypes.float8_e8m0fnu).view(np.uint8)[0]
        assert ref == b
        # the block maximum lands in the top binade of E2M1: amax / scale in [4, 8)
        r = float(a) / 2.0 ** (b - 127)
        assert 4.0 <= r < 8.0, (a, b)


def _fp4_lib_codes(W, scales):
    """E2M1 codes of W / scale computed by the ml_dtypes cast (library)."""
    s = np.repeat(np.ldexp(1.0, scales.astype(np.int32) - 127), 32, axis=1)
    v = (W.astype(np.float64) / s).astype(np.float32)  # exact: power-of-two scaling
    c = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def test_encode_fp4_matches_library_cast(orc):
    W = (RNG.standard_normal((64, 256)) * 0.02).astype(np.float32)
    W[:, [3, 100]] *= 20.0
    W[5, :32] = 0.0
    W[6, 32:64] = -1e-40  # subnormal block
    codes, scales, flags = orc.encode_fp4(W)
    assert flags == 0
    assert np.array_equal(codes, _fp4_lib_codes(W, scales))
    # element 2j in the low nibble: pin the packing with a one-element block
    Z = np.zeros((1, 32), np.float32)
    Z[0, 1] = 6.0
    c, s, _ = orc.encode_fp4(Z)
    assert s[0, 0] == 127 and c[0, 0] == 0x70 and not c[0, 1:].any()


def test_fp4_round_trip_exact_on_grid(orc):
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)
    N, K = 200, 128
    mags = grid[RNG.integers(0, 8, (N, K))]
    mags.reshape(N, -1, 32)[:, :, 0] = RNG.choice([4.0, 6.0], (N, K // 32))  # block max in [4, 6]
    sign = RNG.choice([-1.0, 1.0], (N, K)).astype(np.float32)
    e = RNG.integers(-20, 20, (N, K // 32))
    W = (sign * mags * np.repeat(np.ldexp(1.0, e), 32, axis=1)).astype(np.float32)
    codes, scales, _ = orc.encode_fp4(W)
    assert np.array_equal(scales.astype(np.int64) - 127, e)
    D = orc.dequant(orc.FMT_FP4, codes, scales, N, K)
    assert np.array_equal(D.view(np.uint32), W.view(np.uint32))  # bit-exact incl. signed zeros


def test_fp4_dequant_matches_library_decode_and_error_bound(orc):
    W = (RNG.standard_normal((128, 512)) * 0.02).astype(np.float32)
    W[:, 7] *= 20
    codes, scales, _ = orc.encode_fp4(W)
    D = orc.dequant(orc.FMT_FP4, codes, scales, *W.shape)
    c = np.empty(W.shape, np.uint8)
    c[:, 0::2], c[:, 1::2] = codes & 15, codes >> 4
    s = np.repeat(np.ldexp(1.0, scales.astype(np.int32) - 127), 32, axis=1)
    ref = (c.view(ml_dtypes.float4_e2m1fn).astype(np.float64) * s).astype(np.float32)
    assert np.array_equal(D.view(np.uint32), ref.view(np.uint32))
    # |w - dq| <= half the local grid gap (x scale); above 6 saturation bounds it by 2 x scale
    v = np.abs(W.astype(np.float64)) / s
    gap = np.where(v <= 2, 0.5, np.where(v <= 4, 1.0, 2.0))
    bound = np.where(v <= 6, gap / 2, 2.0) * s
    assert np.all(np.abs(W.astype(np.float64) - D) <= bound)


def test_fp4_negative_values_rounding_to_zero_keep_the_sign(orc):
    W = np.zeros((1, 32), np.float32)
    W[0, 0] = 4.0
    W[0, 1] = -0.1  # |v| = 0.1 < 0.25 -> magnitude 0 with the sign bit set
    codes, scales, _ = orc.encode_fp4(W)
    assert (codes[0, 0] >> 4) == 8
    D = orc.dequant(orc.FMT_FP4, codes, scales, 1, 32)
    assert math.copysign(1.0, float(D[0, 1])) == -1.0 and D[0, 1] == 0.0


def test_fp4_nonfinite_block_flags_and_zeroes(orc):
    W = (RNG.standard_normal((2, 64)) * 0.02).astype(np.float32)
    W[1, 40] = np.nan
    codes, scales, flags = orc.encode_fp4(W)
    assert flags & orc.FLAG_NONFINITE
    assert not codes[1, 16:32].any() and scales[1, 1] == 0
    assert np.array_equal(codes[:1], orc.encode_fp4(W[:1])[0])


# --------------------------------------------------------------------------
# symmetric int4 / int8 with MSE clip search
# --------------------------------------------------------------------------

def _unpack_int(codes, bits, K):
    if bits == 4:
        q = np.empty((codes.shape[0], K), np.int64)
        q[:, 0::2], q[:, 1::2] = (codes & 15).astype(np.int64) - 8, (codes >> 4).astype(np.int64) - 8
        return q
    return codes.astype(np.int64)


def _brute_q(w, s, qmax):
    """Exhaustive search of the integer in [-qmax, qmax] nearest to the float32
    quotient w / s, ties to the even integer."""
    if s == 0:
        return np.zeros_like(w, dtype=np.int64)
    quot = (w.astype(np.float32) / np.float32(s)).astype(np.float64)
    cand = np.arange(-qmax, qmax + 1)
    d = np.abs(quot[:, None] - cand[None, :])
    best = d.min(axis=1, keepdims=True)
    ok = d == best
    # among ties prefer the even integer
    pick = np.where(ok & (cand[None, :] % 2 == 0), 1, 0) + ok.astype(int)
    return cand[np.argmax(pick, axis=1)]


@pytest.mark.parametrize("bits", [4, 8])
def test_int_encode_brute_force(orc, bits):
    qmax = 7 if bits == 4 else 127
    clips = orc.INT4_CLIPS if bits == 4 else np.array([1.0, 0.9, 0.8, 0.7], np.float32)
    W = (RNG.standard_normal((24, 128)) * 0.02).astype(np.float32)
    W[:, 9] *= 20.0
    W[3, :32] = 0.0
    W[4, 32:64] = 1e-9  # tiny block: fp16 scale underflows toward subnormal / zero
    enc = orc.encode_int4 if bits == 4 else orc.encode_int8
    codes, scales, flags = enc(W, clips)
    assert flags == 0
    q = _unpack_int(codes, bits, W.shape[1])
    for n in range(W.shape[0]):
        for b in range(W.shape[1] // 32):
            w = W[n, b * 32:(b + 1) * 32]
            s = float(scales[n, b])
            assert np.array_equal(q[n, b * 32:(b + 1) * 32], _brute_q(w, s, qmax)), (n, b)
            amax = np.float32(np.max(np.abs(w)))
            errs, svals = [], []
            for a in clips:
                sc = np.float16(np.float32(np.float32(a) * amax) / np.float32(qmax))  # library RNE cast
                qq = _brute_q(w, float(sc), qmax)
                errs.append(float(np.sum((w.astype(np.float64) - qq * float(sc)) ** 2)))
                svals.append(sc)
            chosen = float(np.sum((w.astype(np.float64) - q[n, b * 32:(b + 1) * 32] * s) ** 2))
            assert chosen <= min(errs) * (1 + 1e-12) + 1e-300
            assert any(np.float16(s) == sv for sv in svals)
            # the first clip reaching the minimum is kept
            first = int(np.argmin(errs))
            if errs.count(errs[first]) == 1 or min(errs) == 0:
                assert np.float16(s) == svals[first] or min(errs) == 0


def test_int_exact_ties_round_to_even(orc):
    """Quotients exactly halfway between integers round to the even one: with
    amax = 7 and clip 1, the int4 scale is exactly 1."""
    w = np.array([7.0, 2.5, -2.5, 1.5, -1.5, 0.5, -0.5, 3.5, -3.5, 4.5, 5.5, 6.5] + [0.0] * 20, np.float32)
    codes, scales, _ = orc.encode_int4(w[None], np.array([1.0], np.float32))
    assert scales[0, 0] == 1.0
    q = _unpack_int(codes, 4, 32)[0]
    assert list(q[:12]) == [7, 2, -2, 2, -2, 0, 0, 4, -4, 4, 6, 6]
    w8 = np.zeros((1, 32), np.float32)
    w8[0, :6] = [127.0, 2.5, -2.5, 100.5, 101.5, -0.5]
    codes8, scales8, _ = orc.encode_int8(w8)
    assert scales8[0, 0] == 1.0
    assert list(codes8[0, :6]) == [127, 2, -2, 100, 102, 0]


def test_int_clip_tie_keeps_the_first(orc):
    """Two clips whose fp16 scales sit one ulp either side of the optimum
    c = amax / 7 give the same q and exactly the same SSE 49 u^2: the first
    clip in list order is kept."""
    c, u = 0.140625, 2.0 ** -13  # c on the fp16 grid, u its spacing there
    w = np.zeros((1, 32), np.float32)
    w[0, 0] = 7 * c
    clips = np.array([1 - u / c, 1 + u / c], np.float32)
    for order in (clips, clips[::-1].copy()):
        codes, scales, _ = orc.encode_int4(w, order)
        sc = np.float16(np.float32(np.float32(order[0]) * np.float32(7 * c)) / np.float32(7))
        assert scales[0, 0] == sc, (order, scales[0, 0], sc)
        assert _unpack_int(codes, 4, 32)[0, 0] == 7


def test_int_special_blocks(orc):
    W = np.zeros((3, 32), np.float32)
    W[0, 5] = 0.7  # single non-zero element, alpha = 1: q = qmax, s = fp16(0.7/7)
    W[2, :] = 65504.0 * 8  # scale 0.1*... overflow for int4 -> no finite clip
    codes, scales, flags = orc.encode_int4(W, np.array([1.0], np.float32))
    assert flags & orc.FLAG_SCALE_OVERFLOW
    q = _unpack_int(codes, 4, 32)
    assert q[0, 5] == 7 and np.count_nonzero(q[0]) == 1
    assert scales[0, 0] == np.float16(np.float32(0.7) / np.float32(7))
    assert not q[1].any() and scales[1, 0] == 0  # all-zero block
    assert not q[2].any() and scales[2, 0] == 0
    D = orc.dequant(orc.FMT_INT4, codes, scales, 3, 32)
    assert D[0, 5] == np.float32(7) * np.float32(scales[0, 0])


def test_int_dequant_matches_numpy(orc):
    W = (RNG.standard_normal((16, 256)) * 0.02).astype(np.float32)
    for bits, enc, fmt in ((4, orc.encode_int4, orc.FMT_INT4), (8, orc.encode_int8, orc.FMT_INT8)):
        codes, scales, _ = enc(W)
        D = orc.dequant(fmt, codes, scales, *W.shape)
        ref = (_unpack_int(codes, bits, 256).astype(np.float32)
               * np.repeat(scales.astype(np.float32), 32, axis=1))
        assert np.array_equal(D, ref)


def test_relerr_ordering_and_page_band(orc):
    """fp4 error > int4-clip error > int8 error on outlier-bearing weights
    (the pages' quality-gate ordering); the levels sit near the printed ones."""
    gold = {r[0]: float(r[1]) for r in _rows("weight_relerr.txt")}
    W = (RNG.standard_normal((512, 1024)) * 0.02).astype(np.float32)
    W[:, RNG.permutation(1024)[:8]] *= 20.0
    N, K = W.shape
    err = {}
    c, s, _ = orc.encode_fp4(W)
    err["fp4"] = orc.dequant(orc.FMT_FP4, c, s, N, K)
    c, s, _ = orc.encode_int4(W)
    err["int4_clip"] = orc.dequant(orc.FMT_INT4, c, s, N, K)
    c, s, _ = orc.encode_int8(W)
    err["int8"] = orc.dequant(orc.FMT_INT8, c, s, N, K)
    rel = {k: float(np.linalg.norm(W - v) / np.linalg.norm(W)) for k, v in err.items()}
    assert rel["fp4"] > rel["int4_clip"] > rel["int8"]
    W0 = (RNG.standard_normal((512, 1024)) * 0.02).astype(np.float32)  # no outliers
    for name, fmt, enc in (("int8", orc.FMT_INT8, orc.encode_int8), ("int4_clip", orc.FMT_INT4, orc.encode_int4),
                           ("fp4", orc.FMT_FP4, orc.encode_fp4)):
        out = enc(W0)
        r = float(np.linalg.norm(W0 - orc.dequant(fmt, out[0], out[1], 512, 1024)) / np.linalg.norm(W0))
        assert 0.75 * gold[name] < r < 1.35 * gold[name], (name, r)


# --------------------------------------------------------------------------
# int4km k-means (LUT values: parity unpinned; invariants pinned)
# --------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# int4 affine (asymmetric) per block 32
# ---------------------------------------------------------------------------

def _aff_unpack(c, a, K):
    nb = K // 32
    q = np.stack([c & 15, c >> 4], axis=-1).reshape(c.shape[0], K).astype(np.int64)
    s = a[:, : 2 * nb].copy().view(np.float16).astype(np.float32)
    zb = a[:, 2 * nb:]
    z = np.stack([zb & 15, zb >> 4], axis=-1).reshape(c.shape[0], -1)[:, :nb].astype(np.int64)
    return q, s, z


def test_int4aff_brute_force(orc):
    """Scale = numpy's fp16 cast of (hi - lo) / 15 over a range holding 0;
    zero point and codes are the nearest grid points (brute force over
    0..15, ties to even), for blocks of several shapes of distribution."""
    rng = np.random.default_rng(21)
    rows = [rng.standard_normal(64) * 0.02, np.abs(rng.standard_normal(64)) * 0.03 + 0.01,
            -np.abs(rng.standard_normal(64)) * 0.03 - 0.02, rng.uniform(-1, 3, 64), rng.standard_normal(64) * 5e-5]
    W = np.array(rows, np.float32)
    c, a, fl = orc.encode_int4aff(W)
    assert fl == 0
    q, s, z = _aff_unpack(c, a, 64)
    for n in range(W.shape[0]):
        for b in range(2):
            w = W[n, 32 * b: 32 * b + 32]
            lo, hi = min(w.min(), np.float32(0)), max(w.max(), np.float32(0))
            s_ref = np.float16(np.float32(hi - lo) / np.float32(15)).astype(np.float32)
            assert s[n, b] == s_ref
            grid = np.arange(16)
            zt = np.float32(-lo) / s_ref
            dz = np.abs(grid - zt)
            cand = grid[dz == dz.min()]
            assert z[n, b] == (cand[cand % 2 == 0][0] if len(cand) > 1 else cand[0])
            for i in range(32):
                t = np.float32(w[i] / s_ref) + z[n, b]
                d = np.abs(grid - t)
                cand = grid[d == d.min()]
                # rint ties to even on the unshifted quotient: even z keeps the parity
                want = cand[0] if len(cand) == 1 else cand[(cand - z[n, b]) % 2 == 0][0]
                assert q[n, 32 * b + i] == want, (n, b, i)


def test_int4aff_dequant_zero_exact_and_error_bound(orc):
    rng = np.random.default_rng(22)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    W[:, ::7] = 0.0
    W[3, :32] = 0.0  # an all-zero block
    c, a, fl = orc.encode_int4aff(W)
    D = orc.dequant(orc.FMT_INT4AFF, c, a, 64, 256)
    q, s, z = _aff_unpack(c, a, 256)
    assert (D[W == 0] == 0).all()
    assert (s[3, 0] == 0) and (z[3, 0] == 0) and (q[3, :32] == 0).all()
    srep = np.repeat(s, 32, axis=1)
    assert (np.abs(W - D) <= srep * (1 + 1e-6)).all()
    ref = (srep.astype(np.float64) * (q - np.repeat(z, 32, axis=1))).astype(np.float32)
    assert np.array_equal(D, ref)


def test_int4aff_special_blocks(orc):
    W = np.zeros((2, 64), np.float32)
    W[0, 5] = np.inf
    W[1, 40] = 70000.0  # (hi - lo) / 15 still fits fp16
    c, a, fl = orc.encode_int4aff(W)
    q, s, z = _aff_unpack(c, a, 64)
    assert fl == orc.FLAG_NONFINITE
    assert s[0, 0] == 0 and (q[0, :32] == 0).all()
    W2 = np.zeros((1, 32), np.float32)
    W2[0, 0] = 65504.0 * 20
    _, _, fl2 = orc.encode_int4aff(W2)
    assert fl2 == orc.FLAG_SCALE_OVERFLOW


def test_int4aff_gains_over_symmetric_page_band(orc):
    """The palettization page's quantization notes ("coreai-optimization
    (coreai-opt) reference", sec. "Quantization"): at int4 the asymmetric
    scheme gains 3-5 dB over symmetric on real weights.  Synthetic bounds:
    a zero-centred Gaussian gains less than that band, a one-sided
    distribution more."""
    rng = np.random.default_rng(23)
    def snr_gain(W):
        N, K = W.shape
        c, a, _ = orc.encode_int4aff(W)
        c2, s2, _ = orc.encode_int4(W, clips=np.array([1.0], np.float32))
        e = lambda D: ((W.astype(np.float64) - D) ** 2).sum()
        Da = orc.dequant(orc.FMT_INT4AFF, c, a, N, K)
        Ds = orc.dequant(orc.FMT_INT4, c2, s2, N, K)
        return 10 * np.log10(e(Ds) / e(Da))
    g_gauss = snr_gain((rng.standard_normal((256, 512)) * 0.02).astype(np.float32))
    g_skew = snr_gain((np.abs(rng.standard_normal((256, 512))) * 0.02 + 0.005).astype(np.float32))
    assert 0.5 < g_gauss < 3.0 < 5.0 < g_skew


def test_kmeans_signed_zero_order(orc):
    """Sorting puts -0 before +0 (a total order), so initial centres read from
    a run of signed zeros are fixed: 16 x -0 then 16 x +0 give centres 1..7 at
    -0 and 8..15 at +0; centre 0 takes every point (ties to the lower index)
    and its double sum starting at +0 stays +0."""
    W = np.array([[-0.0] * 16 + [0.0] * 16], np.float32)
    rng = np.random.default_rng(3)
    W = W[:, rng.permutation(32)]
    lut, idx, flags = orc.kmeans_int4km(W)
    assert flags == 0
    bits = lut.view(np.uint16)[0].tolist()
    assert bits == [0x0000] + [0x8000] * 7 + [0x0000] * 8
    assert (idx == 0).all()


def test_kmeans_exact_on_few_distinct_values(orc):
    """A row of <= 16 fp16-representable values, each occurring at least
    n/16 times, is a fixed point of Lloyd from the quantile start (every
    value is some starting centre: a run of >= n/16 equal sorted values holds
    a quantile position), so it reconstructs exactly."""
    N, K = 32, 256
    W = np.zeros((N, K), np.float32)
    for n in range(N):
        nd = int(RNG.integers(1, 17))
        vals = np.unique(np.float16(RNG.standard_normal(nd) * 0.05)).astype(np.float32)
        nd = len(vals)
        counts = np.full(nd, K // 16)
        counts += np.bincount(RNG.integers(0, nd, K - counts.sum()), minlength=nd)
        W[n] = RNG.permutation(np.repeat(vals, counts))
    lut, idx, flags = orc.kmeans_int4km(W)
    assert flags == 0
    D = orc.dequant(orc.FMT_INT4KM, idx, lut, N, K)
    assert np.array_equal(D, W)
    # rows with fewer than 16 values keep duplicate centres: an index must
    # name the lowest of equal nearest entries
    got = np.empty((N, K), np.int64)
    got[:, 0::2], got[:, 1::2] = idx & 15, idx >> 4
    d = np.abs(W.astype(np.float64)[:, :, None] - lut.astype(np.float64)[:, None, :])
    assert np.array_equal(got, np.argmin(d, axis=2))


def test_kmeans_sse_monotone_and_nearest_indices(orc):
    W = (RNG.standard_normal((64, 512)) * 0.02).astype(np.float32)
    W[:, 3] *= 20
    lut, idx, flags, sse = orc.kmeans_int4km(W, want_sse=True)
    assert flags == 0
    assert np.all(np.diff(sse, axis=1) <= 1e-18)
    L = lut.astype(np.float64)
    d = np.abs(W.astype(np.float64)[:, :, None] - L[:, None, :])
    nearest = np.argmin(d, axis=2)  # argmin returns the lowest index on ties
    got = np.empty_like(nearest)
    got[:, 0::2], got[:, 1::2] = idx & 15, idx >> 4
    assert np.array_equal(got, nearest)
    assert np.all(np.diff(L, axis=1) >= 0)  # centres stay ordered on these rows


def test_kmeans_matches_sklearn_lloyd(orc):
    """Same quantile start, 20 Lloyd steps: scikit-learn's KMeans (float64
    centres) lands within fp16 rounding of the oracle's LUT on almost every
    row; the oracle rounds centres to float each step, so rare rows may take a
    different tie path."""
    from sklearn.cluster import KMeans
    W = (RNG.standard_normal((40, 512)) * 0.02).astype(np.float32)
    lut, _, _ = orc.kmeans_int4km(W)
    agree = 0
    for n in range(W.shape[0]):
        s = np.sort(W[n])
        init = s[[((2 * k + 1) * 512) // 32 for k in range(16)]].astype(np.float64)[:, None]
        km = KMeans(16, init=init, n_init=1, max_iter=20, tol=0.0, algorithm="lloyd")
        km.fit(W[n].astype(np.float64)[:, None])
        ref = np.sort(km.cluster_centers_[:, 0]).astype(np.float16)
        if np.array_equal(ref, lut[n]):
            agree += 1
    assert agree >= 0.9 * W.shape[0], agree


def test_kmeans_quantile_start(orc):
    W = (RNG.standard_normal((8, 256)) * 0.02).astype(np.float32)
    lut, _, _ = orc.kmeans_int4km(W, iters=0)
    for n in range(8):
        s = np.sort(W[n])
        assert np.array_equal(lut[n], s[[((2 * k + 1) * 256) // 32 for k in range(16)]].astype(np.float16))


# --------------------------------------------------------------------------
# int8km: 256-entry LUT per group of 32 output rows
# --------------------------------------------------------------------------

def _km8_nearest(W, lut):
    """Brute-force nearest LUT entry of every weight (lowest index on ties),
    the LUT of row n being lut[n // 32]."""
    N, K = W.shape
    L = lut.astype(np.float64)[np.arange(N) // 32]  # [N, 256]
    d = np.abs(W.astype(np.float64)[:, :, None] - L[:, None, :])
    return np.argmin(d, axis=2)


def test_int8km_quantile_start_and_groups(orc):
    """iters = 0: each group's LUT is fp16 of its sorted values at the
    (k + 1/2)/256 quantiles; N = 70 makes groups of 32, 32 and a last one of 6
    rows; indices are the nearest entry of the row's own group."""
    N, K = 70, 96
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[32:64] *= 10.0  # a group on another scale: a mix-up of groups shows
    lut, idx, flags = orc.kmeans_int8km(W, iters=0)
    assert flags == 0 and lut.shape == (3, 256) and idx.shape == (N, K)
    for g, (r0, r1) in enumerate([(0, 32), (32, 64), (64, 70)]):
        s = np.sort(W[r0:r1].reshape(-1))
        n = s.size
        want = s[[((2 * k + 1) * n) // 512 for k in range(256)]].astype(np.float16)
        assert np.array_equal(lut[g], want), g
    assert np.array_equal(idx.astype(np.int64), _km8_nearest(W, lut))


def test_int8km_exact_on_few_distinct_values(orc):
    """A group of <= 256 fp16-representable values, each at least n/256 times,
    is a fixed point of Lloyd from the quantile start: exact reconstruction."""
    N, K = 64, 256
    W = np.zeros((N, K), np.float32)
    for g in range(2):
        nd = int(RNG.integers(100, 257))
        vals = np.unique(np.float16(RNG.standard_normal(nd) * 0.05)).astype(np.float32)
        nd = len(vals)
        n = 32 * K
        counts = np.full(nd, n // 256)
        counts += np.bincount(RNG.integers(0, nd, n - counts.sum()), minlength=nd)
        W[32 * g:32 * g + 32] = RNG.permutation(np.repeat(vals, counts)).reshape(32, K)
    lut, idx, flags = orc.kmeans_int8km(W)
    assert flags == 0
    D = orc.dequant(orc.FMT_INT8KM, idx, lut, N, K)
    assert np.array_equal(D, W)
    assert np.array_equal(idx.astype(np.int64), _km8_nearest(W, lut))


def test_int8km_sse_monotone_nearest_and_independent_groups(orc):
    N, K = 40, 128
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[:, 5] *= 20
    lut, idx, flags, sse = orc.kmeans_int8km(W, want_sse=True)
    assert flags == 0 and sse.shape == (2, 21)
    assert np.all(np.diff(sse, axis=1) <= 1e-18)
    assert np.array_equal(idx.astype(np.int64), _km8_nearest(W, lut))
    assert np.all(np.diff(lut.astype(np.float64), axis=1) >= 0)
    # a change in the second group leaves the first group's fit untouched
    W2 = W.copy()
    W2[35:] = (RNG.standard_normal((5, K)) * 0.5).astype(np.float32)
    lut2, idx2, _ = orc.kmeans_int8km(W2)
    assert np.array_equal(lut2[0], lut[0]) and np.array_equal(idx2[:32], idx[:32])
    assert not np.array_equal(lut2[1], lut[1])


def test_int8km_nonfinite_group(orc):
    W = (RNG.standard_normal((64, 64)) * 0.02).astype(np.float32)
    W[40, 7] = np.inf
    lut, idx, flags = orc.kmeans_int8km(W)
    assert flags & orc.FLAG_NONFINITE
    assert not lut[1].view(np.uint16).any() and not idx[32:].any()
    lut0, idx0, f0 = orc.kmeans_int8km(W[:32])
    assert f0 == 0 and np.array_equal(lut0[0], lut[0]) and np.array_equal(idx0, idx[:32])


def test_int8km_matches_sklearn_lloyd(orc):
    """Same quantile start, 20 Lloyd steps on one group: scikit-learn's
    KMeans (float64 centres) lands within fp16 rounding of most entries."""
    from sklearn.cluster import KMeans
    N, K = 32, 64
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    lut, _, _ = orc.kmeans_int8km(W)
    v = np.sort(W.reshape(-1))
    init = v[[((2 * k + 1) * v.size) // 512 for k in range(256)]].astype(np.float64)[:, None]
    km = KMeans(256, init=init, n_init=1, max_iter=20, tol=0.0, algorithm="lloyd")
    km.fit(W.reshape(-1).astype(np.float64)[:, None])
    ref = np.sort(km.cluster_centers_[:, 0]).astype(np.float16)
    assert np.mean(ref == lut[0]) >= 0.9


def test_int8km_error_below_int4km_page_band(orc):
    """The pages measure the 4-bit schemes' weight error at 3.6x int8km's on a
    real head.  On Gaussian weights int8km's relative error is below
    int4km's / 3.6 (measured ratio ~6).  (Heavy tails are another matter:
    20 Lloyd steps from the quantile start do not yet spread 256 centres
    over a group's far tail.)"""
    g = np.random.default_rng(11)
    W = (g.standard_normal((64, 512)) * 0.02).astype(np.float32)
    lut8, idx8, _ = orc.kmeans_int8km(W)
    lut4, idx4, _ = orc.kmeans_int4km(W)
    e8 = np.linalg.norm(orc.dequant(orc.FMT_INT8KM, idx8, lut8, 64, 512) - W) / np.linalg.norm(W)
    e4 = np.linalg.norm(orc.dequant(orc.FMT_INT4KM, idx4, lut4, 64, 512) - W) / np.linalg.norm(W)
    assert e8 * 3.6 < e4, (e8, e4)


# --------------------------------------------------------------------------
# mixed int4km + int8 outlier columns
# --------------------------------------------------------------------------

def _outlier_weights(N, K, cols, seed):
    g = np.random.default_rng(seed)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[:, cols] *= 20.0
    return W


def test_outlier_columns_brute_force_and_planted(orc):
    N, K = 24, 256
    g = np.random.default_rng(3)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[:, 17] = W[:, 200]  # equal column maxima: the lower index goes first
    W[5, 99] = np.nan     # a non-finite column counts as the most outlying
    for C in (0, 32, 64):
        got = orc.outlier_columns(W, C)
        m = np.abs(W.astype(np.float64)).max(axis=0)
        m = np.where(np.isnan(np.abs(W)).any(axis=0), np.inf, m)
        order = np.lexsort((np.arange(K), -m))  # largest maximum first, then lower index
        assert np.array_equal(got, np.sort(order[:C]).astype(np.int32)), C
    planted = np.sort(np.random.default_rng(4).choice(K, 32, replace=False))
    Wp = _outlier_weights(N, K, planted, 5)
    assert np.array_equal(orc.outlier_columns(Wp, 32), planted)


def test_int4km_o8_parts_and_special_cases(orc):
    """The main part is the int4km fit of the remaining columns in order, the
    outlier part the int8 encode of the outlier columns in order; C = 0 is
    plain int4km; the dequantized matrix puts each part back in its columns."""
    N, K, C = 40, 320, 64
    cols = np.sort(np.random.default_rng(6).choice(K, C, replace=False)).astype(np.int32)
    W = _outlier_weights(N, K, cols, 7)
    c, lut, idx, oc, osc, fl = orc.encode_int4km_o8(W, C)
    assert fl == 0 and np.array_equal(c, cols)
    main = np.setdiff1d(np.arange(K), cols)
    lut_m, idx_m, _ = orc.kmeans_int4km(W[:, main])
    assert np.array_equal(lut, lut_m) and np.array_equal(idx, idx_m)
    oc_r, osc_r, _ = orc.encode_int8(W[:, cols])
    assert np.array_equal(oc, oc_r) and np.array_equal(osc.view(np.uint16), osc_r.view(np.uint16))
    D = orc.dequant_int4km_o8(c, lut, idx, oc, osc, N, K)
    e = np.empty((N, K - C), np.int64)
    e[:, 0::2], e[:, 1::2] = idx & 15, idx >> 4
    assert np.array_equal(D[:, main], lut.astype(np.float32)[np.arange(N)[:, None], e])
    sc = np.repeat(osc.astype(np.float32), 32, axis=1)
    assert np.array_equal(D[:, cols], oc.astype(np.float32) * sc)
    # no outliers: plain int4km
    c0, lut0, idx0, _, _, _ = orc.encode_int4km_o8(W, 0)
    lut4, idx4, _ = orc.kmeans_int4km(W)
    assert len(c0) == 0 and np.array_equal(lut0, lut4) and np.array_equal(idx0, idx4)
    D0 = orc.dequant_int4km_o8(c0, lut0, idx0, np.zeros((N, 0), np.int8), np.zeros((N, 0), np.float16), N, K)
    assert np.array_equal(D0, orc.dequant(orc.FMT_INT4KM, idx4, lut4, N, K))


def test_int4km_o8_matvec_and_error(orc):
    """The matvec is x Wdq^T; on weights with 32 outlier columns (x20) the
    mixed format's weight error is far below plain int4km's."""
    N, K, C = 64, 512, 32
    cols = np.sort(np.random.default_rng(8).choice(K, C, replace=False)).astype(np.int32)
    W = _outlier_weights(N, K, cols, 9)
    c, lut, idx, oc, osc, _ = orc.encode_int4km_o8(W, C)
    D = orc.dequant_int4km_o8(c, lut, idx, oc, osc, N, K).astype(np.float64)
    x = RNG.standard_normal((3, K)).astype(np.float16)
    r = orc.matvec_int4km_o8(c, lut, idx, oc, osc, x, N, K)
    assert np.allclose(r, x.astype(np.float64) @ D.T, rtol=1e-12, atol=1e-15)
    lut4, idx4, _ = orc.kmeans_int4km(W)
    e_mixed = np.linalg.norm(D - W) / np.linalg.norm(W)
    e_km = np.linalg.norm(orc.dequant(orc.FMT_INT4KM, idx4, lut4, N, K) - W) / np.linalg.norm(W)
    assert e_mixed * 3 < e_km, (e_mixed, e_km)


# --------------------------------------------------------------------------
# matvec and gather
# --------------------------------------------------------------------------

def _encode_all(orc, W):
    N, K = W.shape
    out = {}
    c, s, _ = orc.encode_fp4(W)
    out[orc.FMT_FP4] = (c, s)
    c, s, _ = orc.encode_int4(W)
    out[orc.FMT_INT4] = (c, s)
    lut, idx, _ = orc.kmeans_int4km(W)
    out[orc.FMT_INT4KM] = (idx, lut)
    c, s, _ = orc.encode_int8(W)
    out[orc.FMT_INT8] = (c, s)
    c, a, _ = orc.encode_int4aff(W)
    out[orc.FMT_INT4AFF] = (c, a)
    lut8, idx8, _ = orc.kmeans_int8km(W)
    out[orc.FMT_INT8KM] = (idx8, lut8)
    return out


def test_matvec_one_hot_is_a_column_bit_exact(orc):
    N, K = 48, 192
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    for fmt, (c, a) in _encode_all(orc, W).items():
        D = orc.dequant(fmt, c, a, N, K)
        ks = [0, 1, 31, 32, 33, 100, K - 1]
        x = np.zeros((len(ks), K), np.float16)
        x[np.arange(len(ks)), ks] = 1.0
        r = orc.matvec(fmt, c, a, x, N, K)
        for i, k in enumerate(ks):
            assert np.array_equal(r[i], D[:, k].astype(np.float64)), (fmt, k)


def test_matvec_matches_numpy_and_integer_sums(orc):
    N, K = 64, 256
    W = (RNG.standard_normal((N, K)) * 0.02).astype(np.float32)
    x = RNG.standard_normal((3, K)).astype(np.float16)
    for fmt, (c, a) in _encode_all(orc, W).items():
        D = orc.dequant(fmt, c, a, N, K).astype(np.float64)
        r = orc.matvec(fmt, c, a, x, N, K)
        ref = x.astype(np.float64) @ D.T
        assert np.allclose(r, ref, rtol=1e-12, atol=1e-15)
        rows = np.array([N - 1, 0, 17])
        assert np.array_equal(orc.matvec(fmt, c, a, x, N, K, rows=rows), r[:, rows])
    # integer-valued weights (fp4 grid x 2^1), all-ones x: exact integer sums
    Wi = (RNG.integers(-3, 4, (N, K)) * 2).astype(np.float32)
    Wi[:, ::32] = 12.0
    c, s, _ = orc.encode_fp4(Wi)
    r = orc.matvec(orc.FMT_FP4, c, s, np.ones((1, K), np.float16), N, K)
    assert np.array_equal(r[0], Wi.sum(axis=1).astype(np.float64))


def test_gather_is_dense_matvec_per_slot(orc):
    E, N, K, B, topk = 6, 32, 128, 3, 2
    Ws = (RNG.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    enc = [_encode_all(orc, Ws[e]) for e in range(E)]
    ids = np.array([[0, 5], [2, 2], [7, -1]], np.int32)  # duplicate, then two bad ids
    for x_per_slot in (0, 1):
        x = RNG.standard_normal((B, topk, K) if x_per_slot else (B, K)).astype(np.float16)
        for fmt in enc[0]:
            cs = np.stack([enc[e][fmt][0] for e in range(E)])
            aus = np.stack([enc[e][fmt][1] for e in range(E)])
            y, flags = orc.gather_matvec(fmt, cs, aus, E, N, K, ids, x, x_per_slot)
            assert flags & orc.FLAG_BAD_EXPERT
            for b in range(B):
                for j in range(topk):
                    e = ids[b, j]
                    if 0 <= e < E:
                        xb = x[b, j] if x_per_slot else x[b]
                        ref = orc.matvec(fmt, cs[e], aus[e], xb[None], N, K)[0]
                        assert np.array_equal(y[b, j], ref)
                    else:
                        assert not y[b, j].any()


def test_fp4_cos_vs_fp16_page_band(orc):
    """cos(fp4 output, fp16-weight output) at the pages' three decode shapes."""
    for name, K, N, cos_ref in _rows("fp4_cos_vs_fp16.txt"):
        K, N, cos_ref = int(K), int(N), float(cos_ref)
        n = min(N, 4096)  # a row sample of the big head: cos is a per-output statistic
        W = (RNG.standard_normal((n, K)) * 0.02).astype(np.float32)
        x = RNG.standard_normal((1, K)).astype(np.float16)
        c, s, _ = orc.encode_fp4(W)
        y4 = orc.matvec(orc.FMT_FP4, c, s, x, n, K)[0]
        y16 = x.astype(np.float64) @ W.astype(np.float16).astype(np.float64).T
        cos = float(y4 @ y16[0] / (np.linalg.norm(y4) * np.linalg.norm(y16)))
        assert abs(cos - cos_ref) < 0.003, (name, cos)
