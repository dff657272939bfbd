"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute the same
way: a library decoder (torch's float8_e4m3fn), closed forms worked by hand,
an error bound, brute force with an independent decoder, exact integer
arithmetic, and a negative control with the wrong scale layout.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from fp8_block_scaled_group_b200 import inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

E4M3_POS_FINITE = [c for c in range(0x00, 0x7F)]  # 0x7F is NaN


def torch_decode(codes):
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_encode(vals_f32):
    t = torch.from_numpy(np.ascontiguousarray(vals_f32, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


# ------------------------------------------------------------------ codec --

def test_decode_all_codes_match_library(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ours = np.array([oracle_mod.e4m3_decode(c) for c in codes])
    lib = torch_decode(codes)
    nan_ours = np.isnan(ours)
    assert np.array_equal(nan_ours, np.isnan(lib))
    assert list(np.nonzero(nan_ours)[0]) == [0x7F, 0xFF]
    assert np.array_equal(ours[~nan_ours], lib[~nan_ours])
    assert np.array_equal(np.signbit(ours[~nan_ours]), np.signbit(lib[~nan_ours]))


def test_decode_landmarks(oracle_mod):
    d = oracle_mod.e4m3_decode
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert d(0x01) == 2.0 ** -9
    assert d(0x07) == 7 * 2.0 ** -9
    assert d(0x08) == 2.0 ** -6
    assert d(0x38) == 1.0
    assert d(0x76) == 224.0 and d(0x77) == 240.0
    assert d(0x00) == 0.0 and np.signbit(d(0x80))


def test_every_e4m3_value_is_exactly_bf16(oracle_mod):
    # dispatch_proj.rs, `dequant_fp8_bf16_into` doc: every FP8 E4M3 value is
    # exactly representable in BF16.
    vals = np.array([oracle_mod.e4m3_decode(c) for c in range(256) if c not in (0x7F, 0xFF)],
                    dtype=np.float64)
    f32 = vals.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), vals)
    bf = inputs.f32_to_bf16_bits(f32)
    assert np.array_equal(inputs.bf16_bits_to_f32(bf).astype(np.float64), vals)


def test_reencode_roundtrip(oracle_mod):
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = np.float32(oracle_mod.e4m3_decode(c))
        assert oracle_mod.e4m3_encode(v) == c, hex(c)


def test_midpoints_round_to_even(oracle_mod):
    for c in range(0x00, 0x7E):
        lo, hi = oracle_mod.e4m3_decode(c), oracle_mod.e4m3_decode(c + 1)
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2  # midpoints are exact in fp32
        even = c if c % 2 == 0 else c + 1
        assert oracle_mod.e4m3_encode(mid) == even
        assert oracle_mod.e4m3_encode(-mid) == even | 0x80
        assert oracle_mod.e4m3_encode(np.nextafter(mid, np.float32(0))) == c
        assert oracle_mod.e4m3_encode(np.nextafter(mid, np.float32(1e9))) == c + 1


def test_encoder_matches_library_exhaustively_in_range(oracle_mod):
    """Every fp32 pattern in [2^-11, 448] (both signs): oracle == torch's RNE encoder.

    Below 2^-11 every value rounds to a signed zero; torch's encoder agrees
    with round-to-nearest-even there and inside the finite range, so only the
    saturation above 448 is checked separately.
    """
    lo = np.float32(2.0 ** -11).view(np.uint32)
    hi = np.float32(448.0).view(np.uint32)
    step = 1 << 24
    for start in range(int(lo), int(hi) + 1, step):
        stop = min(start + step, int(hi) + 1)
        pats = np.arange(start, stop, dtype=np.uint32)
        vals = pats.view(np.float32)
        ours = oracle_mod.e4m3_encode_array(vals)
        assert np.array_equal(ours, torch_encode(vals)), hex(start)
        if start == int(lo):
            neg = -vals[:1 << 16]
            assert np.array_equal(oracle_mod.e4m3_encode_array(neg), torch_encode(neg))


def test_encoder_tiny_and_saturation(oracle_mod):
    rng = np.random.default_rng(7)
    tiny = rng.uniform(0, 2.0 ** -11, 4096).astype(np.float32)
    assert np.all(oracle_mod.e4m3_encode_array(tiny) == 0x00)
    assert np.all(oracle_mod.e4m3_encode_array(-tiny) == 0x80)
    sub32 = np.array([1e-45, 1e-40, 1.17e-38], np.float32)  # fp32 subnormals and near
    assert np.all(oracle_mod.e4m3_encode_array(sub32) == 0x00)
    assert np.all(oracle_mod.e4m3_encode_array(-sub32) == 0x80)
    big = np.array([448.0, np.nextafter(np.float32(448), np.float32(1e9)), 463.99, 464.0,
                    479.9, 480.0, 1e6, 3.4e38], np.float32)
    assert np.all(oracle_mod.e4m3_encode_array(big) == 0x7E)
    assert np.all(oracle_mod.e4m3_encode_array(-big) == 0xFE)


# --------------------------------------------------- hand-worked groups --

def _one_group(vals):
    row = np.zeros((1, 128), np.float32)
    row[0, :len(vals)] = vals
    return inputs.f32_to_bf16_bits(row)


def test_group_all_zero(oracle_mod):
    q, s_r, s_k = oracle_mod.quant_act(_one_group([]))
    s = s_r[0, 0]
    # scale = 1e-10f / 448f: a fp32 number near 2.2321e-13, finite and positive
    assert np.isfinite(s) and 2.2320e-13 < s < 2.2322e-13
    assert s == np.float32(1e-10) / np.float32(448.0)
    assert np.all(q == 0x00)
    negz = np.full((1, 128), 0x8000, np.uint16)  # -0.0 everywhere
    q2, s2, _ = oracle_mod.quant_act(negz)
    assert np.all(q2 == 0x80) and s2[0, 0] == s


def test_group_single_outlier(oracle_mod):
    for v, j in [(-37.5, 5), (448.0, 0), (3.0, 127), (-1e-3, 64)]:
        row = np.zeros(128, np.float32)
        row[j] = v
        q, s_r, _ = oracle_mod.quant_act(inputs.f32_to_bf16_bits(row[None]))
        vb = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(np.float32([v])))[0]
        assert s_r[0, 0] == np.float32(abs(vb)) / np.float32(448.0)
        assert q[0, j] == (0xFE if v < 0 else 0x7E)
        assert np.all(np.delete(q[0], j) == 0x00)


def test_group_exact_scale_landmarks(oracle_mod):
    # amax = 56 = 448 * 2^-3  ->  scale 0.125 exactly; every x below is exact.
    vals = [56.0, -56.0, 28.0, 2.0 ** -12, -(2.0 ** -12), 2.0 ** -13, 3 * 2.0 ** -13, 1.0, 0.0]
    q, s_r, _ = oracle_mod.quant_act(_one_group(vals))
    assert s_r[0, 0] == 0.125
    # 56/0.125 = 448 -> 0x7E; -448 -> 0xFE; 224 -> 0x76; 2^-9 -> 0x01 (smallest subnormal);
    # 2^-10 is the midpoint of 0 and 2^-9 -> ties to even 0x00; 3*2^-10 -> midpoint of
    # 0x01 and 0x02 -> 0x02; 8.0 -> 0x50; 0 -> 0x00
    assert list(q[0, :9]) == [0x7E, 0xFE, 0x76, 0x01, 0x81, 0x00, 0x02, 0x50, 0x00]


def test_group_2v_v(oracle_mod):
    for v in [1.0, 0.375, 13.0]:
        q, s_r, _ = oracle_mod.quant_act(_one_group([2 * v, v]))
        assert s_r[0, 0] == np.float32(2 * v) / np.float32(448.0)
        assert q[0, 0] == 0x7E and q[0, 1] == 0x76  # 448 and 224


def test_group_saturation_never_nan(oracle_mod):
    """Find bf16 amax values whose fp32 quotient amax / (amax/448) exceeds 448:
    they must still encode to 448, never to NaN."""
    hs = np.arange(0x3F80, 0x4780, dtype=np.uint16)  # bf16 1.0 .. 65536
    a = inputs.bf16_bits_to_f32(hs)
    s = a / np.float32(448.0)
    t = a / s
    over = hs[t > np.float32(448.0)]
    assert over.size > 0
    for h in over[:32]:
        row = np.zeros((1, 128), np.uint16)
        row[0, 0] = h
        row[0, 1] = h | 0x8000
        q, _, _ = oracle_mod.quant_act(row)
        assert q[0, 0] == 0x7E and q[0, 1] == 0xFE
        assert not np.any((q & 0x7F) == 0x7F)


def test_negative_tiny_keeps_sign(oracle_mod):
    q, s_r, _ = oracle_mod.quant_act(_one_group([448.0, -(2.0 ** -11), 2.0 ** -11]))
    assert s_r[0, 0] == 1.0
    assert q[0, 1] == 0x80 and q[0, 2] == 0x00


def test_bf16_subnormal_inputs(oracle_mod):
    row = np.full((1, 128), 0x0001, np.uint16)  # smallest positive bf16 subnormal
    row[0, 1::2] = 0x8001
    q, s_r, _ = oracle_mod.quant_act(row)
    assert s_r[0, 0] == np.float32(1e-10) / np.float32(448.0)
    assert np.all(q[0, 0::2] == 0x00) and np.all(q[0, 1::2] == 0x80)


# ------------------------------------------ division, not reciprocal --

def _rn24(v: Fraction) -> Fraction:
    """The binary32 value nearest to a positive normal-range rational, ties to
    even, by exact integer arithmetic."""
    e = v.numerator.bit_length() - v.denominator.bit_length()
    if Fraction(2) ** e > v:
        e -= 1
    if Fraction(2) ** (e + 1) <= v:
        e += 1
    quantum = Fraction(2) ** (e - 23)
    return round(v / quantum) * quantum  # Fraction.__round__ rounds half to even


def _e4m3_nearest(t: Fraction) -> int:
    """Nearest finite E4M3 code to a rational (OCP E4M3FN grid, ties to the
    even mantissa, saturating at 448), by exhaustive comparison."""
    sign = 0x80 if t < 0 else 0
    a = abs(t)
    best = None
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        key = (abs(v - a), c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return sign | best[1]


def _bf16_value(bits: int) -> Fraction:
    return Fraction(float(np.array([bits << 16], np.uint32).view(np.float32)[0]))


def test_codes_follow_ieee_division_not_a_reciprocal_product(oracle_mod):
    """The quotient x / s is one IEEE fp32 division. Multiplying by the
    rounded reciprocal instead changes some codes; such (x, amax) pairs are
    searched for, and each code is decided with exact rational arithmetic."""
    rng = np.random.default_rng(0)
    xs_bits = np.arange(0, 0x7F80, dtype=np.uint32)
    xs = (xs_bits << 16).view(np.float32)
    witnesses = []
    for ab in rng.integers(0x3C00, 0x4700, 400):
        amax = np.float32((np.uint32(ab) << np.uint32(16)).view(np.float32))
        s = amax / np.float32(448.0)
        xv = xs[xs <= amax]
        by_div = torch_encode(xv / s)
        by_rcp = torch_encode(xv * (np.float32(1.0) / s))
        for i in np.nonzero(by_div != by_rcp)[0][:2]:
            witnesses.append((int(ab), int(xv[i].view(np.uint32) >> 16)))
        if len(witnesses) >= 6:
            break
    assert len(witnesses) >= 6
    for amax_bits, x_bits in witnesses:
        amax, x = _bf16_value(amax_bits), _bf16_value(x_bits)
        s = _rn24(amax / 448)
        want = _e4m3_nearest(_rn24(x / s))
        other = _e4m3_nearest(_rn24(x * _rn24(1 / s)))
        assert want != other
        row = np.zeros((1, 128), np.uint16)
        row[0, 0], row[0, 1] = amax_bits, x_bits
        q, s_r, _ = oracle_mod.quant_act(row)
        assert Fraction(float(s_r[0, 0])) == s
        assert q[0, 1] == want, (hex(amax_bits), hex(x_bits))


# ------------------------------------------------------- error bounds --

def _check_quant_error_bound(x_f32, q, scale_of):
    """|deq(q) * s - x| <= max(2^-4 |x|, 2^-10 s): RNE into 3 mantissa bits
    (relative half-ulp 2^-4) or, in the subnormal range, half of 2^-9 * s."""
    deq = torch_decode(q.ravel()).reshape(q.shape)
    s = scale_of
    err = np.abs(deq * s - x_f32.astype(np.float64))
    bound = np.maximum(2.0 ** -4 * np.abs(x_f32.astype(np.float64)), 2.0 ** -10 * s) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_activation_quant_error_bound_and_amax(oracle_mod):
    x = inputs.activations(17, 1024, seed=11)
    q, s_r, _ = oracle_mod.quant_act(x)
    xf = inputs.bf16_bits_to_f32(x)
    s_full = np.repeat(s_r.astype(np.float64), 128, axis=1)
    _check_quant_error_bound(xf, q, s_full)
    # the element that sets amax lands on +-448 in every group
    deq = torch_decode(q.ravel()).reshape(q.shape)
    gmax = np.abs(deq).reshape(17, 8, 128).max(axis=2)
    assert np.all(gmax == 448.0)


def test_weight_quant_blocks(oracle_mod):
    w = inputs.weights(256, 384, seed=5)
    wq, ws = oracle_mod.quant_weight(w)
    assert ws.shape == (2, 3)
    wf = inputs.bf16_bits_to_f32(w)
    s_full = np.repeat(np.repeat(ws.astype(np.float64), 128, axis=0), 128, axis=1)
    _check_quant_error_bound(wf, wq, s_full)
    deq = torch_decode(wq.ravel()).reshape(wq.shape)
    bmax = np.abs(deq).reshape(2, 128, 3, 128).max(axis=(1, 3))
    assert np.all(bmax == 448.0)
    # blocks are independent: changing one block leaves the others' codes alone
    w2 = w.copy()
    w2[:128, :128] = inputs.f32_to_bf16_bits(np.full((128, 128), 3.0, np.float32))
    wq2, ws2 = oracle_mod.quant_weight(w2)
    assert np.array_equal(wq2[128:], wq[128:]) and np.array_equal(wq2[:128, 128:], wq[:128, 128:])
    assert ws2[0, 0] == np.float32(3.0) / np.float32(448.0) and np.array_equal(ws2.ravel()[1:], ws.ravel()[1:])
    assert np.all(wq2[:128, :128] == 0x7E)


# ----------------------------------------------------------- layouts --

@pytest.mark.parametrize("m", [1, 15, 16, 17, 25])
def test_scale_layout_identity(oracle_mod, m):
    x = inputs.activations(m, 512, seed=3)
    q, s_r, s_k = oracle_mod.quant_act(x)
    mp = -(-m // 16) * 16
    assert s_k.shape == (4, mp)
    assert np.array_equal(s_k[:, :m].view(np.uint32), s_r.T.view(np.uint32))
    assert np.all(s_k[:, m:].view(np.uint32) == 0)
    assert oracle_mod.m_pad(m) == mp


# -------------------------------------------------------------- GEMM --

def _brute_force(q, s_r, wq, ws):
    """Dequantize with the library decoder, expand scales, matmul in float64."""
    a = torch_decode(q.ravel()).reshape(q.shape) * np.repeat(s_r.astype(np.float64), 128, axis=1)
    ws_full = np.repeat(np.repeat(ws.astype(np.float64), 128, axis=0), 128, axis=1)
    b = torch_decode(wq.ravel()).reshape(wq.shape) * ws_full
    return a @ b.T


@pytest.mark.parametrize("m,n,k", [(1, 128, 128), (5, 256, 256), (17, 128, 384), (16, 256, 256)])
def test_gemm_ref_vs_brute_force(oracle_mod, m, n, k):
    x = inputs.activations(m, k, seed=m * 7 + k)
    w = inputs.weights(n, k, seed=n + k)
    q, s_r, _ = oracle_mod.quant_act(x)
    wq, ws = oracle_mod.quant_weight(w)
    ref = oracle_mod.gemm_ref(q, s_r, wq, ws)
    bf = _brute_force(q, s_r, wq, ws)
    assert np.allclose(ref, bf, rtol=1e-12, atol=1e-12 * np.abs(bf).max())
    rows = np.array([m - 1, 0], np.int64)
    assert np.array_equal(oracle_mod.gemm_ref(q, s_r, wq, ws, rows=rows), ref[rows])
    assert np.array_equal(oracle_mod.gemm_ref(q, s_r, wq, ws, threads=3), ref)


def test_gemm_ref_integer_case(oracle_mod):
    """Unit scales and codes of small integers: the result is an exact integer matmul."""
    rng = np.random.default_rng(0)
    ints = np.array([-3, -2, -1, 0, 1, 2, 3, 4], np.int64)
    code_of = {int(v): oracle_mod.e4m3_encode(float(v)) for v in ints}
    ia = rng.choice(ints, size=(9, 256))
    ib = rng.choice(ints, size=(128, 256))
    qa = np.vectorize(code_of.get)(ia).astype(np.uint8)
    qb = np.vectorize(code_of.get)(ib).astype(np.uint8)
    ref = oracle_mod.gemm_ref(qa, np.ones((9, 2), np.float32), qb, np.ones((1, 2), np.float32))
    assert np.array_equal(ref, (ia @ ib.T).astype(np.float64))
    # scaling one group's activation scale by 2 doubles exactly that group's share
    s2 = np.ones((9, 2), np.float32)
    s2[:, 1] = 2.0
    ref2 = oracle_mod.gemm_ref(qa, s2, qb, np.ones((1, 2), np.float32))
    expect = ia[:, :128] @ ib[:, :128].T + 2 * (ia[:, 128:] @ ib[:, 128:].T)
    assert np.array_equal(ref2, expect.astype(np.float64))


def test_tolerance_accepts_bf16_rounding_and_rejects_wrong_layout(oracle_mod):
    """Negative control (dispatch_proj.rs, `cublas_fp8_proj_prequant` doc: the
    row-major scales read as K-major gave rel_rms 7.7e-2): the acceptance test
    passes a correctly rounded output and fails the wrong-layout reading."""
    m, n, k = 25, 256, 1024
    x = inputs.activations(m, k, seed=21)
    w = inputs.weights(n, k, seed=22)
    q, s_r, s_k = oracle_mod.quant_act(x)
    wq, ws = oracle_mod.quant_weight(w)
    ref = oracle_mod.gemm_ref(q, s_r, wq, ws)
    y = inputs.f32_to_bf16_bits(ref.astype(np.float32))
    bad, worst = oracle_mod.check_tolerance(y, ref)
    assert bad == 0 and worst < 0.5
    # the row-major buffer, zero-padded to the K-major extent, read as [K/128, ceil16(M)]
    g, mp = s_k.shape
    flat = np.zeros(g * mp, np.float32)
    flat[:m * g] = s_r.ravel()
    wrong_a = flat.reshape(g, mp)[:, :m].T.copy()
    ref_wrong = oracle_mod.gemm_ref(q, wrong_a, wq, ws)
    y_wrong = inputs.f32_to_bf16_bits(ref_wrong.astype(np.float32))
    bad_w, _ = oracle_mod.check_tolerance(y_wrong, ref)
    assert bad_w > 0
    rel_rms = np.sqrt(np.mean((ref_wrong - ref) ** 2) / np.mean(ref ** 2))
    assert rel_rms > 1e-2
    # a 2 % gain error is also rejected
    assert oracle_mod.check_tolerance(inputs.f32_to_bf16_bits((ref * 1.02).astype(np.float32)), ref)[0] > 0


def test_tolerance_formula_by_hand(oracle_mod):
    """|y - ref| <= 8e-3 |ref| + 1e-3 rms(ref), rms over every compared
    element. ref = [100, 0, 0, 0]: rms = 50, so the bounds are 0.85 and 0.05."""
    ref = np.array([100.0, 0.0, 0.0, 0.0])
    y = inputs.f32_to_bf16_bits(np.array([100.5, 0.046875, -0.046875, 0.0625], np.float32))
    bad, worst = oracle_mod.check_tolerance(y, ref)
    assert bad == 1 and worst == pytest.approx(0.0625 / 0.05)
    # mostly the relative term: ref [1000, 0] (rms 707.1, bound 8 + 0.71 = 8.71)
    ref = np.array([1000.0, 0.0])
    assert oracle_mod.check_tolerance(inputs.f32_to_bf16_bits(np.array([1008.0, 0.0], np.float32)), ref)[0] == 0
    assert oracle_mod.check_tolerance(inputs.f32_to_bf16_bits(np.array([1016.0, 0.0], np.float32)), ref)[0] == 1


def test_inputs_are_deterministic_and_shaped():
    a = inputs.activations(16, 512, seed=1001)
    b = inputs.activations(16, 512, seed=1001)
    assert a.dtype == np.uint16 and a.shape == (16, 512) and np.array_equal(a, b)
    xf = inputs.bf16_bits_to_f32(inputs.activations(64, 4096, seed=1))
    frac_big = np.mean(np.abs(xf) > 6.0)
    assert 0.005 < frac_big < 0.015  # ~1 % outliers at sigma 20, almost all beyond 6
    wf = inputs.bf16_bits_to_f32(inputs.weights(256, 1024, seed=2))
    assert abs(wf.std() - 0.02) < 1e-3
