"""Pins of the oracle's NVFP4 and FP8-dequantization steps.

The NVFP4 element format (E2M1) is checked against a library codec
(ml_dtypes' float4_e2m1fn) and against brute-force nearest search over its
eight magnitudes; the packer against blocks worked by hand and against
brute force per element; the NVFP4 GEMM reference against a dense float64
matmul of operands decoded by the library and against an integer case worked
by hand; the FP8-to-bf16 dequantizer against a bit-level single rounding of
the exact product and against a constructed double-rounding witness.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

from fp8_block_scaled_group_b200 import inputs

# The E2M1 magnitudes by code, from the format's definition (OCP Microscaling
# Formats, E2M1: bias 1, one mantissa bit, no Inf or NaN).
E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def lib_e2m1_encode(vals_f32):
    return np.ascontiguousarray(vals_f32, dtype=np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)


def lib_e2m1_decode(codes):
    return np.asarray(codes, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def lib_e4m3_decode(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def brute_nearest_e2m1(t: float) -> int:
    """Nearest of the 16 codes by distance, a tie going to the even code."""
    a = abs(t)
    d = [abs(m - a) for m in E2M1_MAGNITUDES]
    best = min(d)
    idx = [i for i, v in enumerate(d) if v == best]
    code = idx[0] if len(idx) == 1 else [i for i in idx if i % 2 == 0][0]
    return code | (8 if np.signbit(t) else 0)


def unpack(q):
    """[R, K/2] bytes -> [R, K] codes, even K index from the low nibble."""
    out = np.empty((q.shape[0], q.shape[1] * 2), np.uint8)
    out[:, 0::2] = q & 0xF
    out[:, 1::2] = q >> 4
    return out


# ---------------------------------------------------------------- E2M1 --

def test_e2m1_decode_matches_format_and_library(oracle_mod):
    ours = np.array([oracle_mod.e2m1_decode(c) for c in range(16)])
    assert list(ours[:8]) == E2M1_MAGNITUDES
    assert list(-ours[8:]) == E2M1_MAGNITUDES
    assert all(np.signbit(ours[8:])) and not any(np.signbit(ours[:8]))
    lib = lib_e2m1_decode(np.arange(16))
    assert np.array_equal(ours, lib) and np.array_equal(np.signbit(ours), np.signbit(lib))


def test_e2m1_every_code_round_trips(oracle_mod):
    for c in range(16):
        assert oracle_mod.e2m1_encode(oracle_mod.e2m1_decode(c)) == c


def test_e2m1_midpoints_go_to_the_even_code(oracle_mod):
    # between each pair of neighbours, the midpoint takes the code whose
    # mantissa bit is 0
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for t, code in cases.items():
        assert oracle_mod.e2m1_encode(t) == code
        assert oracle_mod.e2m1_encode(-t) == code | 8
    # saturation at 6, and the sign of zero
    assert oracle_mod.e2m1_encode(6.5) == 7 and oracle_mod.e2m1_encode(1e30) == 7
    assert oracle_mod.e2m1_encode(float("inf")) == 7
    assert oracle_mod.e2m1_encode(-1e30) == 15
    assert oracle_mod.e2m1_encode(-0.0) == 8 and oracle_mod.e2m1_encode(-0.2) == 8


def test_e2m1_encoder_matches_library_on_a_dense_sweep(oracle_mod):
    # every fp32 whose low 12 mantissa bits are zero, in [0, 16): about 2^20
    # values covering every binade, midpoint and saturation region, plus
    # random fp32 and their negatives
    hi = np.arange(0, 0x41800000 >> 12, dtype=np.uint32) << 12
    rng = np.random.default_rng(7)
    rnd = rng.uniform(-10.0, 10.0, 200_000).astype(np.float32)
    tiny = (rng.standard_normal(50_000) * 0.3).astype(np.float32)
    t = np.concatenate([hi.view(np.float32), -hi.view(np.float32), rnd, tiny])
    ours = oracle_mod.e2m1_encode_array(t)
    assert np.array_equal(ours, lib_e2m1_encode(t))


def test_e2m1_encoder_is_brute_force_nearest(oracle_mod):
    rng = np.random.default_rng(11)
    t = np.concatenate([np.arange(-8.0, 8.0, 1.0 / 64), rng.uniform(-7, 7, 3000)]).astype(np.float32)
    ours = oracle_mod.e2m1_encode_array(t)
    assert [int(c) for c in ours] == [brute_nearest_e2m1(float(v)) for v in t]


# ---------------------------------------------------------- NVFP4 packer --

def bf16_row(vals, k=16):
    row = np.zeros(k, np.float32)
    row[:len(vals)] = vals
    bits = inputs.f32_to_bf16_bits(row)
    assert np.array_equal(inputs.bf16_bits_to_f32(bits), row), "hand-worked values must be bf16-exact"
    return bits[None, :]


def test_pack_hand_worked_unit_scale(oracle_mod):
    # amax 6 with s2 = 1: the block scale is 6/6 = 1 (E4M3 0x38) and every
    # value below is an E2M1 magnitude, coded as is
    q, sf = oracle_mod.nvfp4_quant(bf16_row([6.0, 3.0, -1.5, 0.5]), 1.0)
    assert sf.tolist() == [[0x38]]
    # codes 7, 5 | 0xB, 1 | zeros: even index in the low nibble
    assert q.tolist() == [[0x57, 0x1B, 0, 0, 0, 0, 0, 0]]


def test_pack_hand_worked_rounding_and_second_level(oracle_mod):
    # amax 12: scale 2 (0x40); 12/2 = 6 -> 7; 1/2 = 0.5 -> 1; 5/2 = 2.5 is a
    # midpoint of 2 and 3 and goes to the even code 4 (2.0)
    q, sf = oracle_mod.nvfp4_quant(bf16_row([12.0, 1.0, 5.0]), 1.0)
    assert sf.tolist() == [[0x40]] and q[0, :2].tolist() == [0x17, 0x04]
    # the same block as the first hand case with s2 = 0.5: 6 / (6 * 0.5) = 2
    # gives block code 2.0, and the effective scale 2 * 0.5 = 1 codes as before
    q, sf = oracle_mod.nvfp4_quant(bf16_row([6.0, 3.0, -1.5, 0.5]), 0.5)
    assert sf.tolist() == [[0x40]] and q[0, :2].tolist() == [0x57, 0x1B]


def test_pack_scale_saturates_then_elements_saturate(oracle_mod):
    # amax 5376 = 6 * 448 * 2: amax/6 = 896 saturates to 448 (0x7E); 5376/448
    # = 12 saturates to 6; 1344/448 = 3 is exact
    q, sf = oracle_mod.nvfp4_quant(bf16_row([5376.0, 1344.0]), 1.0)
    assert sf.tolist() == [[0x7E]] and q[0, 0] == (0x7 | (0x5 << 4))


def test_pack_subnormal_and_zero_block_scales(oracle_mod):
    # amax 6 * 2^-8: the block scale 2^-8 is the E4M3 subnormal 2 * 2^-9
    q, sf = oracle_mod.nvfp4_quant(bf16_row([6.0 * 2.0 ** -8, -3.0 * 2.0 ** -8]), 1.0)
    assert sf.tolist() == [[0x02]] and q[0, 0] == (0x7 | (0xD << 4))
    # amax 6 * 2^-11: amax/6 = 2^-11 rounds to an E4M3 zero; every element is
    # then a zero with its own sign
    q, sf = oracle_mod.nvfp4_quant(bf16_row([6.0 * 2.0 ** -11, -2.0 ** -12]), 1.0)
    assert sf.tolist() == [[0x00]] and q[0, 0] == 0x80
    q, sf = oracle_mod.nvfp4_quant(bf16_row([-2.0 ** -12, 6.0 * 2.0 ** -11]), 1.0)
    assert sf.tolist() == [[0x00]] and q[0, 0] == 0x08
    # an all-zero block
    q, sf = oracle_mod.nvfp4_quant(bf16_row([]), 1.0)
    assert sf.tolist() == [[0x00]] and not q.any()


def test_pack_rejects_bad_arguments(oracle_mod):
    x = bf16_row([1.0], k=32)
    for s2 in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(ValueError):
            oracle_mod.nvfp4_quant(x, s2)
    with pytest.raises(ValueError):
        oracle_mod.nvfp4_quant(np.zeros((1, 24), np.uint16), 1.0)


@pytest.mark.parametrize("use_global", [False, True])
def test_pack_is_nearest_per_element_with_the_stated_block_scale(oracle_mod, use_global):
    # activations with outliers (the FP8 path's recipe) and small weights
    for x in (inputs.activations(6, 256, seed=5), inputs.weights(6, 256, seed=6)):
        s2 = oracle_mod.nvfp4_global_scale(x) if use_global else 1.0
        q, sf = oracle_mod.nvfp4_quant(x, s2)
        xf = inputs.bf16_bits_to_f32(x).reshape(6, 16, 16)
        amax = np.abs(xf).max(axis=2)
        t = amax / (np.float32(6.0) * np.float32(s2))                   # fp32, as stated
        assert np.array_equal(sf, oracle_mod.e4m3_encode_array(t).reshape(6, 16))
        s = (lib_e4m3_decode(sf).astype(np.float32) * np.float32(s2))   # fp32 product
        codes = unpack(q).reshape(6, 16, 16)
        for r in range(6):
            for b in range(16):
                for j in range(16):
                    v = xf[r, b, j]
                    want = (8 if np.signbit(v) else 0) if s[r, b] == 0 else \
                        brute_nearest_e2m1(float(np.float32(v) / s[r, b]))
                    assert codes[r, b, j] == want, (r, b, j)


def test_pack_saturation_is_bounded_by_the_scale_rounding(oracle_mod):
    # a normal E4M3 block scale is amax/(6 s2) to within 2^-4 relative, so no
    # element lands above 6 * (1 + 2^-4) before saturation
    x = inputs.activations(32, 1024, seed=9)
    q, sf = oracle_mod.nvfp4_quant(x, 1.0)
    xf = inputs.bf16_bits_to_f32(x).reshape(32, 64, 16)
    s = lib_e4m3_decode(sf)
    normal = (sf >= 0x08) & (sf < 0x7E)
    ratio = np.abs(xf).max(axis=2)[normal] / s[normal]
    assert ratio.max() <= 6.0 * (1 + 2.0 ** -4)


def test_global_scale_closed_forms(oracle_mod):
    assert oracle_mod.nvfp4_global_scale(bf16_row([2688.0])) == 1.0
    assert oracle_mod.nvfp4_global_scale(bf16_row([-5376.0])) == 2.0
    assert oracle_mod.nvfp4_global_scale(bf16_row([])) == float(np.float32(1e-10) / np.float32(2688.0))
    # with s2 from the tensor's own amax, its largest block takes scale 448
    w = inputs.weights(8, 512, seed=3)
    s2 = oracle_mod.nvfp4_global_scale(w)
    _, sf = oracle_mod.nvfp4_quant(w, s2)
    assert sf.max() == 0x7E


# ------------------------------------------------------ NVFP4 reference --

def dense(q, sf, s2):
    codes = unpack(q)
    return lib_e2m1_decode(codes) * np.repeat(lib_e4m3_decode(sf), 16, axis=1) * float(s2)


def test_gemm_ref_matches_dense_matmul(oracle_mod):
    x = inputs.activations(7, 320, seed=21)
    w = inputs.weights(9, 320, seed=22)
    s2w = oracle_mod.nvfp4_global_scale(w)
    qa, sfa = oracle_mod.nvfp4_quant(x, 1.0)
    qw, sfw = oracle_mod.nvfp4_quant(w, s2w)
    ref = oracle_mod.nvfp4_gemm_ref(qa, sfa, 1.0, qw, sfw, s2w)
    want = dense(qa, sfa, 1.0) @ dense(qw, sfw, s2w).T
    assert np.allclose(ref, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    rows = np.array([6, 0, 3])
    assert np.array_equal(oracle_mod.nvfp4_gemm_ref(qa, sfa, 1.0, qw, sfw, s2w, rows=rows), ref[rows])


def test_gemm_ref_integer_case_by_hand(oracle_mod):
    # row a: block 0 all 1.0 (code 2) scale 1 (0x38); block 1 all 2.0 (code 4)
    # scale 2 (0x40). Weight row: block 0 all 3.0 (code 5) scale 0.5 (0x30);
    # block 1 all -0.5 (code 9) scale 4 (0x48). s2a = 1, s2w = 0.25:
    #   (16*1*3*1*0.5 + 16*2*(-0.5)*2*4) * 0.25 = (24 - 128) / 4 = -26
    qa = np.array([[0x22] * 8 + [0x44] * 8], np.uint8)
    sfa = np.array([[0x38, 0x40]], np.uint8)
    qw = np.array([[0x55] * 8 + [0x99] * 8], np.uint8)
    sfw = np.array([[0x30, 0x48]], np.uint8)
    assert oracle_mod.nvfp4_gemm_ref(qa, sfa, 1.0, qw, sfw, 0.25).tolist() == [[-26.0]]


def test_gemm_ref_negative_controls(oracle_mod):
    x = inputs.activations(8, 256, seed=31)
    w = inputs.weights(16, 256, seed=32)
    qa, sfa = oracle_mod.nvfp4_quant(x, 1.0)
    qw, sfw = oracle_mod.nvfp4_quant(w, 1.0)
    ref = oracle_mod.nvfp4_gemm_ref(qa, sfa, 1.0, qw, sfw, 1.0)
    rms = np.sqrt(np.mean(ref ** 2))
    # nibbles read in the other order
    swapped = ((qw & 0xF) << 4) | (qw >> 4)
    bad = oracle_mod.nvfp4_gemm_ref(qa, sfa, 1.0, swapped, sfw, 1.0)
    assert np.abs(bad - ref).max() > 0.1 * rms
    # weight scales read as if they were [K/16, N]
    sfw_t = np.ascontiguousarray(sfw.reshape(-1)[np.arange(sfw.size).reshape(sfw.shape[1], -1).T.reshape(-1)]
                                 .reshape(sfw.shape))
    bad = oracle_mod.nvfp4_gemm_ref(qa, sfa, 1.0, qw, sfw_t, 1.0)
    assert np.abs(bad - ref).max() > 0.1 * rms


# ------------------------------------------------ FP8 dequant to bf16 --

def bf16_round_once(v: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits, one round-to-nearest-even on the float64 bit
    pattern (normal range only)."""
    bits = np.ascontiguousarray(v, dtype=np.float64).view(np.uint64)
    lsb = (bits >> np.uint64(45)) & np.uint64(1)
    r = (bits + np.uint64((1 << 44) - 1) + lsb) >> np.uint64(45) << np.uint64(45)
    f32 = r.view(np.float64).astype(np.float32)            # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


@pytest.mark.parametrize("per_row", [False, True])
def test_dequant_is_one_rounding_of_the_exact_product(oracle_mod, per_row):
    w = inputs.weights(256, 384, seed=41)
    wq, ws = oracle_mod.quant_weight_rowwise(w) if per_row else oracle_mod.quant_weight(w)
    out = oracle_mod.dequant_fp8_bf16(wq, ws)
    scale = np.repeat(ws[:, None], 384, axis=1) if per_row else \
        np.repeat(np.repeat(ws, 128, axis=0), 128, axis=1)
    exact = lib_e4m3_decode(wq) * scale.astype(np.float64)   # exact in float64
    nz = exact != 0
    assert np.array_equal(out[nz], bf16_round_once(exact[nz]))
    assert np.array_equal(out[~nz], np.where(np.signbit(exact[~nz]), 0x8000, 0).astype(np.uint16))
    # the dequantized weight stays close to the bf16 weight it came from
    wf = inputs.bf16_bits_to_f32(w)
    assert np.abs(inputs.bf16_bits_to_f32(out) - wf).max() <= np.abs(wf).max() / 16


def test_dequant_does_not_round_twice(oracle_mod):
    # find fp32 scales s for which code 1.5 (0x3C) times s, rounded first to
    # fp32 and then to bf16, differs from the exact product rounded once; the
    # oracle must give the single rounding
    base = np.float32(2.0 / 3.0).view(np.uint32)
    s = (base + np.arange(-300_000, 300_000, dtype=np.int64)).astype(np.uint32).view(np.float32)
    p32 = np.float32(1.5) * s
    via_f32 = bf16_round_once(p32.astype(np.float64))
    once = bf16_round_once(1.5 * s.astype(np.float64))
    witnesses = np.nonzero(via_f32 != once)[0][:4]
    assert witnesses.size >= 2
    for i in witnesses:
        # the exact product and the bf16 chosen, checked with rationals
        exact = Fraction(3, 2) * Fraction(float(s[i]))
        got = oracle_mod.dequant_fp8_bf16(np.full((1, 128), 0x3C, np.uint8), np.array([s[i]], np.float32))[0, 0]
        assert got == once[i] and got != via_f32[i]
        lo = Fraction(float(inputs.bf16_bits_to_f32(np.array([got], np.uint16))[0]))
        other = Fraction(float(inputs.bf16_bits_to_f32(np.array([via_f32[i]], np.uint16))[0]))
        assert abs(exact - lo) < abs(exact - other)


def test_dequant_rejects_untiled_shapes(oracle_mod):
    with pytest.raises(AssertionError):
        oracle_mod.dequant_fp8_bf16(np.zeros((128, 200), np.uint8), np.ones((1, 1), np.float32))
