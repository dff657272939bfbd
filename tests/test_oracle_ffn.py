"""Pins of the oracle's dense-FFN pieces against computations it does not share.

The FFN (quantize once for gate and up, SiLU(gate) * up rounded to bf16,
quantize again for down) is checked here against:
  * a 200-digit decimal evaluation of silu(g) * u with exact rational
    rounding to bf16 (Python's decimal and fractions modules),
  * constructed rounding ties, where the answer follows from silu(g) < g,
  * signed zeros, underflow and overflow worked by hand,
  * a numpy float64 composition of the stages with codes decoded by torch.
"""
import math
from decimal import Decimal, localcontext
from fractions import Fraction

import numpy as np
import pytest
import torch

from fp8_block_scaled_group_b200 import inputs

BF16_INF = 0x7F80


def bits_to_float(b: int) -> float:
    return float(np.array([int(b) << 16], np.uint32).view(np.float32)[0])


def round_magnitude_to_bf16(a: Fraction, tie_ok: bool) -> int:
    """bf16 magnitude bits of a > 0, nearest, ties to even (exact rationals)."""
    assert a > 0
    e = math.frexp(float(a))[1] - 1  # 2^e <= a < 2^(e+1), up to one step
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (-133) if e < -126 else Fraction(2) ** (e - 7)
    n = a / quantum
    fl = n.numerator // n.denominator
    frac = n - fl
    if frac == Fraction(1, 2):
        assert tie_ok, "value is a rounding tie at this precision"
        r = fl if fl % 2 == 0 else fl + 1
    else:
        assert tie_ok or abs(frac - Fraction(1, 2)) > Fraction(1, 10 ** 180), "too close to a tie"
        r = fl + 1 if frac > Fraction(1, 2) else fl
    mag = r * quantum
    if mag >= Fraction(2) ** 128:
        return BF16_INF
    return int(np.array([float(mag)], np.float32).view(np.uint32)[0] >> 16)


def ref_silu_mul(gb: int, ub: int) -> int:
    """bf16 of the real silu(g) * u, from a 200-digit decimal evaluation."""
    g, u = bits_to_float(gb), bits_to_float(ub)
    sign = (gb ^ ub) & 0x8000
    p = g * u  # exact in binary64: two 8-bit significands
    if p == 0.0:
        return sign
    with localcontext() as ctx:
        ctx.prec = 200
        v = Decimal(p) / (1 + (-Decimal(g)).exp())
    # Fraction(v) is exact; abs() on a Decimal would round it to the
    # default 28-digit context
    return sign | round_magnitude_to_bf16(abs(Fraction(v)), tie_ok=False)


def ref_round_bf16(x: float) -> int:
    if x == 0.0:
        return 0x8000 if math.copysign(1.0, x) < 0 else 0
    sign = 0x8000 if x < 0 else 0
    return sign | round_magnitude_to_bf16(Fraction(abs(x)), tie_ok=True)


def bf16(vals):
    return inputs.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


# ------------------------------------------------------------- SiLU * up --

def test_silu_mul_matches_high_precision_decimal(oracle_mod):
    rng = np.random.default_rng(20261202)
    g_parts = [bf16(rng.normal(0, 3, 1500)), bf16(rng.normal(0, 40, 400))]
    raw = rng.integers(0, 0x10000, 3000, dtype=np.uint32).astype(np.uint16)
    fin = raw[(raw & 0x7F80) != 0x7F80]
    mag = np.abs(inputs.bf16_bits_to_f32(fin))
    g_parts.append(fin[mag <= 300][:400])
    g = np.concatenate(g_parts)
    u_parts = [bf16(rng.normal(0, 2, g.size // 2))]
    raw = rng.integers(0, 0x10000, 4 * g.size, dtype=np.uint32).astype(np.uint16)
    u_parts.append(raw[(raw & 0x7F80) != 0x7F80][: g.size - u_parts[0].size])
    u = np.concatenate(u_parts)
    assert u.size == g.size
    h = oracle_mod.silu_mul_bf16(g, u)
    want = np.array([ref_silu_mul(int(a), int(b)) for a, b in zip(g, u)], np.uint16)
    bad = np.nonzero(h != want)[0]
    assert bad.size == 0, [(hex(g[i]), hex(u[i]), hex(h[i]), hex(want[i])) for i in bad[:5]]
    # the sample reaches the paths that matter
    hv = inputs.bf16_bits_to_f32(h)
    assert np.any(np.isinf(hv)) and np.any(hv == 0) and np.any((hv != 0) & (np.abs(hv) < 2.0 ** -126))


@pytest.mark.parametrize("g,u,want", [
    # g*u sits exactly halfway between two bf16 values; silu(g) < g puts the
    # real value just below it, so it rounds toward zero, not to even.
    (48.0, 1 + 1 / 128, 48.25),      # tie 48.375 between 48.25 and 48.5 (even)
    (24.0, 1 + 1 / 128, 24.125),     # tie 24.1875 between 24.125 and 24.25 (even)
    (48.0, -(1 + 1 / 128), -48.25),
    (96.0, 1 + 3 / 128, 98.0),       # tie 98.25 between 98.0 (even) and 98.5
    (192.0, 1 + 1 / 128, 193.0),     # tie 193.5 between 193 and 194 (even)
])
def test_silu_mul_ties_round_toward_zero(oracle_mod, g, u, want):
    gb, ub = bf16([g])[0], bf16([u])[0]
    assert bits_to_float(gb) == g and bits_to_float(ub) == u
    p = Fraction(g) * Fraction(u)
    # g*u is exactly a tie of the bf16 grid
    h_lo, h_hi = ref_round_bf16(float(p) * (1 - 2 ** -40)), ref_round_bf16(float(p) * (1 + 2 ** -40))
    assert h_lo != h_hi
    got = oracle_mod.silu_mul_bf16(np.array([gb]), np.array([ub]))[0]
    assert bits_to_float(got) == want
    assert got == ref_silu_mul(int(gb), int(ub))


def test_silu_mul_moderate_gate_scan(oracle_mod):
    # Gates in (8, 32] with every u in [1, 2): e^-g is small but still moves
    # the rounding when g*u lies just above a tie, so the result is not
    # simply bf16(g*u) there. The scan must contain such non-tie cases.
    g_vals = [8.0625 + j / 16 for j in range(16)] + [10.5, 12.25, 16.5, 20.0, 24.0, 31.0, 32.0]
    gb = bf16(g_vals)
    ub = np.arange(0x3F80, 0x4000, dtype=np.uint16)
    G, U = (a.ravel() for a in np.meshgrid(gb, ub, indexing="ij"))
    h = oracle_mod.silu_mul_bf16(G, U)
    want = np.array([ref_silu_mul(int(a), int(b)) for a, b in zip(G, U)], np.uint16)
    assert np.array_equal(h, want)
    prod = inputs.bf16_bits_to_f32(G).astype(np.float64) * inputs.bf16_bits_to_f32(U)
    is_tie = np.array([ref_round_bf16(x * (1 - 2 ** -40)) != ref_round_bf16(x * (1 + 2 ** -40)) for x in prod])
    moved = (h != np.array([ref_round_bf16(float(x)) for x in prod], np.uint16)) & ~is_tie
    assert moved.sum() >= 20


def test_silu_mul_large_gate_is_rounded_product(oracle_mod):
    # for g > 32 and g*u not on a tie the result is bf16(g*u)
    g = bf16([33.0, 40.0, 100.0, 1e4, 3e38])
    u = bf16([1.0, -3.0, 0.5, 1e-3, 1.0])
    h = oracle_mod.silu_mul_bf16(g, u)
    prod = inputs.bf16_bits_to_f32(g).astype(np.float64) * inputs.bf16_bits_to_f32(u)
    want = np.array([ref_round_bf16(float(x)) for x in prod], np.uint16)
    assert np.array_equal(h, want)


def test_silu_mul_signed_zero_underflow_overflow(oracle_mod):
    f = lambda gv, uv: int(oracle_mod.silu_mul_bf16(bf16([gv]), bf16([uv]))[0])
    assert f(0.0, 1.0) == 0x0000 and f(0.0, -1.0) == 0x8000
    assert f(-0.0, 1.0) == 0x8000 and f(-0.0, -1.0) == 0x0000
    assert f(3.0, 0.0) == 0x0000 and f(3.0, -0.0) == 0x8000 and f(-3.0, 0.0) == 0x8000
    # e^-200 * 200 is far below the smallest bf16 subnormal (2^-133): signed zero
    assert f(-200.0, 1.0) == 0x8000 and f(-200.0, -1.0) == 0x0000
    # silu(-100) * 2^100 ~ -100 * (2/e)^100: a normal number
    v = f(-100.0, 2.0 ** 100)
    assert v == ref_silu_mul(int(bf16([-100.0])[0]), int(bf16([2.0 ** 100])[0]))
    assert 0x8080 <= v < 0xFF80
    # overflow of the bf16 range gives infinity with the product's sign
    assert f(3e38, 3e38) == 0x7F80 and f(3e38, -3e38) == 0xFF80
    # silu(1) = 1/(1+e^-1) = 0.73105857863... -> 0.73046875 (187/256), bf16 0x3F3B
    assert f(1.0, 1.0) == 0x3F3B
    # silu(-1) = -(1 - silu(1)) ... = -0.26894142137 -> -0.26953125 (-69/256)
    assert bits_to_float(f(-1.0, 1.0)) == -69 / 256


def test_round_bf16_array(oracle_mod):
    rng = np.random.default_rng(7)
    vals = [0.0, -0.0, 1.0, -1.0, 2.0 ** -130, -(2.0 ** -140), 3.4e38, -3.4e38, 1e39]
    # exact ties between neighbouring bf16 values, both parities
    for e in (-130, -127, -20, 0, 7, 100):
        for k in (0, 1, 2, 3, 77):
            q = 2.0 ** (e - 7) if e >= -126 else 2.0 ** -133
            base = (2.0 ** e if e >= -126 else 0.0) + k * q
            vals.append(base + q / 2)
            vals.append(-(base + q / 2))
    vals += list(rng.normal(0, 1, 500)) + list(rng.normal(0, 1, 200) * 1e-39) + list(rng.normal(0, 1e30, 100))
    vals = np.array(vals, np.float64)
    got = oracle_mod.round_bf16(vals)
    want = np.array([ref_round_bf16(float(x)) for x in vals], np.uint16)
    assert np.array_equal(got, want)


# ---------------------------------------------- SiLU * up, then quantized --

@pytest.mark.parametrize("m", [1, 15, 17])
def test_silu_mul_quant_is_quant_of_h(oracle_mod, m):
    i = 384
    rng = np.random.default_rng(m)
    g = bf16(rng.normal(0, 3, (m, i)))
    u = bf16(rng.normal(0, 2, (m, i)))
    q, s_row, s_k = oracle_mod.silu_mul_quant(g, u)
    h = np.array([ref_silu_mul(int(a), int(b)) for a, b in zip(g.ravel(), u.ravel())],
                 np.uint16).reshape(m, i)
    q2, s_row2, s_k2 = oracle_mod.quant_act(h)
    assert np.array_equal(q, q2)
    assert np.array_equal(s_row.view(np.uint32), s_row2.view(np.uint32))
    assert np.array_equal(s_k.view(np.uint32), s_k2.view(np.uint32))
    mp = oracle_mod.m_pad(m)
    assert s_k.shape == (i // 128, mp) and not np.any(s_k[:, m:].view(np.uint32))


def test_silu_mul_quant_reads_stacked_halves_in_place(oracle_mod):
    # gate and up as the two halves of one [m, 2i] row (row stride 2i): the
    # same result as contiguous copies of the halves
    m, i = 5, 256
    rng = np.random.default_rng(9)
    gu = bf16(rng.normal(0, 3, (m, 2 * i)))
    got = oracle_mod.silu_mul_quant_stacked(gu)
    want = oracle_mod.silu_mul_quant(np.ascontiguousarray(gu[:, :i]), np.ascontiguousarray(gu[:, i:]))
    for a, b in zip(got, want):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


# ------------------------------------------------------- FFN composition --

def deq(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def numpy_gemm(q, s_row, wq, ws):
    a = deq(q) * np.repeat(s_row.astype(np.float64), 128, axis=1)
    w = deq(wq) * np.repeat(np.repeat(ws.astype(np.float64), 128, axis=0), 128, axis=1)
    return a @ w.T


def test_ffn_ref_stages(oracle_mod):
    m, d, i = 5, 256, 384
    x = inputs.activations(m, d, seed=11)
    w_gu = inputs.weights(2 * i, d, seed=12)
    w_dn = inputs.weights(d, i, seed=13)
    wq_gu, ws_gu = oracle_mod.quant_weight(w_gu)
    wq_dn, ws_dn = oracle_mod.quant_weight(w_dn)
    out = oracle_mod.ffn_ref(x, wq_gu, ws_gu, wq_dn, ws_dn)
    q_x, s_x, _ = oracle_mod.quant_act(x)
    assert np.array_equal(out["q_x"], q_x)
    gu = numpy_gemm(q_x, s_x, wq_gu, ws_gu)
    gate = np.array([ref_round_bf16(float(v)) for v in gu[:, :i].ravel()], np.uint16).reshape(m, i)
    up = np.array([ref_round_bf16(float(v)) for v in gu[:, i:].ravel()], np.uint16).reshape(m, i)
    assert np.array_equal(out["gate"], gate) and np.array_equal(out["up"], up)
    h = np.array([ref_silu_mul(int(a), int(b)) for a, b in zip(gate.ravel(), up.ravel())],
                 np.uint16).reshape(m, i)
    q_h, s_h, s_h_k = oracle_mod.quant_act(h)
    assert np.array_equal(out["q_h"], q_h)
    assert np.array_equal(out["s_h"].view(np.uint32), s_h.view(np.uint32))
    assert np.array_equal(out["s_h_kmajor"].view(np.uint32), s_h_k.view(np.uint32))
    y = numpy_gemm(q_h, s_h, wq_dn, ws_dn)
    assert np.allclose(out["y"], y, rtol=1e-12, atol=1e-12 * np.sqrt(np.mean(y * y)))
    # the gate half really feeds SiLU: swapping gate and up changes the result
    q_sw, _, _ = oracle_mod.silu_mul_quant(up, gate)
    assert not np.array_equal(q_sw, q_h)
