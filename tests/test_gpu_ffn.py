"""Parity of the dense FFN path (through the C ABI) with the CPU oracle.

SiLU(gate) * up and its quantization: bit-exact against the oracle on seeded
gate/up inputs and on constructed special values, plus an exhaustive device
check of the fp32 fast path against the fp64 path over all 2^32 bf16 pairs.

The whole FFN, link by link:
  q_x, s_x      bit-exact against the oracle's quantization of x
  gate | up     within the GEMM tolerance of the oracle's float64 GEMM
  q_h, s_h      bit-identical to fp8q_silu_mul_quant run on that gate | up
  y             bit-identical to fp8q_gemm_blockscaled run on that q_h
  y end to end  against the oracle's FFN (its own gate/up, h and codes):
                |y - ref| <= 8e-3 |ref| + 2e-2 rms(ref), and the relative
                rms error below 5e-3. The looser bound covers h codes that
                land on the other side of an e4m3 rounding boundary when the
                projections' bf16 outputs differ in the last bit.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group_b200 import api, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_quant_equal(got, want, what=""):
    q, s_row, s_k = (None if a is None else (a.cpu().numpy() if isinstance(a, torch.Tensor) else a) for a in got)
    q_o, s_row_o, s_k_o = want
    assert np.array_equal(q, q_o), f"{what}: {int((q != q_o).sum())} FP8 bytes differ"
    if s_row is not None:
        assert np.array_equal(s_row.view(np.uint32), s_row_o.view(np.uint32)), f"{what}: row-major scales differ"
    assert np.array_equal(s_k.view(np.uint32), s_k_o.view(np.uint32)), f"{what}: K-major scales differ"


# --------------------------------------------------------- SiLU * up ------

@pytest.mark.parametrize("m", [1, 4, 17, 33, 130])
@pytest.mark.parametrize("i", [128, 1152, 17408])
def test_silu_mul_quant_bitexact(m, i):
    gb, ub = inputs.gate_up(m, i, seed=500 + m)
    got = api.silu_mul_quant(to_dev_bf16(gb), to_dev_bf16(ub))
    torch.cuda.synchronize()
    assert_quant_equal(got, oracle.silu_mul_quant(gb, ub), f"m={m} i={i}")


@pytest.mark.parametrize("m,i", [(3, 256), (25, 17408)])
def test_silu_mul_quant_strided_halves(m, i):
    gb, ub = inputs.gate_up(m, i, seed=77)
    both = np.concatenate([gb, ub], axis=1)  # [m, 2i]: gate then up, as the FFN lays them out
    buf = to_dev_bf16(both)
    got = api.silu_mul_quant(buf[:, :i], buf[:, i:])
    torch.cuda.synchronize()
    assert_quant_equal(got, oracle.silu_mul_quant(gb, ub), "strided")


def special_gate_up():
    """Rows of hand-picked (gate, up) values: exact ties with large gates,
    zeros of both signs, large negative gates (underflow to zero), bf16
    subnormal results, products near the top of the range, tiny gates.
    No pair overflows bf16: an infinite h would make its group's scale
    infinite, which is outside the quantizer's contract."""
    f = lambda v: inputs.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))
    pairs = [(48.0, 1 + 1 / 128), (24.0, 1 + 1 / 128), (96.0, 1 + 3 / 128), (192.0, 1 + 1 / 128),
             (48.0, -(1 + 1 / 128)), (0.0, 1.0), (-0.0, 1.0), (3.0, -0.0), (-200.0, 1.0), (-200.0, -1.0),
             (-100.0, 2.0 ** 100), (-90.0, 1.0), (-80.0, 1e-3), (1e-30, 1e-10), (-1e-38, 3.0), (3e38, 1.0),
             (1e19, 1e19), (1.8e19, 1.8e19), (-24.0, 1.0), (-24.5, 1.0), (-23.75, 1.0), (17.0, 1 + 1 / 128),
             (8.0625, 1.5), (8.0625, 1.5078125), (1.0, 1.0), (-1.0, 1.0), (0.5, -2.0), (88.0, 3.0)]
    rng = np.random.default_rng(3)
    g = np.concatenate([f([p[0] for p in pairs]), f(rng.normal(0, 3, 256 - len(pairs)))])
    u = np.concatenate([f([p[1] for p in pairs]), f(rng.normal(0, 3, 256 - len(pairs)))])
    # row 1: every bf16 gate in [8, 32) against one up value, row 2: negatives
    g1 = np.arange(0x4100, 0x4200, dtype=np.uint16)[:256]
    g2 = g1 | np.uint16(0x8000)
    u1 = f(np.full(256, 1.0078125))
    return np.stack([g, g1, g2, g[::-1]]), np.stack([u, u1, u1, u[::-1]])


def test_silu_mul_quant_special_values():
    gb, ub = special_gate_up()
    got = api.silu_mul_quant(to_dev_bf16(gb), to_dev_bf16(ub))
    torch.cuda.synchronize()
    assert_quant_equal(got, oracle.silu_mul_quant(gb, ub), "special")


def test_silu_mul_fast_path_exhaustive():
    pairs, taken, bad, worst = api.check_silu_mul()
    print(f"pairs {pairs} fast-path {taken} ({taken / pairs:.3f}) mismatches {bad} worst {worst:.2f} ulp")
    assert pairs == 65280 * 65280  # every finite bf16 gate x every finite bf16 up
    assert bad == 0, f"{bad} pairs where the fp32 path rounds differently from the fp64 path"
    assert taken > pairs // 4
    # the fast result stands only if v(1 +- 2^-20) round alike: at least 8 ulps of v
    assert worst < 4.0, f"fp32 path error {worst} ulps: too close to the 8-ulp band"


# --------------------------------------------------------------- FFN ------

def ffn_weights(d, i, seed):
    wq_gu, ws_gu = oracle.quant_weight(inputs.weights(2 * i, d, seed))
    wq_dn, ws_dn = oracle.quant_weight(inputs.weights(d, i, seed + 1))
    return wq_gu, ws_gu, wq_dn, ws_dn


def run_ffn(xb, wq_gu, ws_gu, wq_dn, ws_dn):
    m, d = xb.shape
    i = wq_gu.shape[0] // 2
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    ws = torch.empty(api.ffn_workspace_layout(m, d, i)[5], dtype=torch.uint8, device=DEV)
    w = (dev(wq_gu), dev(ws_gu), dev(wq_dn), dev(ws_dn))
    y = api.ffn(to_dev_bf16(xb), *w, workspace=ws)
    torch.cuda.synchronize()
    return y, api.ffn_intermediates(ws, m, d, i), w


def check_ffn_rows(xb, rows, wq_gu, ws_gu, wq_dn, ws_dn):
    m, d = xb.shape
    i = wq_gu.shape[0] // 2
    y, mid, w = run_ffn(xb, wq_gu, ws_gu, wq_dn, ws_dn)
    rows = np.asarray(rows)
    # link 1: x quantized once, exactly as the activation quantizer does
    q_x_o, s_x_o, _ = oracle.quant_act(xb[rows])
    assert np.array_equal(mid["q_x"].cpu().numpy()[rows], q_x_o)
    s_x_k = mid["s_x_kmajor"].cpu().numpy()
    assert np.array_equal(s_x_k[:, rows].T.view(np.uint32), s_x_o.view(np.uint32))
    assert not np.any(s_x_k[:, m:].view(np.uint32))
    # link 2: gate | up against the float64 GEMM of the same codes
    gu_ref = oracle.gemm_ref(q_x_o, s_x_o, wq_gu, ws_gu, threads=8)
    gu = bf16_bits(mid["gate_up"])[rows]
    bad, worst = oracle.check_tolerance(gu, gu_ref)
    assert bad == 0, f"gate|up: {bad} elements out of tolerance (worst {worst:.2f})"
    # link 3: q_h, s_h are SiLU*up of that gate | up, quantized
    gate_up = mid["gate_up"]
    q_h, _, s_h = api.silu_mul_quant(gate_up[:, :i], gate_up[:, i:], row_major=False)
    torch.cuda.synchronize()
    assert torch.equal(q_h, mid["q_h"]) and torch.equal(s_h.view(torch.int32), mid["s_h_kmajor"].view(torch.int32))
    # link 4: y is the down projection of that q_h
    y2 = api.gemm_blockscaled(mid["q_h"], mid["s_h_kmajor"], w[2], w[3])
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    # end to end against the oracle's own FFN
    ref = oracle.ffn_ref(xb[rows], wq_gu, ws_gu, wq_dn, ws_dn, threads=8)
    yv = inputs.bf16_bits_to_f32(bf16_bits(y)[rows]).astype(np.float64)
    r = ref["y"]
    rms = float(np.sqrt(np.mean(r * r)))
    err = np.abs(yv - r)
    assert np.all(err <= 8e-3 * np.abs(r) + 2e-2 * rms), f"worst |y-ref|/rms = {err.max() / rms:.3e}"
    rel = float(np.sqrt(np.mean(err * err)) / rms)
    assert rel < 5e-3, f"relative rms error {rel:.3e}"
    flips = int((ref["q_h"] != mid["q_h"].cpu().numpy()[rows]).sum())
    return rel, flips


@pytest.mark.parametrize("m,d,i", [(1, 256, 384), (17, 256, 384), (130, 384, 256), (300, 256, 1152)])
def test_ffn_small_full(m, d, i):
    xb = inputs.activations(m, d, seed=900 + m)
    check_ffn_rows(xb, np.arange(m), *ffn_weights(d, i, seed=901))


@pytest.mark.parametrize("wl", inputs.FFN_CONFIGS, ids=lambda w: w.name)
def test_ffn_workloads_sampled(wl):
    xb = wl.x()
    wq_gu, ws_gu = oracle.quant_weight(wl.w_gate_up())
    wq_dn, ws_dn = oracle.quant_weight(wl.w_down())
    rows = sorted({0, wl.m - 1, wl.m // 2, (7 * wl.m) // 11})
    check_ffn_rows(xb, rows, wq_gu, ws_gu, wq_dn, ws_dn)


def test_ffn_m_zero_launches_nothing():
    lib = api._lib.load()
    before = api.launch_count()
    assert lib.fp8q_ffn(None, None, None, None, None, None, None, 0, 0, 256, 384, None) == 0
    assert api.launch_count() == before
