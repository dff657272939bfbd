"""Parity of the NVFP4 kernels (through the C ABI) with the CPU oracle.

Packed E2M1 bytes and E4M3 scales (both layouts) and the FP8-to-bf16
dequantizer: bit-exact. NVFP4 GEMM outputs: every compared element within
|y - ref| <= 8e-3 |ref| + 1e-3 rms(ref) of the float64 reference.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group_b200 import api, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
GUARD = 4096


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def bf16_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def sf_mma_layout(sf_row, k):
    """The row-major [rows, k/16] scales placed as the MMA layout the header
    describes: atom (r/128, k/64) of 512 bytes, K-fastest, byte
    (r%32)*16 + ((r%128)/32)*4 + (k/16)%4 inside; pad rows zero."""
    rows = sf_row.shape[0]
    pad = (rows + 127) // 128 * 128
    out = np.zeros(pad * k // 16, np.uint8)
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(k // 16, dtype=np.int64)[None, :]
    off = ((r >> 7) * (k >> 6) + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3)
    out[off] = sf_row
    return out


def test_e2m1_conversion_exhaustive_over_the_rounding_range():
    """Every fp32 in [2^-3, 8] (both signs) covers every E2M1 rounding
    boundary; tiny, huge and special values are sampled."""
    lo = int(np.float32(0.125).view(np.uint32))
    hi = int(np.float32(8.0).view(np.uint32))
    step = 1 << 24
    for start in range(lo, hi + 1, step):
        v = np.arange(start, min(start + step, hi + 1), dtype=np.uint32).view(np.float32)
        for sign in (1.0, -1.0):
            t = v * np.float32(sign)
            got = api.convert_e2m1(torch.from_numpy(t).to(DEV)).cpu().numpy()
            assert np.array_equal(got, oracle.e2m1_encode_array(t)), hex(start)
    rng = np.random.default_rng(5)
    extra = np.concatenate([rng.uniform(0, 0.125, 1 << 16).astype(np.float32),
                            np.array([0.0, 1e-45, 1e-38, 0.25, 5.0, 6.0, 7.0, 1e6, 3.4e38, np.inf], np.float32)])
    extra = np.concatenate([extra, -extra])
    got = api.convert_e2m1(torch.from_numpy(extra).to(DEV)).cpu().numpy()
    assert np.array_equal(got, oracle.e2m1_encode_array(extra))


def pack_case(xb, s2):
    rows, k = xb.shape
    q_o, sf_o = oracle.nvfp4_quant(xb, s2)
    q, sf_row, sf_mma = api.nvfp4_quant(to_dev_bf16(xb), s2)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(sf_row.cpu().numpy(), sf_o)
    assert np.array_equal(sf_mma.cpu().numpy(), sf_mma_layout(sf_o, k))
    return q, sf_mma, q_o, sf_o


@pytest.mark.parametrize("rows,k", [(1, 64), (17, 512), (128, 256), (129, 5120), (300, 2048)])
@pytest.mark.parametrize("use_global", [False, True])
def test_nvfp4_quant_bitexact(rows, k, use_global):
    for xb in (inputs.activations(rows, k, seed=rows + k), inputs.weights(rows, k, seed=rows * 3 + k)):
        s2 = oracle.nvfp4_global_scale(xb) if use_global else 1.0
        pack_case(xb, s2)


def test_nvfp4_quant_special_blocks():
    k = 128
    rows = np.zeros((4, k), np.float32)
    rows[1, :16] = -0.0
    rows[1, 16:32] = [-2.0 ** -12] + [6.0 * 2.0 ** -11] * 15          # scale rounds to zero
    rows[2, :16] = [5376.0, 1344.0] + [0.0] * 14                         # scale saturates at 448
    rows[3, :16] = [6.0 * 2.0 ** -8] + [-3.0 * 2.0 ** -8] * 15           # E4M3-subnormal scale
    pack_case(inputs.f32_to_bf16_bits(rows), 1.0)


@pytest.mark.parametrize("per_row", [False, True])
@pytest.mark.parametrize("n,k", [(128, 128), (256, 384), (6144, 5120)])
def test_dequant_fp8_bf16_bitexact(n, k, per_row):
    wb = inputs.weights(n, k, seed=n + k)
    wq, ws = oracle.quant_weight_rowwise(wb) if per_row else oracle.quant_weight(wb)
    y = api.dequant_fp8_bf16(torch.from_numpy(wq).to(DEV), torch.from_numpy(ws).to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(y), oracle.dequant_fp8_bf16(wq, ws))


def gemm_case(m, n, k, seed, rows=None):
    xb = inputs.activations(m, k, seed)
    wb = inputs.weights(n, k, seed + 1)
    s2w = oracle.nvfp4_global_scale(wb)
    qa_o, sfa_o = oracle.nvfp4_quant(xb, 1.0)
    qw_o, sfw_o = oracle.nvfp4_quant(wb, s2w)
    qa = torch.from_numpy(qa_o).to(DEV)
    qw = torch.from_numpy(qw_o).to(DEV)
    sfa = torch.from_numpy(sf_mma_layout(sfa_o, k)).to(DEV)
    sfw = torch.from_numpy(sf_mma_layout(sfw_o, k)).to(DEV)
    raw = torch.full((2 * m * n + GUARD,), 0xA5, dtype=torch.uint8, device=DEV)
    y = raw[:2 * m * n].view(torch.bfloat16).view(m, n)
    api.nvfp4_gemm(qa, sfa, 1.0, qw, sfw, s2w, out=y)
    torch.cuda.synchronize()
    assert api.device_error() == 0
    assert bool((raw[2 * m * n:] == 0xA5).all().item()), "GEMM wrote past its output"
    rows = np.arange(m, dtype=np.int64) if rows is None else rows
    ref = oracle.nvfp4_gemm_ref(qa_o, sfa_o, 1.0, qw_o, sfw_o, s2w, rows=rows)
    return oracle.check_tolerance(bf16_bits(y)[rows], ref)


@pytest.mark.parametrize("m,n,k", [(1, 128, 256), (17, 256, 512), (128, 384, 256), (129, 512, 1024),
                                   (300, 768, 2048), (256, 256, 5120),
                                   # one row of 128-column tiles: K split over clusters of 5, 8 and 8
                                   # CTAs, with K stages that do not divide evenly
                                   (64, 1024, 1280), (33, 2048, 3584), (128, 768, 5120),
                                   # M <= 32: 32-row A stages, split (2) and persistent (400 tiles)
                                   (32, 1024, 1280), (8, 51200, 256)])
def test_nvfp4_gemm_full(m, n, k):
    bad, worst = gemm_case(m, n, k, seed=m + n + k)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


@pytest.mark.parametrize("m,n,k", [(25, 6144, 5120), (1168, 17408, 5120)])
def test_nvfp4_gemm_workload_sampled(m, n, k):
    rng = np.random.default_rng(m)
    rows = np.unique(np.concatenate([[0, m - 1], rng.choice(m, min(m, 32), replace=False)])).astype(np.int64)
    bad, worst = gemm_case(m, n, k, seed=7, rows=rows)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


def test_nvfp4_gemm_integer_case_exact():
    # unit scales (E4M3 1.0 = 0x38), codes of small integers: exact sums
    rng = np.random.default_rng(2)
    m, n, k = 40, 256, 512
    ca = rng.choice(np.array([0x0, 0x2, 0x4, 0xA, 0xC], np.uint8), size=(m, k))   # 0, 1, 2, -1, -2
    cw = rng.choice(np.array([0x0, 0x2, 0xA], np.uint8), size=(n, k))              # 0, 1, -1
    ca[:, 64:] = 0
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    qa_o, qw_o = pack(ca), pack(cw)
    sfa_o = np.full((m, k // 16), 0x38, np.uint8)
    sfw_o = np.full((n, k // 16), 0x38, np.uint8)
    y = api.nvfp4_gemm(torch.from_numpy(qa_o).to(DEV), torch.from_numpy(sf_mma_layout(sfa_o, k)).to(DEV), 1.0,
                       torch.from_numpy(qw_o).to(DEV), torch.from_numpy(sf_mma_layout(sfw_o, k)).to(DEV), 1.0)
    ref = oracle.nvfp4_gemm_ref(qa_o, sfa_o, 1.0, qw_o, sfw_o, 1.0)
    assert np.array_equal(inputs.bf16_bits_to_f32(bf16_bits(y)).astype(np.float64), ref)


@pytest.mark.parametrize("m,n,k", [(17, 256, 512), (300, 512, 1024)])
def test_nvfp4_linear_matches_pack_then_gemm(m, n, k):
    xb = inputs.activations(m, k, seed=m)
    wb = inputs.weights(n, k, seed=n)
    s2w = oracle.nvfp4_global_scale(wb)
    qw, _, sfw = api.nvfp4_quant(to_dev_bf16(wb), s2w, row_major=False)
    y = api.nvfp4_linear(to_dev_bf16(xb), qw, sfw, s2w)
    qa, _, sfa = api.nvfp4_quant(to_dev_bf16(xb), 1.0, row_major=False)
    y2 = api.nvfp4_gemm(qa, sfa, 1.0, qw, sfw, s2w)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(y), bf16_bits(y2))
    qa_o, sfa_o = oracle.nvfp4_quant(xb, 1.0)
    qw_o, sfw_o = oracle.nvfp4_quant(wb, s2w)
    bad, worst = oracle.check_tolerance(bf16_bits(y), oracle.nvfp4_gemm_ref(qa_o, sfa_o, 1.0, qw_o, sfw_o, s2w))
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


def test_nvfp4_from_fp8_weight():
    """The pages' from-FP8 arm: dequantize the FP8 weight to bf16, pack it
    with s2 = 1, run the projection."""
    m, n, k = 33, 256, 1024
    xb = inputs.activations(m, k, seed=3)
    wq_o, ws_o = oracle.quant_weight(inputs.weights(n, k, seed=4))
    w_bf16 = api.dequant_fp8_bf16(torch.from_numpy(wq_o).to(DEV), torch.from_numpy(ws_o).to(DEV))
    qw, _, sfw = api.nvfp4_quant(w_bf16, 1.0, row_major=False)
    y = api.nvfp4_linear(to_dev_bf16(xb), qw, sfw, 1.0)
    torch.cuda.synchronize()
    wd = oracle.dequant_fp8_bf16(wq_o, ws_o)
    qa_o, sfa_o = oracle.nvfp4_quant(xb, 1.0)
    qw_o, sfw_o = oracle.nvfp4_quant(wd, 1.0)
    bad, worst = oracle.check_tolerance(bf16_bits(y), oracle.nvfp4_gemm_ref(qa_o, sfa_o, 1.0, qw_o, sfw_o, 1.0))
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"
