"""Pins of the oracle's per-row FP8 weight format (scale block 1 x K).

Checked against: the activation quantizer (itself pinned) on rows of one
128-group, closed forms worked by hand, a numpy float64 dequantized matmul
with codes decoded by torch, and the block-scaled reference on weights whose
128 x 128 block scales are constant along K.
"""
import numpy as np
import pytest
import torch

from fp8_block_scaled_group_b200 import inputs


def deq(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_rowwise_quant_of_one_group_rows_is_the_activation_quantizer(oracle_mod):
    w = inputs.weights(256, 128, seed=5, sigma=1.0)
    wq, ws = oracle_mod.quant_weight_rowwise(w)
    q, s_row, _ = oracle_mod.quant_act(w)
    assert np.array_equal(wq, q)
    assert np.array_equal(ws.view(np.uint32), s_row[:, 0].view(np.uint32))


def test_rowwise_quant_closed_forms(oracle_mod):
    f = lambda v: inputs.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))
    k = 384
    rows = np.zeros((4, k), np.float32)
    rows[1, 300] = -3.5                  # single outlier
    rows[2, 5], rows[2, 200] = 8.0, 4.0  # 2v and v
    rows[3, :] = 0.25
    rows[3, 17] = 1.0
    wq, ws = oracle_mod.quant_weight_rowwise(f(rows))
    assert ws[0] == np.float32(np.float32(1e-10) / np.float32(448.0)) and not wq[0].any()
    assert ws[1] == np.float32(3.5) / np.float32(448.0) and wq[1, 300] == 0xFE
    assert np.count_nonzero(wq[1]) == 1
    assert ws[2] == np.float32(8.0) / np.float32(448.0) and wq[2, 5] == 0x7E and wq[2, 200] == 0x76
    assert wq[3, 17] == 0x7E and np.all(np.delete(wq[3], 17) == 0x6E)  # 0.25 * 448 = 112 = 1.75 * 2^6 -> 0x6E


def test_rowwise_quant_error_bound(oracle_mod):
    w = inputs.weights(130 * 2, 640, seed=9)[:200]
    wq, ws = oracle_mod.quant_weight_rowwise(w)
    x = inputs.bf16_bits_to_f32(w).astype(np.float64)
    rec = deq(wq) * ws.astype(np.float64)[:, None]
    # e4m3 keeps 3 fraction bits: relative error <= 2^-4 above the subnormal range
    big = np.abs(x) >= 2.0 ** -6 * ws[:, None]
    assert np.all(np.abs(rec - x)[big] <= 2.0 ** -4 * np.abs(x)[big] + 1e-30)
    amax = np.abs(x).max(axis=1)
    assert np.all(ws == (amax.astype(np.float32) / np.float32(448.0)))


@pytest.mark.parametrize("m,n,k", [(1, 128, 128), (5, 256, 384), (17, 128, 1152)])
def test_rowwise_gemm_ref_vs_numpy(oracle_mod, m, n, k):
    xb = inputs.activations(m, k, seed=m + k)
    q, s_row, _ = oracle_mod.quant_act(xb)
    wq, ws = oracle_mod.quant_weight_rowwise(inputs.weights(n, k, seed=n))
    ref = oracle_mod.gemm_ref(q, s_row, wq, ws)
    a = deq(q) * np.repeat(s_row.astype(np.float64), 128, axis=1)
    b = deq(wq) * ws.astype(np.float64)[:, None]
    want = a @ b.T
    assert np.allclose(ref, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_rowwise_geometry_matches_block_geometry_on_constant_scales(oracle_mod):
    m, n, k = 3, 256, 512
    xb = inputs.activations(m, k, seed=4)
    q, s_row, _ = oracle_mod.quant_act(xb)
    wq, _ = oracle_mod.quant_weight(inputs.weights(n, k, seed=4))
    c = np.array([0.5, 3.0], np.float32)              # one value per 128-row block
    ws_block = np.repeat(c[:, None], k // 128, axis=1)  # constant along K
    ws_row = np.repeat(c, 128)                          # the same per row
    assert np.array_equal(oracle_mod.gemm_ref(q, s_row, wq, ws_block), oracle_mod.gemm_ref(q, s_row, wq, ws_row))
    # negative control: the rows' scales in the wrong order change the result
    assert not np.allclose(oracle_mod.gemm_ref(q, s_row, wq, ws_row[::-1].copy()),
                           oracle_mod.gemm_ref(q, s_row, wq, ws_row))
