"""Parity of the per-row FP8 weight format (scale block 1 x K) with the oracle.

Weight codes and per-row scales: bit-exact. GEMM and linear outputs: every
compared element within |y - ref| <= 8e-3 |ref| + 1e-3 rms(ref) of the
float64 reference, at edge shapes in full, at the decode shapes in full and
at the prefill shape on sampled rows; the fused linear is bit-identical to
quantize-then-GEMM.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group_b200 import api, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def bf16_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@functools.lru_cache(maxsize=None)
def oracle_w_rowwise(n, k, seed):
    wb = inputs.weights(n, k, seed)
    wq, ws = oracle.quant_weight_rowwise(wb)
    return wb, wq, ws


@pytest.mark.parametrize("n,k", [(128, 128), (256, 640), (384, 17408), (6144, 5120)])
def test_quant_weight_rowwise_bitexact(n, k):
    wb, wq_o, ws_o = oracle_w_rowwise(n, k, seed=n + k)
    wq, ws = api.quant_weight_rowwise(to_dev_bf16(wb))
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy(), wq_o)
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), ws_o.view(np.uint32))


def rowwise_case(m, n, k, seed, rows=None, p=0.01, sigma=20.0):
    xb = inputs.activations(m, k, seed, p, sigma)
    q, s_row, s_k = oracle.quant_act(xb)
    _, wq_o, ws_o = oracle_w_rowwise(n, k, seed)
    y = api.gemm_blockscaled(torch.from_numpy(q).to(DEV), torch.from_numpy(s_k).to(DEV),
                             torch.from_numpy(wq_o).to(DEV), torch.from_numpy(ws_o).to(DEV))
    torch.cuda.synchronize()
    rows = np.arange(m, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    ref = oracle.gemm_ref(q, s_row, wq_o, ws_o, rows=rows, threads=8)
    return oracle.check_tolerance(bf16_bits(y)[rows], ref)


@pytest.mark.parametrize("m,n,k", [(1, 128, 128), (16, 512, 512), (17, 128, 640), (64, 256, 384), (65, 256, 384),
                                   (100, 256, 256), (129, 128, 1024), (300, 384, 1024)])
def test_gemm_rowwise_edges_full(m, n, k):
    bad, worst = rowwise_case(m, n, k, seed=m + 3 * n + k)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


@pytest.mark.parametrize("m,n,k", [(16, 6144, 5120), (25, 6144, 5120), (25, 5120, 17408)])
def test_gemm_rowwise_decode_full(m, n, k):
    bad, worst = rowwise_case(m, n, k, seed=1002)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


def test_gemm_rowwise_prefill_sampled():
    m, n, k = 1168, 17408, 5120
    rows = [0, 1, 127, 128, 255, 256, 600, 1023, 1024, 1151, 1166, 1167]
    bad, worst = rowwise_case(m, n, k, seed=1004, rows=rows)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


@pytest.mark.parametrize("m,n,k", [(25, 6144, 5120), (300, 384, 1024)])
def test_linear_rowwise_is_quant_then_gemm(m, n, k):
    xb = inputs.activations(m, k, seed=m)
    _, wq_o, ws_o = oracle_w_rowwise(n, k, seed=k)
    x = to_dev_bf16(xb)
    wq, ws = torch.from_numpy(wq_o).to(DEV), torch.from_numpy(ws_o).to(DEV)
    y = api.linear(x, wq, ws)
    q, _, s_k = api.quant_act(x, row_major=False)
    y2 = api.gemm_blockscaled(q, s_k, wq, ws)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_weight_format_argument_checked():
    lib = api._lib.load()
    a = torch.zeros(16, dtype=torch.uint8, device=DEV)
    assert lib.fp8q_gemm_ex(api._p(a), api._p(a), api._p(a), api._p(a), 7, api._p(a), 1, 128, 128, None) == 8
