"""Launch shapes past the 65535-block limit of the second and third grid axes.

The SiLU*up quantizer's CTAs, the weight quantizer's 128 x 128 blocks and the
decode GEMM's 128-row weight slices are all counted on the first grid axis,
so token and block counts above 65535 run. Each call here is checked against
the CPU oracle: bit-exact for FP8 bytes and scales, the GEMM within its
tolerance, on block rows on both sides of 65536.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group_b200 import api, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
BLOCKS = 65537  # 128-row weight blocks: one more than the second grid axis holds


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_silu_mul_quant_more_tokens_than_grid_y():
    m, i = 70000, 256
    gb, ub = inputs.gate_up(m, i, seed=901)
    q, s_row, s_k = api.silu_mul_quant(to_dev_bf16(gb), to_dev_bf16(ub))
    torch.cuda.synchronize()
    q_o, s_row_o, s_k_o = oracle.silu_mul_quant(gb, ub)
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(s_row.cpu().numpy().view(np.uint32), s_row_o.view(np.uint32))
    assert np.array_equal(s_k.cpu().numpy().view(np.uint32), s_k_o.view(np.uint32))


@pytest.fixture(scope="module")
def tall_weight():
    """A [128 * 65537, 128] bf16 weight (seeded, N(0, 0.02) on the device) and
    its block quantization by the library."""
    n, k = 128 * BLOCKS, 128
    gen = torch.Generator(device=DEV)
    gen.manual_seed(902)
    w = (torch.randn((n, k), generator=gen, device=DEV, dtype=torch.float32) * 0.02).to(torch.bfloat16)
    wq, ws = api.quant_weight(w)
    torch.cuda.synchronize()
    yield w, wq, ws
    del w, wq, ws
    torch.cuda.empty_cache()


SAMPLED_BLOCKS = [0, 1, 40000, 65535, 65536]


def test_quant_weight_more_blocks_than_grid_y(tall_weight):
    w, wq, ws = tall_weight
    for b in SAMPLED_BLOCKS:
        rows = slice(128 * b, 128 * (b + 1))
        wq_o, ws_o = oracle.quant_weight(bf16_bits(w[rows]))
        assert np.array_equal(wq[rows].cpu().numpy(), wq_o), f"block row {b}"
        assert np.array_equal(ws[b:b + 1].cpu().numpy().view(np.uint32), ws_o.view(np.uint32)), f"block row {b}"


def test_decode_gemm_more_slices_than_grid_y(tall_weight):
    w, wq, ws = tall_weight
    m, k = 16, 128
    xb = inputs.activations(m, k, seed=903)
    q, _, s_k = api.quant_act(to_dev_bf16(xb))
    y = api.gemm_blockscaled(q, s_k, wq, ws)
    torch.cuda.synchronize()
    q_o, s_row_o, _ = oracle.quant_act(xb)
    for b in SAMPLED_BLOCKS:
        cols = slice(128 * b, 128 * (b + 1))
        ref = oracle.gemm_ref(q_o, s_row_o, wq[cols].cpu().numpy(), ws[b:b + 1].cpu().numpy())
        bad, worst = oracle.check_tolerance(bf16_bits(y[:, cols]), ref)
        assert bad == 0, f"weight block row {b}: {bad} outputs out of tolerance (worst err/bound {worst:.3f})"
