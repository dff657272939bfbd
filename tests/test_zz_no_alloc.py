"""fp8q_linear_noalloc: the fused linear for callers that cannot allocate.

Some callers are handed inputs and outputs but cannot get a device buffer
for the linear's intermediate FP8 activation (a plugin inside a runtime that
owns the device-memory budget, or a loop where cudaMalloc could stall the
device). This entry point keeps that intermediate in a fixed array inside
the library. Here it is called through the C ABI several times in a row:
first a problem that fills 96 % of the array (M=900 at K=17408), then a
smaller prefill-width one and a decode-width one, so each later call runs
over the earlier calls' leftovers. It runs the same kernels as fp8q_linear
on the same inputs, so each output must equal fp8q_linear's bit for bit.

Collected last on purpose: a run that stops at the first failure has then
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_block_scaled_group_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
SCRATCH_BYTES = 16 << 20  # the array's stated size


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


CASES = [(900, 256, 17408, 7), (300, 384, 5120, 5), (17, 256, 1024, 6)]


def test_noalloc_cases_span_the_scratch():
    need = [api.linear_workspace_bytes(m, k) for m, _, k, _ in CASES]
    assert need[0] <= SCRATCH_BYTES and need[0] > 0.95 * SCRATCH_BYTES
    assert need == sorted(need, reverse=True)


def test_noalloc_matches_linear_bit_for_bit_calls_in_a_row():
    lib = _lib.load()
    for m, n, k, seed in CASES:
        x = _dev_bf16(inputs.activations(m, k, seed))
        wq, ws = api.quant_weight(_dev_bf16(inputs.weights(n, k, seed)))
        y_ref = api.linear(x, wq, ws)
        y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        st = lib.fp8q_linear_noalloc(_ptr(x), _ptr(wq), _ptr(ws), _ptr(y), m, n, k, _stream())
        assert st == 0, lib.fp8q_status_string(st).decode()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), \
            f"M={m} N={n} K={k}: fp8q_linear_noalloc differs from fp8q_linear"
    assert api.device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = _lib.load()
    m, n, k = 4096, 128, 17408  # needs ~73 MB of scratch, more than the 16 MiB held
    assert api.linear_workspace_bytes(m, k) > SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device=DEV)
    st = lib.fp8q_linear_noalloc(_ptr(dummy), _ptr(dummy), _ptr(dummy), _ptr(dummy), m, n, k, _stream())
    assert st == 4  # FP8Q_ERR_WORKSPACE, nothing enqueued
