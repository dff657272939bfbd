"""The bounded waits' error path, run on the GPU without faulting it.

fp8q_diag_stalled_linear launches the fused linear's two kernels with their
copies suppressed and a wait budget of about a millisecond, so every wait
that needs a copy runs out. Each kernel must then raise its bit of the
device error word, drain, free its tensor memory and return; the context must
stay usable, which the normal linear right after checks against the oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
BUDGET = 2_000_000  # SM clocks, about a millisecond


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("m,n,k", [(300, 512, 1024), (17, 384, 1024)])
def test_stalled_kernels_report_a_timeout_and_the_context_survives(m, n, k):
    lib = _lib.load()
    assert api.device_error() == 0
    xb, wb = inputs.activations(m, k, 31), inputs.weights(n, k, 32)
    x = _dev_bf16(xb)
    wq, ws = api.quant_weight(_dev_bf16(wb))
    work = torch.zeros(api.linear_workspace_bytes(m, k), dtype=torch.uint8, device=DEV)
    y = torch.zeros((m, n), dtype=torch.bfloat16, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.fp8q_diag_stalled_linear(_p(x), _p(wq), _p(ws), _p(y), _p(work), work.numel(), m, n, k, BUDGET, stream)
    assert st == 0, lib.fp8q_status_string(st).decode()
    code = ctypes.c_uint32(0)
    st = lib.fp8q_device_error(stream, ctypes.byref(code))
    assert st == 6  # FP8Q_ERR_DEVICE_TIMEOUT
    assert code.value & 1, "the GEMM did not report its timeout"
    assert code.value & 4, "the quantizer did not report its timeout"
    assert api.device_error() == 0  # read-and-clear

    # The same context runs the normal path correctly right after.
    y = api.linear(x, wq, ws)
    torch.cuda.synchronize()
    q_o, s_row_o, _ = oracle.quant_act(xb)
    wq_o, ws_o = oracle.quant_weight(wb)
    ref = oracle.gemm_ref(q_o, s_row_o, wq_o, ws_o, threads=4)
    bad, worst = oracle.check_tolerance(y.view(torch.int16).cpu().numpy().view(np.uint16), ref)
    assert bad == 0, f"{bad} outputs outside tolerance after the stalled launch (worst {worst:.3f})"
    assert api.device_error() == 0


def test_stalled_linear_argument_errors():
    lib = _lib.load()
    d = torch.empty(256, dtype=torch.uint8, device=DEV)
    args = [_p(d)] * 5 + [d.numel(), 16, 128, 128]
    assert lib.fp8q_diag_stalled_linear(*args, 0, None) == 8               # FP8Q_ERR_ARG: no budget
    assert lib.fp8q_diag_stalled_linear(*args, 3_000_000_000, None) == 8   # beyond the one-second bound
