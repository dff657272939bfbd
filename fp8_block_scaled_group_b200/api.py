"""PyTorch-facing calls of the fp8q C ABI.

Each function takes CUDA tensors, checks dtype/shape/contiguity, allocates
outputs with torch when the caller gives none, and passes raw device
pointers plus the current CUDA stream to libfp8q.so. No arithmetic of the
method happens here.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

AUTO, SINGLE, MULTI = 0, 1, 2
WEIGHT_BLOCK128, WEIGHT_PER_ROW = 0, 1
GROUP = 128


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _p(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, dtype, shape, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def m_pad(m: int) -> int:
    return int(_lib.load().fp8q_m_pad(m))


def quant_pick(m: int, k: int, sm_count: int, requested: int = AUTO) -> _lib.QuantPick:
    out = _lib.QuantPick()
    _lib.check(_lib.load().fp8q_quant_pick(m, k, sm_count, requested, ctypes.byref(out)), "fp8q_quant_pick")
    return out


def quant_floor_min_m(k: int, sm_count: int, groups_per_cta: int, rows_per_cta: int,
                      min_ctas_per_sm: float) -> int:
    return int(_lib.load().fp8q_quant_floor_min_m(k, sm_count, groups_per_cta, rows_per_cta, min_ctas_per_sm))


def quant_act(x: torch.Tensor, variant: int = AUTO, row_major: bool = True, out=None, stream=None):
    """x bf16 [M, K] -> (q uint8 [M, K], s_row fp32 [M, K/128] or None, s_kmajor fp32 [K/128, ceil16(M)])."""
    m, k = x.shape
    _need(x, torch.bfloat16, (m, k), "x")
    g, mp = k // GROUP, m_pad(m)
    if out is None:
        q = torch.empty((m, k), dtype=torch.uint8, device=x.device)
        s_row = torch.empty((m, g), dtype=torch.float32, device=x.device) if row_major else None
        s_k = torch.empty((g, mp), dtype=torch.float32, device=x.device)
    else:
        q, s_row, s_k = out
    lib = _lib.load()
    if variant == AUTO:
        st = lib.fp8q_quant_act(_p(x), _p(q), _p(s_row), _p(s_k), m, k, _stream(stream))
    else:
        st = lib.fp8q_quant_act_variant(_p(x), _p(q), _p(s_row), _p(s_k), m, k, variant, _stream(stream))
    _lib.check(st, "fp8q_quant_act")
    return q, s_row, s_k


def quant_weight(w: torch.Tensor, stream=None):
    """w bf16 [N, K] -> (wq uint8 [N, K], w_scale fp32 [N/128, K/128])."""
    n, k = w.shape
    _need(w, torch.bfloat16, (n, k), "w")
    wq = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    ws = torch.empty((n // GROUP, k // GROUP), dtype=torch.float32, device=w.device)
    _lib.check(_lib.load().fp8q_quant_weight(_p(w), _p(wq), _p(ws), n, k, _stream(stream)), "fp8q_quant_weight")
    return wq, ws


def quant_weight_rowwise(w: torch.Tensor, stream=None):
    """w bf16 [N, K] -> (wq uint8 [N, K], w_scale fp32 [N]), one scale per weight row."""
    n, k = w.shape
    _need(w, torch.bfloat16, (n, k), "w")
    wq = torch.empty((n, k), dtype=torch.uint8, device=w.device)
    ws = torch.empty((n,), dtype=torch.float32, device=w.device)
    _lib.check(_lib.load().fp8q_quant_weight_rowwise(_p(w), _p(wq), _p(ws), n, k, _stream(stream)),
               "fp8q_quant_weight_rowwise")
    return wq, ws


def _weight_format(w_scale: torch.Tensor, n: int, k: int) -> int:
    """The weight format its scale tensor's shape selects: [N/128, K/128] or [N]."""
    if tuple(w_scale.shape) == (n,):
        _need(w_scale, torch.float32, (n,), "w_scale")
        return WEIGHT_PER_ROW
    _need(w_scale, torch.float32, (n // GROUP, k // GROUP), "w_scale")
    return WEIGHT_BLOCK128


def gemm_blockscaled(q: torch.Tensor, s_kmajor: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """q uint8 [M,K], s_kmajor fp32 [K/128, ceil16(M)], wq uint8 [N,K], w_scale fp32 [N/128,K/128]
    (block-scaled) or [N] (per row) -> y bf16 [M,N]."""
    m, k = q.shape
    n = wq.shape[0]
    _need(q, torch.uint8, (m, k), "q")
    _need(s_kmajor, torch.float32, (k // GROUP, m_pad(m)), "s_kmajor")
    _need(wq, torch.uint8, (n, k), "wq")
    fmt = _weight_format(w_scale, n, k)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=q.device) if out is None else out
    _need(y, torch.bfloat16, (m, n), "y")
    _lib.check(_lib.load().fp8q_gemm_ex(_p(q), _p(s_kmajor), _p(wq), _p(w_scale), fmt, _p(y), m, n, k,
                                         _stream(stream)), "fp8q_gemm_ex")
    return y


def linear_workspace_bytes(m: int, k: int) -> int:
    return int(_lib.load().fp8q_linear_workspace_bytes(m, k))


def linear_scale_offset(m: int, k: int) -> int:
    return int(_lib.load().fp8q_linear_scale_offset(m, k))


def linear(x: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor, workspace: torch.Tensor | None = None,
           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Fused W8A8 linear: x bf16 [M,K] -> y bf16 [M,N] (quantize + block-scaled GEMM in one call)."""
    m, k = x.shape
    n = wq.shape[0]
    _need(x, torch.bfloat16, (m, k), "x")
    _need(wq, torch.uint8, (n, k), "wq")
    fmt = _weight_format(w_scale, n, k)
    need = linear_workspace_bytes(m, k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(y, torch.bfloat16, (m, n), "y")
    _lib.check(_lib.load().fp8q_linear_ex(_p(x), _p(wq), _p(w_scale), fmt, _p(y), _p(workspace),
                                           workspace.numel(), m, n, k, _stream(stream)), "fp8q_linear_ex")
    return y


def silu_mul_quant(gate: torch.Tensor, up: torch.Tensor, row_major: bool = True, out=None, stream=None):
    """gate, up bf16 [M, I] (rows may be strided, e.g. the two halves of a
    [M, 2I] buffer) -> quant_act(bf16(silu(gate) * up)) as
    (q uint8 [M, I], s_row fp32 [M, I/128] or None, s_kmajor fp32 [I/128, ceil16(M)])."""
    if gate.shape != up.shape or gate.dim() != 2:
        raise ValueError("gate and up must be 2-D with the same shape")
    m, i = gate.shape
    for name, t in (("gate", gate), ("up", up)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.stride(1) != 1:
            raise ValueError(f"{name} must be a bf16 CUDA tensor with unit column stride")
    ld = gate.stride(0) if m > 1 else i
    if m > 1 and up.stride(0) != ld:
        raise ValueError("gate and up must share one row stride")
    g, mp = i // GROUP, m_pad(m)
    if out is None:
        q = torch.empty((m, i), dtype=torch.uint8, device=gate.device)
        s_row = torch.empty((m, g), dtype=torch.float32, device=gate.device) if row_major else None
        s_k = torch.empty((g, mp), dtype=torch.float32, device=gate.device)
    else:
        q, s_row, s_k = out
    _lib.check(_lib.load().fp8q_silu_mul_quant(_p(gate), _p(up), ld, _p(q), _p(s_row), _p(s_k), m, i,
                                                _stream(stream)), "fp8q_silu_mul_quant")
    return q, s_row, s_k


def ffn_workspace_layout(m: int, d: int, i: int) -> list[int]:
    """Byte offsets of q_x, s_x, gate|up, q_h, s_h in the FFN workspace, then its size."""
    off = (_lib.SZ * 6)()
    _lib.check(_lib.load().fp8q_ffn_workspace_layout(m, d, i, off), "fp8q_ffn_workspace_layout")
    return [int(v) for v in off]


def ffn(x: torch.Tensor, wq_gate_up: torch.Tensor, ws_gate_up: torch.Tensor, wq_down: torch.Tensor,
        ws_down: torch.Tensor, workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
        stream=None) -> torch.Tensor:
    """Dense FFN: x bf16 [M, D] -> y bf16 [M, D] with y = down(silu(gate(x)) * up(x)), x quantized once.
    wq_gate_up uint8 [2I, D] (gate rows first), ws_gate_up fp32 [2I/128, D/128],
    wq_down uint8 [D, I], ws_down fp32 [D/128, I/128]."""
    m, d = x.shape
    i = wq_gate_up.shape[0] // 2
    _need(x, torch.bfloat16, (m, d), "x")
    _need(wq_gate_up, torch.uint8, (2 * i, d), "wq_gate_up")
    _need(ws_gate_up, torch.float32, (2 * i // GROUP, d // GROUP), "ws_gate_up")
    _need(wq_down, torch.uint8, (d, i), "wq_down")
    _need(ws_down, torch.float32, (d // GROUP, i // GROUP), "ws_down")
    need = ffn_workspace_layout(m, d, i)[5]
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    y = torch.empty((m, d), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(y, torch.bfloat16, (m, d), "y")
    _lib.check(_lib.load().fp8q_ffn(_p(x), _p(wq_gate_up), _p(ws_gate_up), _p(wq_down), _p(ws_down), _p(y),
                                     _p(workspace), workspace.numel(), m, d, i, _stream(stream)), "fp8q_ffn")
    return y


def ffn_intermediates(workspace: torch.Tensor, m: int, d: int, i: int) -> dict:
    """Views of the FFN's intermediates inside its workspace (after the call has run)."""
    off = ffn_workspace_layout(m, d, i)
    mp = m_pad(m)

    def view(k, dtype, shape):
        n = 1
        for v in shape:
            n *= v
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return workspace[off[k]:off[k] + nbytes].view(dtype).view(*shape)

    return {"q_x": view(0, torch.uint8, (m, d)), "s_x_kmajor": view(1, torch.float32, (d // GROUP, mp)),
            "gate_up": view(2, torch.bfloat16, (m, 2 * i)), "q_h": view(3, torch.uint8, (m, i)),
            "s_h_kmajor": view(4, torch.float32, (i // GROUP, mp))}


def check_silu_mul(stream=None) -> tuple[int, int, int, float]:
    """Exhaustive check of SiLU(gate)*up's fp32 path against its fp64 path; returns
    (pairs, pairs on the fp32 path, of those the mismatches, worst fp32 error in ulps)."""
    counts = torch.zeros(3, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.check(_lib.load().fp8q_check_silu_mul(_p(counts), _p(err), _stream(stream)), "fp8q_check_silu_mul")
    a, b, c = counts.cpu().tolist()
    worst = float(err.cpu().view(torch.float32).item())
    return int(a), int(b), int(c), worst


def linear_decode_fused(x: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                        workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """linear() at decode widths (M <= 32) in one launch: the decode GEMM quantizes x itself.
    Bit-identical to linear(); slower on B200 (see fp8q_linear_decode_fused)."""
    m, k = x.shape
    n = wq.shape[0]
    _need(x, torch.bfloat16, (m, k), "x")
    _need(wq, torch.uint8, (n, k), "wq")
    fmt = _weight_format(w_scale, n, k)
    need = linear_workspace_bytes(m, k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(y, torch.bfloat16, (m, n), "y")
    _lib.check(_lib.load().fp8q_linear_decode_fused(_p(x), _p(wq), _p(w_scale), fmt, _p(y), _p(workspace),
                                                     workspace.numel(), m, n, k, _stream(stream)),
               "fp8q_linear_decode_fused")
    return y


# ---------------------------------------------------------------- NVFP4 --

NVFP4_BLOCK = 16


def nvfp4_sf_mma_bytes(rows: int, k: int) -> int:
    return int(_lib.load().fp8q_nvfp4_sf_mma_bytes(rows, k))


def nvfp4_quant(x: torch.Tensor, s2: float = 1.0, row_major: bool = True, stream=None):
    """x bf16 [R, K] -> (q uint8 [R, K/2] packed E2M1, sf_row uint8 [R, K/16] E4M3
    or None, sf_mma uint8 [nvfp4_sf_mma_bytes(R, K)] in the MMA layout)."""
    r, k = x.shape
    _need(x, torch.bfloat16, (r, k), "x")
    q = torch.empty((r, k // 2), dtype=torch.uint8, device=x.device)
    sf_row = torch.empty((r, k // NVFP4_BLOCK), dtype=torch.uint8, device=x.device) if row_major else None
    sf_mma = torch.empty((nvfp4_sf_mma_bytes(r, k),), dtype=torch.uint8, device=x.device)
    _lib.check(_lib.load().fp8q_nvfp4_quant(_p(x), _p(q), _p(sf_row), _p(sf_mma), float(s2), r, k,
                                             _stream(stream)), "fp8q_nvfp4_quant")
    return q, sf_row, sf_mma


def nvfp4_gemm(qa: torch.Tensor, sfa_mma: torch.Tensor, s2a: float, qw: torch.Tensor, sfw_mma: torch.Tensor,
               s2w: float, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """qa uint8 [M, K/2] + MMA-layout scales, qw uint8 [N, K/2] + MMA-layout scales -> y bf16 [M, N]."""
    m, half_k = qa.shape
    k = 2 * half_k
    n = qw.shape[0]
    _need(qa, torch.uint8, (m, half_k), "qa")
    _need(qw, torch.uint8, (n, half_k), "qw")
    _need(sfa_mma, torch.uint8, (nvfp4_sf_mma_bytes(m, k),), "sfa_mma")
    _need(sfw_mma, torch.uint8, (nvfp4_sf_mma_bytes(n, k),), "sfw_mma")
    y = torch.empty((m, n), dtype=torch.bfloat16, device=qa.device) if out is None else out
    _need(y, torch.bfloat16, (m, n), "y")
    _lib.check(_lib.load().fp8q_nvfp4_gemm(_p(qa), _p(sfa_mma), float(s2a), _p(qw), _p(sfw_mma), float(s2w),
                                            _p(y), m, n, k, _stream(stream)), "fp8q_nvfp4_gemm")
    return y


def nvfp4_linear_workspace_bytes(m: int, k: int) -> int:
    return int(_lib.load().fp8q_nvfp4_linear_workspace_bytes(m, k))


def nvfp4_linear(x: torch.Tensor, qw: torch.Tensor, sfw_mma: torch.Tensor, s2w: float, s2a: float = 1.0,
                 workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """NVFP4 projection: x bf16 [M, K] packed inside the call, times the packed weight -> y bf16 [M, N]."""
    m, k = x.shape
    n = qw.shape[0]
    _need(x, torch.bfloat16, (m, k), "x")
    _need(qw, torch.uint8, (n, k // 2), "qw")
    _need(sfw_mma, torch.uint8, (nvfp4_sf_mma_bytes(n, k),), "sfw_mma")
    if workspace is None:
        workspace = torch.empty(nvfp4_linear_workspace_bytes(m, k), dtype=torch.uint8, device=x.device)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device) if out is None else out
    _need(y, torch.bfloat16, (m, n), "y")
    _lib.check(_lib.load().fp8q_nvfp4_linear(_p(x), float(s2a), _p(qw), _p(sfw_mma), float(s2w), _p(y),
                                              _p(workspace), workspace.numel(), m, n, k, _stream(stream)),
               "fp8q_nvfp4_linear")
    return y


def dequant_fp8_bf16(wq: torch.Tensor, w_scale: torch.Tensor, stream=None) -> torch.Tensor:
    """wq uint8 [N, K] with fp32 scales [N/128, K/128] or [N] -> bf16 [N, K]."""
    n, k = wq.shape
    _need(wq, torch.uint8, (n, k), "wq")
    fmt = _weight_format(w_scale, n, k)
    y = torch.empty((n, k), dtype=torch.bfloat16, device=wq.device)
    _lib.check(_lib.load().fp8q_dequant_fp8_bf16(_p(wq), _p(w_scale), fmt, _p(y), n, k, _stream(stream)),
               "fp8q_dequant_fp8_bf16")
    return y


def convert_e2m1(t: torch.Tensor, stream=None) -> torch.Tensor:
    """fp32 CUDA tensor -> uint8 E2M1 codes (one per byte) with the packer's conversion."""
    if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError("t must be a contiguous fp32 CUDA tensor")
    out = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
    _lib.check(_lib.load().fp8q_convert_e2m1(_p(t), _p(out), t.numel(), _stream(stream)), "fp8q_convert_e2m1")
    return out


def convert_e4m3(t: torch.Tensor, stream=None) -> torch.Tensor:
    """fp32 CUDA tensor -> uint8 e4m3 codes with the quantizers' conversion."""
    if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError("t must be a contiguous fp32 CUDA tensor")
    out = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
    _lib.check(_lib.load().fp8q_convert_e4m3(_p(t), _p(out), t.numel(), _stream(stream)), "fp8q_convert_e4m3")
    return out


def check_division(stream=None) -> tuple[int, int, int, int]:
    """Run the exhaustive division check; returns (pairs, code mismatches,
    quotient mismatches, scale or reciprocal mismatches)."""
    counts = torch.zeros(4, dtype=torch.int64, device="cuda")
    _lib.check(_lib.load().fp8q_check_division(_p(counts), _stream(stream)), "fp8q_check_division")
    a, b, c, d = counts.cpu().tolist()
    return int(a), int(b), int(c), int(d)


def launch_count() -> int:
    return int(_lib.load().fp8q_launch_count())


def device_error(stream=None) -> int:
    code = ctypes.c_uint32(0)
    st = _lib.load().fp8q_device_error(_stream(stream), ctypes.byref(code))
    if st not in (0, 6):
        _lib.check(st, "fp8q_device_error")
    return int(code.value)
