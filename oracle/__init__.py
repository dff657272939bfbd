"""CPU oracle for the FP8 block-scaled linear — TEST INFRASTRUCTURE ONLY.

A ctypes wrapper around ``fp8q_oracle.c``: the plain, slow CPU restatement of
per-token-group FP8 activation quantization, 128x128 block weight
quantization, the float64 dequantized GEMM reference, and the dense FFN built
from them: SiLU(gate) * up rounded to bf16 and quantized again for the down
projection, the FP8-to-bf16 weight dequantizer, and the NVFP4 projection
arms: E2M1 elements packed two to a byte with E4M3 scales per 16 along K and
an fp32 second-level scale (pages
"spark_model/layers/ops/dispatch_proj.rs" and
"spark_model/layers/ops/fp8_act_quant_floor.rs").

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never does, and
this package never imports the product.

Every function takes and returns numpy arrays. bf16 values travel as their
uint16 bit patterns and e4m3 values as uint8 codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8q_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GROUP = 128


def build(force: bool = False) -> str:
    """Compile the oracle with plain IEEE arithmetic (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        U32 = ctypes.c_uint32
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode_array.argtypes = [P, ctypes.c_size_t, P]
        lib.oracle_e4m3_encode_array.restype = None
        lib.oracle_m_pad.argtypes = [U32]
        lib.oracle_m_pad.restype = U32
        lib.oracle_quant_act.argtypes = [P, U32, U32, P, P, P]
        lib.oracle_quant_act.restype = ctypes.c_int
        lib.oracle_quant_weight.argtypes = [P, U32, U32, P, P]
        lib.oracle_quant_weight.restype = ctypes.c_int
        lib.oracle_gemm_ref_rows.argtypes = [P, P, P, P, U32, U32, P, ctypes.c_size_t,
                                             ctypes.c_size_t, P]
        lib.oracle_gemm_ref_rows.restype = None
        lib.oracle_gemm_ref_rows_geom.argtypes = [P, P, P, P, U32, U32, U32, U32, P, ctypes.c_size_t,
                                                  ctypes.c_size_t, P]
        lib.oracle_gemm_ref_rows_geom.restype = None
        lib.oracle_quant_weight_rowwise.argtypes = [P, U32, U32, P, P]
        lib.oracle_quant_weight_rowwise.restype = ctypes.c_int
        lib.oracle_check_tolerance.argtypes = [P, P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_double)]
        lib.oracle_check_tolerance.restype = ctypes.c_size_t
        lib.oracle_silu_mul_bf16.argtypes = [ctypes.c_uint16, ctypes.c_uint16]
        lib.oracle_silu_mul_bf16.restype = ctypes.c_uint16
        lib.oracle_silu_mul_bf16_array.argtypes = [P, P, ctypes.c_size_t, P]
        lib.oracle_silu_mul_bf16_array.restype = None
        lib.oracle_round_bf16_array.argtypes = [P, ctypes.c_size_t, P]
        lib.oracle_round_bf16_array.restype = None
        lib.oracle_silu_mul_quant.argtypes = [P, P, ctypes.c_size_t, U32, U32, P, P, P]
        lib.oracle_silu_mul_quant.restype = ctypes.c_int
        lib.oracle_dequant_fp8_bf16.argtypes = [P, P, U32, U32, U32, U32, P]
        lib.oracle_dequant_fp8_bf16.restype = ctypes.c_int
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.oracle_e2m1_encode_array.argtypes = [P, ctypes.c_size_t, P]
        lib.oracle_e2m1_encode_array.restype = None
        lib.oracle_nvfp4_quant.argtypes = [P, U32, U32, ctypes.c_float, P, P]
        lib.oracle_nvfp4_quant.restype = ctypes.c_int
        lib.oracle_nvfp4_global_scale.argtypes = [P, ctypes.c_size_t]
        lib.oracle_nvfp4_global_scale.restype = ctypes.c_float
        lib.oracle_nvfp4_gemm_ref_rows.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, U32, U32, P,
                                                   ctypes.c_size_t, ctypes.c_size_t, P]
        lib.oracle_nvfp4_gemm_ref_rows.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def bf16_to_f32(h: int) -> float:
    return float(_load().oracle_bf16_to_f32(int(h)))


def e4m3_decode(code: int) -> float:
    return float(_load().oracle_e4m3_decode(int(code)))


def e4m3_encode(t: float) -> int:
    return int(_load().oracle_e4m3_encode(float(t)))


def e4m3_encode_array(t: np.ndarray) -> np.ndarray:
    """Encode each fp32 value with the scalar encoder (for sweeps)."""
    t = np.ascontiguousarray(t, dtype=np.float32).ravel()
    out = np.empty(t.size, np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(t), t.size, _ptr(out))
    return out


def m_pad(m: int) -> int:
    return int(_load().oracle_m_pad(int(m)))


def quant_act(x_bf16: np.ndarray):
    """bf16 bits [M,K] -> (q [M,K] u8, s_row [M,K/128] f32, s_kmajor [K/128, ceil16(M)] f32)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    m, k = x.shape
    if k % GROUP:
        raise ValueError("k must be a multiple of 128")
    g = k // GROUP
    q = np.empty((m, k), np.uint8)
    s_row = np.empty((m, g), np.float32)
    s_k = np.empty((g, m_pad(m)), np.float32)
    rc = _load().oracle_quant_act(_ptr(x), m, k, _ptr(q), _ptr(s_row), _ptr(s_k))
    assert rc == 0
    return q, s_row, s_k


def quant_weight(w_bf16: np.ndarray):
    """bf16 bits [N,K] -> (wq [N,K] u8, w_scale [N/128, K/128] f32)."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    n, k = w.shape
    if n % GROUP or k % GROUP:
        raise ValueError("n and k must be multiples of 128")
    wq = np.empty((n, k), np.uint8)
    ws = np.empty((n // GROUP, k // GROUP), np.float32)
    rc = _load().oracle_quant_weight(_ptr(w), n, k, _ptr(wq), _ptr(ws))
    assert rc == 0
    return wq, ws


def quant_weight_rowwise(w_bf16: np.ndarray):
    """bf16 bits [N,K] -> (wq [N,K] u8, w_scale [N] f32), one scale per row."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    n, k = w.shape
    wq = np.empty((n, k), np.uint8)
    ws = np.empty((n,), np.float32)
    rc = _load().oracle_quant_weight_rowwise(_ptr(w), n, k, _ptr(wq), _ptr(ws))
    assert rc == 0
    return wq, ws


def gemm_ref(q: np.ndarray, a_scale_row: np.ndarray, wq: np.ndarray, w_scale: np.ndarray,
             rows: np.ndarray | None = None, threads: int = 1) -> np.ndarray:
    """Float64 reference Y[rows, N] of the block-scaled GEMM.

    ``a_scale_row`` is the row-major [M, K/128] activation scale. The weight
    scale is either block-scaled [N/128, K/128] or per row [N] (its shape
    selects the geometry). ``rows`` selects output rows (default: all).
    ``threads`` > 1 splits the rows over Python threads; the C loop itself
    is unchanged.
    """
    lib = _load()
    q = np.ascontiguousarray(q, dtype=np.uint8)
    a_s = np.ascontiguousarray(a_scale_row, dtype=np.float32)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    ws = np.ascontiguousarray(w_scale, dtype=np.float32)
    m, k = q.shape
    n = wq.shape[0]
    assert wq.shape[1] == k and a_s.shape == (m, k // GROUP)
    if ws.shape == (n,):
        block_n, block_k = 1, k
    else:
        assert ws.shape == (n // GROUP, k // GROUP)
        block_n, block_k = GROUP, GROUP
    if rows is None:
        rows_arr = np.arange(m, dtype=np.int64)
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        assert rows_arr.size == 0 or (rows_arr.min() >= 0 and rows_arr.max() < m)
    cnt = rows_arr.size
    ref = np.empty((cnt, n), np.float64)
    args = (_ptr(q), _ptr(a_s), _ptr(wq), _ptr(ws), n, k, block_n, block_k, _ptr(rows_arr))
    if threads <= 1 or cnt <= 1:
        lib.oracle_gemm_ref_rows_geom(*args, 0, cnt, _ptr(ref))
    else:
        bounds = np.linspace(0, cnt, min(threads, cnt) + 1).astype(int)
        with ThreadPoolExecutor(len(bounds) - 1) as ex:
            futs = [ex.submit(lib.oracle_gemm_ref_rows_geom, *args, int(a), int(b - a), _ptr(ref))
                    for a, b in zip(bounds[:-1], bounds[1:])]
            for f in futs:
                f.result()
    return ref


def check_tolerance(y_bf16: np.ndarray, ref: np.ndarray):
    """Return (number of failing elements, worst err/bound ratio) for
    |y-ref| <= 8e-3|ref| + 1e-3 rms(ref)."""
    y = np.ascontiguousarray(y_bf16, dtype=np.uint16).ravel()
    r = np.ascontiguousarray(ref, dtype=np.float64).ravel()
    assert y.size == r.size
    worst = ctypes.c_double(0.0)
    bad = _load().oracle_check_tolerance(_ptr(y), _ptr(r), y.size, ctypes.byref(worst))
    return int(bad), float(worst.value)


# ------------------------------------------------------------ dense FFN --

def silu_mul_bf16(gate_bf16: np.ndarray, up_bf16: np.ndarray) -> np.ndarray:
    """h = bf16_rne(silu(gate) * up), elementwise over bf16 bit arrays."""
    g = np.ascontiguousarray(gate_bf16, dtype=np.uint16)
    u = np.ascontiguousarray(up_bf16, dtype=np.uint16)
    assert g.shape == u.shape
    h = np.empty(g.shape, np.uint16)
    _load().oracle_silu_mul_bf16_array(_ptr(g), _ptr(u), g.size, _ptr(h))
    return h


def round_bf16(v: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits, round to nearest, ties to even."""
    a = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(a.shape, np.uint16)
    _load().oracle_round_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


def silu_mul_quant(gate_bf16: np.ndarray, up_bf16: np.ndarray):
    """bf16 bits gate, up [M, I] -> quant_act(silu(gate) * up) as
    (q [M,I] u8, s_row [M,I/128] f32, s_kmajor [I/128, ceil16(M)] f32)."""
    g = np.ascontiguousarray(gate_bf16, dtype=np.uint16)
    u = np.ascontiguousarray(up_bf16, dtype=np.uint16)
    assert g.shape == u.shape and g.ndim == 2
    m, i = g.shape
    if i % GROUP:
        raise ValueError("the intermediate width must be a multiple of 128")
    q = np.empty((m, i), np.uint8)
    s_row = np.empty((m, i // GROUP), np.float32)
    s_k = np.empty((i // GROUP, m_pad(m)), np.float32)
    rc = _load().oracle_silu_mul_quant(_ptr(g), _ptr(u), i, m, i, _ptr(q), _ptr(s_row), _ptr(s_k))
    assert rc == 0
    return q, s_row, s_k


def silu_mul_quant_stacked(gate_up_bf16: np.ndarray):
    """silu_mul_quant over the two halves of one [M, 2I] array (gate columns
    first), read in place with row stride 2I."""
    gu = np.ascontiguousarray(gate_up_bf16, dtype=np.uint16)
    m, two_i = gu.shape
    i = two_i // 2
    if i % GROUP or two_i != 2 * i:
        raise ValueError("the intermediate width must be a multiple of 128")
    q = np.empty((m, i), np.uint8)
    s_row = np.empty((m, i // GROUP), np.float32)
    s_k = np.empty((i // GROUP, m_pad(m)), np.float32)
    lib = _load()
    up = ctypes.c_void_p(gu.ctypes.data + 2 * i)  # bytes to the first up column
    rc = lib.oracle_silu_mul_quant(_ptr(gu), up, two_i, m, i, _ptr(q), _ptr(s_row), _ptr(s_k))
    assert rc == 0
    return q, s_row, s_k


def ffn_ref(x_bf16: np.ndarray, wq_gate_up: np.ndarray, ws_gate_up: np.ndarray,
            wq_down: np.ndarray, ws_down: np.ndarray, threads: int = 1) -> dict:
    """The dense FFN, each stage by its definition:
        q_x, s_x  = quant_act(x)                           (once, for both)
        gate, up  = bf16(gemm_ref(q_x, W_gate)), bf16(gemm_ref(q_x, W_up))
        q_h, s_h  = quant_act(bf16(silu(gate) * up))
        y         = gemm_ref(q_h, W_down)                  (float64)
    The gate and up weights are one [2I, D] matrix, gate rows first.
    Returns every stage in a dict."""
    q_x, s_x, _ = quant_act(x_bf16)
    gu = gemm_ref(q_x, s_x, wq_gate_up, ws_gate_up, threads=threads)
    i = wq_gate_up.shape[0] // 2
    gate = round_bf16(gu[:, :i])
    up = round_bf16(gu[:, i:])
    q_h, s_h, s_h_k = silu_mul_quant(gate, up)
    y = gemm_ref(q_h, s_h, wq_down, ws_down, threads=threads)
    return {"q_x": q_x, "s_x": s_x, "gate": gate, "up": up,
            "q_h": q_h, "s_h": s_h, "s_h_kmajor": s_h_k, "y": y}


# ------------------------------------------------ FP8 weight back to bf16 --

def dequant_fp8_bf16(wq: np.ndarray, w_scale: np.ndarray) -> np.ndarray:
    """e4m3 codes [N,K] and their fp32 scales -> bf16 bits [N,K], each the
    bf16 nearest to code * scale. The scale's shape selects the geometry:
    [N/128, K/128] (128x128 blocks) or [N] (one per row)."""
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    ws = np.ascontiguousarray(w_scale, dtype=np.float32)
    n, k = wq.shape
    if ws.shape == (n,):
        block_n, block_k = 1, k
    else:
        assert ws.shape == (n // GROUP, k // GROUP)
        block_n, block_k = GROUP, GROUP
    out = np.empty((n, k), np.uint16)
    rc = _load().oracle_dequant_fp8_bf16(_ptr(wq), _ptr(ws), n, k, block_n, block_k, _ptr(out))
    assert rc == 0
    return out


# ---------------------------------------------------------------- NVFP4 --

NVFP4_BLOCK = 16


def e2m1_decode(code: int) -> float:
    return float(_load().oracle_e2m1_decode(int(code)))


def e2m1_encode(t: float) -> int:
    return int(_load().oracle_e2m1_encode(float(t)))


def e2m1_encode_array(t: np.ndarray) -> np.ndarray:
    """Encode each fp32 value with the scalar E2M1 encoder (for sweeps)."""
    t = np.ascontiguousarray(t, dtype=np.float32).ravel()
    out = np.empty(t.size, np.uint8)
    _load().oracle_e2m1_encode_array(_ptr(t), t.size, _ptr(out))
    return out


def nvfp4_quant(x_bf16: np.ndarray, s2: float = 1.0):
    """bf16 bits [R,K] -> (q [R,K/2] u8, two E2M1 codes a byte with the even
    K index in the low nibble; sf [R,K/16] u8 E4M3 block scales), packed with
    second-level scale s2."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    r, k = x.shape
    if k % NVFP4_BLOCK:
        raise ValueError("k must be a multiple of 16")
    q = np.empty((r, k // 2), np.uint8)
    sf = np.empty((r, k // NVFP4_BLOCK), np.uint8)
    rc = _load().oracle_nvfp4_quant(_ptr(x), r, k, float(s2), _ptr(q), _ptr(sf))
    if rc != 0:
        raise ValueError("s2 must be a positive, finite fp32 value")
    return q, sf


def nvfp4_global_scale(x_bf16: np.ndarray) -> float:
    """max(amax, 1e-10) / 2688 in fp32: the second-level scale of a synthetic
    NVFP4 checkpoint weight."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    return float(_load().oracle_nvfp4_global_scale(_ptr(x), x.size))


def nvfp4_gemm_ref(qa: np.ndarray, sfa: np.ndarray, s2a: float, qw: np.ndarray, sfw: np.ndarray,
                   s2w: float, rows: np.ndarray | None = None) -> np.ndarray:
    """Float64 reference Y[rows, N] of the NVFP4 projection, operands as
    nvfp4_quant returns them."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    sfa = np.ascontiguousarray(sfa, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sfw = np.ascontiguousarray(sfw, dtype=np.uint8)
    m, half_k = qa.shape
    k = 2 * half_k
    n = qw.shape[0]
    assert qw.shape == (n, half_k) and sfa.shape == (m, k // NVFP4_BLOCK) and sfw.shape == (n, k // NVFP4_BLOCK)
    if rows is None:
        rows_arr = np.arange(m, dtype=np.int64)
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        assert rows_arr.size == 0 or (rows_arr.min() >= 0 and rows_arr.max() < m)
    ref = np.empty((rows_arr.size, n), np.float64)
    _load().oracle_nvfp4_gemm_ref_rows(_ptr(qa), _ptr(sfa), float(s2a), _ptr(qw), _ptr(sfw), float(s2w),
                                       n, k, _ptr(rows_arr), 0, rows_arr.size, _ptr(ref))
    return ref
