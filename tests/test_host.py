"""Host-side logic of libfp8q.so, exercised without a GPU.

Covers: every symbol declared in include/fp8q.h is exported and bound; the
CTA-floor function reproduces the worked table of the page
"spark_model/layers/ops/fp8_act_quant_floor.rs" and the sign of its fifteen
measured arms; the pick keeps kernel and grid together; argument checks
return their status before anything touches a device.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from conftest import ROOT, golden_rows
from fp8_block_scaled_group_b200 import _lib, api

HEADER = os.path.join(ROOT, "include", "fp8q.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8q_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["fp8q_quant_act", "fp8q_gemm_blockscaled", "fp8q_linear", "fp8q_m_pad",
                 "fp8q_quant_pick", "fp8q_quant_weight", "fp8q_status_string"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_functions()
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"{name} has no ctypes binding"
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (fp8q_\w+)", out))
    assert set(names) <= exported
    assert set(_lib.SIGNATURES) == set(names)


def test_c_program_uses_the_abi(tmp_path):
    """include/fp8q.h compiles as pedantic C99, and a C program linked against
    libfp8q.so gets the same answers as the ctypes binding (tests/c_abi_host.c)."""
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path / "c_abi_host")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_host.c"),
                           "-L", lib_dir, "-lfp8q", f"-Wl,-rpath,{lib_dir}", "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"


def test_status_strings_and_version():
    lib = _lib.load()
    for code in range(0, 9):
        s = lib.fp8q_status_string(code).decode()
        assert s.startswith("FP8Q_")
    assert lib.fp8q_status_string(99).decode() == "FP8Q_ERR_UNKNOWN"
    assert b"sm_100a" in lib.fp8q_version()


@pytest.mark.parametrize("m,mp", [(0, 0), (1, 16), (15, 16), (16, 16), (17, 32), (25, 32), (1168, 1168),
                                  (4576, 4576), (4577, 4592)])
def test_m_pad(m, mp):
    assert api.m_pad(m) == mp


def test_floor_reproduces_the_pages_table():
    """sm_count 132, 8 K-groups per CTA, one token per CTA row, 2 CTAs per SM."""
    for k, g, grid_y, min_m in (map(int, r) for r in golden_rows("cta_floor_h100.txt")):
        assert k // 128 == g and -(-g // 8) == grid_y
        assert api.quant_floor_min_m(k, 132, 8, 1, 2) == min_m


def test_floor_reproduces_the_sign_of_fifteen_arms():
    """The arm the floor picks is the arm measured faster, at every one of the 15 arms."""
    rows = golden_rows("quant_arms_h100.txt")
    assert len(rows) == 15
    for m, k, faster in rows:
        m, k = int(m), int(k)
        picks_multi = m >= api.quant_floor_min_m(k, 132, 8, 1, 2)
        assert picks_multi == (faster == "multi"), (m, k)


def test_floor_rows_per_cta_generalisation():
    # min M with ceil(G/8) * ceil(M/rpc) >= ceil(f * sms), checked by brute force
    import math
    for k in [128, 512, 5120, 6144, 17408]:
        for sms in [1, 132, 148]:
            for rpc in [1, 2, 4]:
                for f in [2.0, 2.0 / 3.0, 0.5, 1.0]:
                    mm = api.quant_floor_min_m(k, sms, 8, rpc, f)
                    gy = -(-(k // 128) // 8)
                    floor = max(1, math.ceil(float(np.float32(f)) * sms - 1e-9))  # the ABI takes a float
                    ok = [m for m in range(1, 5000) if gy * -(-m // rpc) >= floor]
                    assert mm == ok[0], (k, sms, rpc, f)
    assert api.quant_floor_min_m(64, 148, 8, 1, 2) == 0
    assert api.quant_floor_min_m(5120, 148, 0, 1, 2) == 0
    assert api.quant_floor_min_m(5120, 148, 8, 1, float("nan")) == 0


def test_b200_floor_picks_the_faster_variant_at_decode_widths():
    """On 148 SMs the pick sends each decode arm to the variant that measured
    faster on B200 (fixture tests/golden/quant_arms_b200.txt)."""
    for m, k, faster in golden_rows("quant_arms_b200.txt"):
        p = api.quant_pick(int(m), int(k), 148)
        assert p.variant == (api.MULTI if faster == "multi" else api.SINGLE), (m, k)


FLOOR_CTAS_148 = 70  # ceil(0.47 * 148)


def test_pick_keeps_kernel_and_grid_together():
    # MULTI is the streaming kernel: one CTA per 16-group chunk, at most 3 per SM.
    for m in [1, 16, 17, 25, 53, 60, 100, 1168, 4576]:
        for k in [512, 5120, 6144, 17408]:
            auto = api.quant_pick(m, k, 148)
            g = k // 128
            chunks = -(-(m * g) // 16)
            grid = min(chunks, 3 * 148)
            assert auto.forced == 0
            assert auto.floor_ctas == FLOOR_CTAS_148
            assert auto.multi_ctas == grid
            assert auto.variant == (api.MULTI if grid >= FLOOR_CTAS_148 else api.SINGLE)
            single = api.quant_pick(m, k, 148, api.SINGLE)
            assert single.variant == api.SINGLE and single.forced == 1
            assert single.grid_x == m * g and single.block_x == 16 and single.groups_per_cta == 1
            multi = api.quant_pick(m, k, 148, api.MULTI)
            assert multi.variant == api.MULTI and multi.grid_x == grid and multi.block_x == 224
            assert multi.groups_per_cta == 16 * -(-chunks // grid)
            assert multi.groups_per_cta * multi.grid_x >= m * g


def test_pick_argument_errors():
    lib = _lib.load()
    out = _lib.QuantPick()
    assert lib.fp8q_quant_pick(16, 5120, 148, 0, None) == 1
    assert lib.fp8q_quant_pick(16, 5000, 148, 0, ctypes.byref(out)) == 2
    assert lib.fp8q_quant_pick(16, 5120, 0, 0, ctypes.byref(out)) == 8
    assert lib.fp8q_quant_pick(16, 5120, 148, 3, ctypes.byref(out)) == 8


def test_workspace_layout():
    for m, k in [(1, 128), (16, 512), (17, 5120), (25, 17408), (4576, 17408)]:
        off = api.linear_scale_offset(m, k)
        assert off >= m * k and off % 256 == 0
        assert api.linear_workspace_bytes(m, k) >= off + 4 * (k // 128) * api.m_pad(m)
        assert api.linear_workspace_bytes(m, k) % 256 == 0


# Argument checks come first, so these run without any device.
A = ctypes.c_void_p(0x10000)   # 16-byte aligned stand-ins, never dereferenced
B = ctypes.c_void_p(0x20000)
C = ctypes.c_void_p(0x30000)
D = ctypes.c_void_p(0x40000)
E = ctypes.c_void_p(0x50000)
ODD = ctypes.c_void_p(0x10008)


def test_quant_act_argument_errors():
    lib = _lib.load()
    assert lib.fp8q_quant_act(None, B, C, D, 16, 512, None) == 1
    assert lib.fp8q_quant_act(A, None, C, D, 16, 512, None) == 1
    assert lib.fp8q_quant_act(A, B, C, None, 16, 512, None) == 1
    assert lib.fp8q_quant_act(A, B, C, D, 16, 500, None) == 2
    assert lib.fp8q_quant_act(A, B, C, D, 16, 0, None) == 2
    assert lib.fp8q_quant_act(A, B, C, D, 1 << 20, 1 << 12, None) == 2
    assert lib.fp8q_quant_act(ODD, B, C, D, 16, 512, None) == 3
    assert lib.fp8q_quant_act(A, B, ODD, D, 16, 512, None) == 3
    assert lib.fp8q_quant_act_variant(A, B, C, D, 16, 512, 7, None) == 8
    assert lib.fp8q_quant_act(A, B, None, D, 0, 512, None) == 0  # M == 0: nothing to do
    assert lib.fp8q_quant_act(None, None, None, None, 0, 512, None) == 0
    assert lib.fp8q_quant_act(None, None, None, None, 0, 500, None) == 2


def test_gemm_and_linear_argument_errors():
    lib = _lib.load()
    assert lib.fp8q_gemm_blockscaled(None, B, C, D, E, 16, 256, 512, None) == 1
    assert lib.fp8q_gemm_blockscaled(A, B, C, D, None, 16, 256, 512, None) == 1
    assert lib.fp8q_gemm_blockscaled(None, None, None, None, None, 0, 256, 512, None) == 0
    assert lib.fp8q_gemm_blockscaled(A, B, C, D, E, 16, 200, 512, None) == 2
    assert lib.fp8q_gemm_blockscaled(A, B, C, D, E, 16, 256, 520, None) == 2
    assert lib.fp8q_gemm_blockscaled(A, B, C, D, ODD, 16, 256, 512, None) == 3
    assert lib.fp8q_gemm_blockscaled(A, B, C, D, E, 0, 256, 512, None) == 0
    need = lib.fp8q_linear_workspace_bytes(16, 512)
    ws = ctypes.c_void_p(0x100000)
    assert lib.fp8q_linear(A, B, C, D, None, need, 16, 256, 512, None) == 1
    assert lib.fp8q_linear(None, None, None, None, None, 0, 0, 256, 512, None) == 0
    assert lib.fp8q_linear(A, B, C, D, ws, need - 1, 16, 256, 512, None) == 4
    assert lib.fp8q_linear(A, B, C, D, ctypes.c_void_p(0x100010), need, 16, 256, 512, None) == 4
    assert lib.fp8q_linear(A, B, C, D, ws, need, 16, 256, 500, None) == 2
    assert lib.fp8q_linear(A, B, C, D, ws, need, 0, 256, 512, None) == 0
    assert lib.fp8q_quant_weight(A, B, None, 256, 512, None) == 1
    assert lib.fp8q_quant_weight(A, B, C, 200, 512, None) == 2
    assert lib.fp8q_quant_weight(ODD, B, C, 256, 512, None) == 3
    assert lib.fp8q_convert_e4m3(None, B, 4, None) == 1
    assert lib.fp8q_convert_e4m3(A, B, 0, None) == 0
    assert lib.fp8q_check_division(None, None) == 1


def test_silu_mul_quant_and_ffn_argument_errors():
    lib = _lib.load()
    # fp8q_silu_mul_quant(gate, up, ld, q, s_row, s_k, m, i, stream)
    assert lib.fp8q_silu_mul_quant(None, None, 128, None, None, None, 0, 128, None) == 0
    assert lib.fp8q_silu_mul_quant(A, B, 128, C, None, D, 1, 100, None) == 2
    assert lib.fp8q_silu_mul_quant(A, B, 64, C, None, D, 1, 128, None) == 2    # ld < i
    assert lib.fp8q_silu_mul_quant(A, B, 260, C, None, D, 1, 256, None) == 2   # ld not a multiple of 8
    assert lib.fp8q_silu_mul_quant(A, B, 256, C, None, None, 1, 256, None) == 1
    assert lib.fp8q_silu_mul_quant(ODD, B, 256, C, None, D, 1, 256, None) == 3
    assert lib.fp8q_silu_mul_quant(A, B, 1 << 16, C, None, D, 1 << 15, 256, None) == 2
    assert lib.fp8q_check_silu_mul(None, A, None) == 1
    # fp8q_ffn(x, w_gu, s_gu, w_dn, s_dn, y, ws, ws_bytes, m, d, i, stream)
    m, d, i = 17, 256, 384
    need = lib.fp8q_ffn_workspace_bytes(m, d, i)
    ws = ctypes.c_void_p(0x1000000)
    assert lib.fp8q_ffn(None, None, None, None, None, None, None, 0, 0, d, i, None) == 0
    assert lib.fp8q_ffn(A, B, C, D, E, A, ws, need, m, d, 100, None) == 2
    assert lib.fp8q_ffn(A, B, C, D, E, None, ws, need, m, d, i, None) == 1
    assert lib.fp8q_ffn(A, B, C, D, E, A, ws, need - 1, m, d, i, None) == 4
    assert lib.fp8q_ffn(A, B, C, D, E, A, ctypes.c_void_p(0x1000010), need, m, d, i, None) == 4
    assert lib.fp8q_ffn(A, B, C, D, ODD, A, ws, need, m, d, i, None) == 3
    # gate|up [m, 2i] past 2^31 elements, and a 2i that would wrap in 32 bits
    big_i = 1 << 30
    assert lib.fp8q_ffn(A, B, C, D, E, A, ws, 1 << 62, 2, d, big_i, None) == 2
    assert lib.fp8q_ffn(A, B, C, D, E, A, ws, 1 << 62, 1, d, (1 << 31) + 128, None) == 2


def test_nvfp4_argument_errors():
    lib = _lib.load()
    # fp8q_nvfp4_quant(x, q, sf_row, sf_mma, s2, rows, k, stream)
    assert lib.fp8q_nvfp4_quant(A, B, None, C, 1.0, 4, 0, None) == 2
    assert lib.fp8q_nvfp4_quant(A, B, None, C, 1.0, 4, 32, None) == 2
    for s2 in (0.0, -1.0, float("inf"), float("nan")):
        assert lib.fp8q_nvfp4_quant(A, B, None, C, s2, 4, 64, None) == 8
    assert lib.fp8q_nvfp4_quant(None, None, None, None, 1.0, 0, 64, None) == 0
    assert lib.fp8q_nvfp4_quant(None, B, None, C, 1.0, 4, 64, None) == 1
    assert lib.fp8q_nvfp4_quant(A, B, None, None, 1.0, 4, 64, None) == 1
    assert lib.fp8q_nvfp4_quant(ODD, B, None, C, 1.0, 4, 64, None) == 3
    assert lib.fp8q_nvfp4_quant(A, B, None, C, 1.0, 1 << 25, 64, None) == 2
    # fp8q_nvfp4_gemm(qa, sfa, s2a, qw, sfw, s2w, y, m, n, k, stream)
    assert lib.fp8q_nvfp4_gemm(A, B, 1.0, C, D, 1.0, E, 4, 256, 128, None) == 2    # k % 256
    assert lib.fp8q_nvfp4_gemm(A, B, 1.0, C, D, 1.0, E, 4, 64, 256, None) == 2     # n % 128
    assert lib.fp8q_nvfp4_gemm(A, B, 0.0, C, D, 1.0, E, 4, 256, 256, None) == 8
    assert lib.fp8q_nvfp4_gemm(A, B, 1.0, C, D, float("nan"), E, 4, 256, 256, None) == 8
    assert lib.fp8q_nvfp4_gemm(None, None, 1.0, None, None, 1.0, None, 0, 256, 256, None) == 0
    assert lib.fp8q_nvfp4_gemm(A, None, 1.0, C, D, 1.0, E, 4, 256, 256, None) == 1
    assert lib.fp8q_nvfp4_gemm(A, B, 1.0, C, ODD, 1.0, E, 4, 256, 256, None) == 3
    assert lib.fp8q_nvfp4_gemm(A, B, 1.0, C, D, 1.0, E, 1 << 23, 256, 256, None) == 2
    # fp8q_nvfp4_linear(x, s2a, qw, sfw, s2w, y, ws, ws_bytes, m, n, k, stream)
    m, n, k = 17, 256, 512
    need = lib.fp8q_nvfp4_linear_workspace_bytes(m, k)
    ws = ctypes.c_void_p(0x1000000)
    assert lib.fp8q_nvfp4_linear(A, 1.0, C, D, 1.0, E, ws, need, m, n, 320, None) == 2
    assert lib.fp8q_nvfp4_linear(A, -2.0, C, D, 1.0, E, ws, need, m, n, k, None) == 8
    assert lib.fp8q_nvfp4_linear(None, 1.0, None, None, 1.0, None, None, 0, 0, n, k, None) == 0
    assert lib.fp8q_nvfp4_linear(A, 1.0, C, D, 1.0, None, ws, need, m, n, k, None) == 1
    assert lib.fp8q_nvfp4_linear(A, 1.0, C, D, 1.0, E, ws, need - 1, m, n, k, None) == 4
    assert lib.fp8q_nvfp4_linear(A, 1.0, C, D, 1.0, E, ctypes.c_void_p(0x1000010), need, m, n, k, None) == 4
    assert lib.fp8q_nvfp4_linear(ODD, 1.0, C, D, 1.0, E, ws, need, m, n, k, None) == 3
    # fp8q_dequant_fp8_bf16(wq, w_scale, format, y, n, k, stream)
    assert lib.fp8q_dequant_fp8_bf16(A, B, 2, C, 128, 128, None) == 8
    assert lib.fp8q_dequant_fp8_bf16(A, B, 0, C, 128, 100, None) == 2
    assert lib.fp8q_dequant_fp8_bf16(A, B, 0, C, 100, 128, None) == 2     # 128 x 128 blocks need n % 128
    assert lib.fp8q_dequant_fp8_bf16(A, None, 1, C, 100, 128, None) == 1  # per row: any n
    assert lib.fp8q_dequant_fp8_bf16(A, B, 1, ODD, 100, 128, None) == 3
    assert lib.fp8q_dequant_fp8_bf16(A, B, 1, C, 1 << 24, 128, None) == 2
    assert lib.fp8q_convert_e2m1(None, B, 4, None) == 1
    assert lib.fp8q_convert_e2m1(A, B, 0, None) == 0


def test_nvfp4_sizes():
    lib = _lib.load()
    for rows, k in [(1, 64), (17, 512), (128, 256), (129, 5120), (1168, 5120), (17408, 5120)]:
        pad = (rows + 127) // 128 * 128
        assert lib.fp8q_nvfp4_sf_mma_bytes(rows, k) == pad * k // 16
        up = lambda v: (v + 255) // 256 * 256
        assert lib.fp8q_nvfp4_linear_workspace_bytes(rows, k) == up(rows * k // 2) + up(pad * k // 16)


def test_ffn_workspace_layout():
    for m, d, i in [(1, 128, 128), (17, 256, 384), (25, 5120, 17408), (1168, 5120, 17408)]:
        off = api.ffn_workspace_layout(m, d, i)
        mp = api.m_pad(m)
        sizes = [m * d, 4 * (d // 128) * mp, 2 * m * 2 * i, m * i, 4 * (i // 128) * mp]
        for k in range(5):
            assert off[k] % 256 == 0 and off[k + 1] >= off[k] + sizes[k]
        assert api.ffn_workspace_layout(m, d, i)[5] == _lib.load().fp8q_ffn_workspace_bytes(m, d, i)
    assert _lib.load().fp8q_ffn_workspace_bytes(1, 100, 128) == 0


def test_no_device_reports_cuda_error_not_crash():
    """With valid arguments and no usable device, calls fail with a status."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    lib = _lib.load()
    assert lib.fp8q_quant_act(A, B, C, D, 16, 512, None) in (5, 7)
    code = ctypes.c_uint32(0)
    assert lib.fp8q_device_error(None, ctypes.byref(code)) in (5, 7)


def test_cpu_baseline_sample_sizing():
    """bench.grow_sample: the CPU oracle baseline times about target seconds
    of work (or the whole step), refining a small first probe's estimate."""
    import bench

    calls = []

    def fake(per_row, fixed=0.3):
        def run(rows):
            calls.append(rows)
            return fixed + rows * per_row
        return run

    rows, t = bench.grow_sample(fake(0.01), 1168, 16, 10.0)
    assert calls[0] == 16 and rows % 16 == 0 and 8.0 <= t and len(calls) <= 4
    calls.clear()
    rows, t = bench.grow_sample(fake(0.01), 100, 16, 10.0)     # the whole step takes less than the target
    assert rows == 100 and calls == [16, 100]
    calls.clear()
    rows, t = bench.grow_sample(fake(1.0), 1168, 16, 10.0)      # the probe alone exceeds the target
    assert rows == 16 and calls == [16]


def test_kernel_digest_ignores_comments_only():
    """bench.strip_comments: the traffic records stay keyed to a kernel's code,
    not to its comments; any code change moves the digest."""
    import bench

    code = "int f(int a) {\n  return a + 1;  // one more\n}\n/* block\n comment */ int g;\n"
    assert bench.strip_comments(code) == "int f(int a) { return a + 1; } int g;"
    assert bench.strip_comments(code.replace("one more", "add one")) == bench.strip_comments(code)
    assert bench.strip_comments(code.replace("a + 1", "a + 2")) != bench.strip_comments(code)
    for kernel in bench.KERNEL_SOURCES:
        assert len(bench.kernel_digest(kernel)) == 16
