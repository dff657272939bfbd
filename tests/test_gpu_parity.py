"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

FP8 bytes and both scale layouts: bit-exact. GEMM outputs: every compared
element satisfies |y - ref| <= 8e-3 |ref| + 1e-3 rms(ref) against the
float64 dequantized reference. Full workload sizes are checked on sampled
rows (first, last, M-1 and random rows; rms over the sampled rows).
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from fp8_block_scaled_group_b200 import api, inputs

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
GUARD = 4096  # bytes of sentinel after each output buffer


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def guarded(nbytes: int, dtype, shape):
    """A device buffer with GUARD sentinel bytes after the payload."""
    el = torch.empty((), dtype=dtype).element_size()
    raw = torch.full((nbytes + GUARD,), 0xA5, dtype=torch.uint8, device=DEV)
    view = raw[:nbytes].view(dtype).view(shape)
    return raw, view


def guard_intact(raw: torch.Tensor, nbytes: int) -> bool:
    return bool((raw[nbytes:] == 0xA5).all().item())


@functools.lru_cache(maxsize=None)
def oracle_act(m, k, seed, p, sigma):
    xb = inputs.activations(m, k, seed, p, sigma)
    q, s_row, s_k = oracle.quant_act(xb)
    return xb, q, s_row, s_k


@functools.lru_cache(maxsize=None)
def oracle_w(n, k, seed):
    wb = inputs.weights(n, k, seed)
    wq, ws = oracle.quant_weight(wb)
    return wb, wq, ws


def run_quant(xb, variant):
    m, k = xb.shape
    g, mp = k // 128, api.m_pad(m)
    x = to_dev_bf16(xb)
    q_raw, q = guarded(m * k, torch.uint8, (m, k))
    r_raw, s_row = guarded(4 * m * g, torch.float32, (m, g))
    k_raw, s_k = guarded(4 * g * mp, torch.float32, (g, mp))
    api.quant_act(x, variant=variant, out=(q, s_row, s_k))
    torch.cuda.synchronize()
    assert guard_intact(q_raw, m * k) and guard_intact(r_raw, 4 * m * g) and guard_intact(k_raw, 4 * g * mp)
    return q.cpu().numpy(), s_row.cpu().numpy(), s_k.cpu().numpy()


def assert_quant_equal(got, want):
    q, s_row, s_k = got
    q_o, s_row_o, s_k_o = want
    assert np.array_equal(q, q_o), f"{int((q != q_o).sum())} FP8 bytes differ"
    assert np.array_equal(s_row.view(np.uint32), s_row_o.view(np.uint32)), "row-major scales differ"
    assert np.array_equal(s_k.view(np.uint32), s_k_o.view(np.uint32)), "K-major scales differ"


WORKLOADS = inputs.all_workloads()


@pytest.mark.parametrize("wl", WORKLOADS, ids=[w.name for w in WORKLOADS])
@pytest.mark.parametrize("variant", [api.SINGLE, api.MULTI, api.AUTO], ids=["single", "multi", "auto"])
def test_quant_act_bitexact_workloads(wl, variant):
    xb, q, s_row, s_k = oracle_act(wl.m, wl.k, wl.seed, wl.outlier_p, wl.outlier_sigma)
    assert_quant_equal(run_quant(xb, variant), (q, s_row, s_k))


@pytest.mark.parametrize("m", [1, 2, 15, 16, 17, 31, 33, 129, 300])
@pytest.mark.parametrize("k", [128, 256, 1152, 2176])
@pytest.mark.parametrize("variant", [api.SINGLE, api.MULTI])
def test_quant_act_bitexact_edges(m, k, variant):
    xb = inputs.activations(m, k, seed=7 * m + k, outlier_p=0.02, outlier_sigma=30.0)
    assert_quant_equal(run_quant(xb, variant), oracle.quant_act(xb))


def special_rows():
    rows = []
    z = np.zeros(128, np.float32)
    rows.append(z)                                                   # all zero
    neg = -np.zeros(128, np.float32)
    rows.append(neg)                                                 # all -0.0
    r = z.copy(); r[5] = -37.5; rows.append(r)                       # single outlier
    r = z.copy(); r[:9] = [56, -56, 28, 2**-12, -2**-12, 2**-13, 3 * 2**-13, 1, 0]; rows.append(r)
    r = z.copy(); r[:3] = [448, -2**-11, 2**-11]; rows.append(r)     # negative tiny keeps its sign
    r = np.linspace(-3, 3, 128).astype(np.float32); rows.append(r)
    r = np.full(128, 1e-38, np.float32); r[::2] *= -1; rows.append(r)  # near fp32 min normal
    r = np.full(128, 3.0e38, np.float32); r[1::3] = -1.0; rows.append(r)  # huge amax
    bits = [inputs.f32_to_bf16_bits(r) for r in rows]
    sub = np.full(128, 0x0001, np.uint16); sub[1::2] = 0x8001; bits.append(sub)   # bf16 subnormals
    # amax values whose fp32 quotient amax/(amax/448) exceeds 448 (saturation path)
    hs = np.arange(0x3F80, 0x4780, dtype=np.uint16)
    a = inputs.bf16_bits_to_f32(hs)
    over = hs[(a / (a / np.float32(448.0))) > np.float32(448.0)]
    for h in over[:8]:
        s = np.zeros(128, np.uint16); s[0] = h; s[7] = h | 0x8000; s[8:16] = 0x3F80
        bits.append(s)
    return np.stack(bits)


@pytest.mark.parametrize("variant", [api.SINGLE, api.MULTI])
def test_quant_act_special_groups(variant):
    sp = special_rows()                       # [R, 128]
    xb = np.ascontiguousarray(np.tile(sp.reshape(1, -1), (3, 1)))  # 3 tokens x R groups
    got = run_quant(xb, variant)
    assert_quant_equal(got, oracle.quant_act(xb))
    assert not np.any((got[0] & 0x7F) == 0x7F), "NaN code emitted"


def test_quant_act_m_zero_touches_nothing():
    x = torch.zeros((0, 512), dtype=torch.bfloat16, device=DEV)
    q = torch.full((16,), 0x5A, dtype=torch.uint8, device=DEV)
    s = torch.full((16,), 7.0, dtype=torch.float32, device=DEV)
    api.quant_act(x, out=(q[:0].view(0, 512), None, s[:0].view(4, 0)))
    torch.cuda.synchronize()
    assert (q == 0x5A).all() and (s == 7.0).all()


def test_convert_matches_oracle_encoder_exhaustively():
    """Every fp32 bit pattern except the NaNs (both zeros, subnormals, normals,
    +-Inf): the hardware e4m3 conversion the kernels use gives the oracle
    encoder's code."""
    step = 1 << 25
    for lo, hi in ((0x00000000, 0x7F800000), (0x80000000, 0xFF800000)):  # +0 .. +Inf, -0 .. -Inf
        for start in range(lo, hi + 1, step):
            pats = np.arange(start, min(start + step, hi + 1), dtype=np.uint32)
            v = pats.view(np.float32)
            got = api.convert_e4m3(torch.from_numpy(v).to(DEV)).cpu().numpy()
            want = oracle.e4m3_encode_array(v)
            assert np.array_equal(got, want), hex(start)


def test_division_exhaustive_against_ieee():
    """The quantizers' reciprocal-plus-correction division gives the code of the
    IEEE quotient for every (x, amax) pair of bf16 values with |x| <= amax."""
    pairs, code_bad, quot_bad, scale_bad = api.check_division()
    assert pairs == 0x7F80 * 0x7F81
    assert scale_bad == 0, "a group scale or its reciprocal differs from IEEE division"
    assert code_bad == 0
    print(f"division check: {pairs} pairs, {code_bad} code mismatches, {quot_bad} quotient mismatches")


@pytest.mark.parametrize("n,k", [(512, 512), (256, 384), (6144, 5120), (5120, 17408)])
def test_quant_weight_bitexact(n, k):
    wb, wq_o, ws_o = oracle_w(n, k, 1000 + n % 7)
    wq, ws = api.quant_weight(to_dev_bf16(wb))
    torch.cuda.synchronize()
    assert np.array_equal(wq.cpu().numpy(), wq_o)
    assert np.array_equal(ws.cpu().numpy().view(np.uint32), ws_o.view(np.uint32))


# --------------------------------------------------------------- GEMM --

def sample_rows(m, count=64, seed=0):
    if m <= count:
        return np.arange(m, dtype=np.int64)
    rng = np.random.default_rng(seed)
    fixed = {0, m - 1, m - 2, 127 % m, 128 % m}
    rest = rng.choice(m, size=count, replace=False)
    rows = sorted(fixed | set(int(r) for r in rest))
    return np.array(rows[:max(count, len(fixed))], dtype=np.int64)


def gemm_case(m, n, k, seed, p=0.01, sigma=20.0, rows=None, threads=8):
    xb, q, s_row, s_k = oracle_act(m, k, seed, p, sigma)
    wb, wq_o, ws_o = oracle_w(n, k, seed)
    q_d = torch.from_numpy(q).to(DEV)
    sk_d = torch.from_numpy(s_k).to(DEV)
    wq_d = torch.from_numpy(wq_o).to(DEV)
    ws_d = torch.from_numpy(ws_o).to(DEV)
    y_raw, y = guarded(2 * m * n, torch.bfloat16, (m, n))
    api.gemm_blockscaled(q_d, sk_d, wq_d, ws_d, out=y)
    torch.cuda.synchronize()
    assert guard_intact(y_raw, 2 * m * n), "GEMM wrote past its output"
    yb = bf16_bits(y)
    rows = np.arange(m, dtype=np.int64) if rows is None else rows
    ref = oracle.gemm_ref(q, s_row, wq_o, ws_o, rows=rows, threads=threads)
    bad, worst = oracle.check_tolerance(yb[rows], ref)
    return bad, worst, yb, (xb, q, s_row, s_k, wq_o, ws_o)


@pytest.mark.parametrize("m,n,k", [(1, 128, 128), (16, 512, 512), (17, 128, 640), (100, 256, 256),
                                   (128, 384, 384), (129, 128, 1024), (200, 640, 896), (256, 256, 2048),
                                   # 64-token decode tiles, and the first width on the pair kernel
                                   (33, 256, 512), (48, 1024, 3072), (64, 384, 1152), (65, 256, 256)])
def test_gemm_edges_full(m, n, k):
    bad, worst, _, _ = gemm_case(m, n, k, seed=m + n + k)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


@pytest.mark.parametrize("wl", [w for w in WORKLOADS if w.number in (1, 2, 3)], ids=lambda w: w.name)
def test_gemm_workloads_full(wl):
    bad, worst, _, _ = gemm_case(wl.m, wl.n, wl.k, wl.seed, wl.outlier_p, wl.outlier_sigma)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


@pytest.mark.parametrize("wl", [w for w in WORKLOADS if w.number in (4, 5)], ids=lambda w: w.name)
def test_gemm_workloads_sampled(wl):
    rows = sample_rows(wl.m, 48, seed=wl.seed)
    bad, worst, _, _ = gemm_case(wl.m, wl.n, wl.k, wl.seed, wl.outlier_p, wl.outlier_sigma, rows=rows)
    assert bad == 0, f"{bad} elements out of tolerance (worst {worst:.3f})"


def test_gemm_integer_case_exact():
    """Unit scales and small-integer codes: every partial sum is an exact
    integer well inside fp32 and bf16, so the output is exact."""
    rng = np.random.default_rng(1)
    ints = np.array([-2, -1, 0, 1, 2], np.int64)
    code = {v: oracle.e4m3_encode(float(v)) for v in ints.tolist()}
    m, n, k = 40, 256, 512
    ia = rng.choice(ints, size=(m, k))
    ib = rng.choice(ints, size=(n, k))
    ia[:, 1:] = 0  # keep |sums| small enough for bf16 to hold them exactly
    qa = np.vectorize(code.get)(ia).astype(np.uint8)
    qb = np.vectorize(code.get)(ib).astype(np.uint8)
    mp = api.m_pad(m)
    sk = np.zeros((k // 128, mp), np.float32)
    sk[:, :m] = 1.0
    y = api.gemm_blockscaled(torch.from_numpy(qa).to(DEV), torch.from_numpy(sk).to(DEV),
                             torch.from_numpy(qb).to(DEV), torch.ones((n // 128, k // 128), device=DEV))
    torch.cuda.synchronize()
    assert np.array_equal(y.float().cpu().numpy(), (ia @ ib.T).astype(np.float32))


def test_gemm_wrong_scale_layout_fails():
    """Negative control: the row-major scales read as K-major (the reading the
    page "dispatch_proj.rs" measured at rel_rms 7.7e-2) must fail the check."""
    m, n, k = 25, 512, 1024
    xb, q, s_row, s_k = oracle_act(m, k, 31, 0.01, 20.0)
    wb, wq_o, ws_o = oracle_w(n, k, 31)
    g, mp = s_k.shape
    flat = np.zeros(g * mp, np.float32)
    flat[:m * g] = s_row.ravel()
    y = api.gemm_blockscaled(torch.from_numpy(q).to(DEV), torch.from_numpy(flat.reshape(g, mp)).to(DEV),
                             torch.from_numpy(wq_o).to(DEV), torch.from_numpy(ws_o).to(DEV))
    torch.cuda.synchronize()
    ref = oracle.gemm_ref(q, s_row, wq_o, ws_o)
    bad, _ = oracle.check_tolerance(bf16_bits(y), ref)
    assert bad > 0


# ------------------------------------------------------------- linear --

@pytest.mark.parametrize("m,n,k", [(16, 512, 512), (25, 6144, 5120), (1, 256, 17408), (17, 5120, 17408),
                                   (32, 256, 640), (31, 128, 1152), (33, 256, 640), (300, 384, 1024)])
def test_linear_matches_quant_then_gemm(m, n, k):
    xb, q, s_row, s_k = oracle_act(m, k, 77, 0.01, 20.0)
    wb, wq_o, ws_o = oracle_w(n, k, 77)
    x = to_dev_bf16(xb)
    wq_d = torch.from_numpy(wq_o).to(DEV)
    ws_d = torch.from_numpy(ws_o).to(DEV)
    need = api.linear_workspace_bytes(m, k)
    ws_raw, workspace = guarded(need, torch.uint8, (need,))
    y = api.linear(x, wq_d, ws_d, workspace=workspace)
    q2, _, sk2 = api.quant_act(x, row_major=False)
    y2 = api.gemm_blockscaled(q2, sk2, wq_d, ws_d)
    torch.cuda.synchronize()
    assert guard_intact(ws_raw, need)
    w = workspace.cpu().numpy()
    off = api.linear_scale_offset(m, k)
    g, mp = k // 128, api.m_pad(m)
    assert np.array_equal(w[:m * k].reshape(m, k), q)
    assert np.array_equal(w[off:off + 4 * g * mp].view(np.uint32).reshape(g, mp), s_k.view(np.uint32))
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    rows = sample_rows(m, 32)
    ref = oracle.gemm_ref(q, s_row, wq_o, ws_o, rows=rows, threads=8)
    bad, worst = oracle.check_tolerance(bf16_bits(y)[rows], ref)
    assert bad == 0, worst


@pytest.mark.parametrize("m,n,k", [(1, 256, 17408), (16, 512, 512), (17, 5120, 17408), (25, 6144, 5120),
                                   (31, 128, 1152), (32, 256, 640)])
@pytest.mark.parametrize("per_row", [False, True], ids=["block128", "per_row"])
def test_linear_decode_fused_is_linear(m, n, k, per_row):
    """The one-launch decode path: same y bits, same workspace bytes."""
    xb, q, s_row, s_k = oracle_act(m, k, 91, 0.01, 20.0)
    wb = inputs.weights(n, k, 91)
    wq_o, ws_o = oracle.quant_weight_rowwise(wb) if per_row else oracle.quant_weight(wb)
    x = to_dev_bf16(xb)
    wq_d = torch.from_numpy(wq_o).to(DEV)
    ws_d = torch.from_numpy(ws_o).to(DEV)
    need = api.linear_workspace_bytes(m, k)
    ws_raw, workspace = guarded(need, torch.uint8, (need,))
    y = api.linear_decode_fused(x, wq_d, ws_d, workspace=workspace)
    y2 = api.linear(x, wq_d, ws_d)
    torch.cuda.synchronize()
    assert guard_intact(ws_raw, need)
    w = workspace.cpu().numpy()
    off = api.linear_scale_offset(m, k)
    g, mp = k // 128, api.m_pad(m)
    assert np.array_equal(w[:m * k].reshape(m, k), q)
    assert np.array_equal(w[off:off + 4 * g * mp].view(np.uint32).reshape(g, mp), s_k.view(np.uint32))
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_linear_decode_fused_rejects_wide_m():
    a = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    st = api._lib.load().fp8q_linear_decode_fused(api._p(a), api._p(a), api._p(a), 0, api._p(a), api._p(a),
                                                  a.numel(), 33, 128, 128, None)
    assert st == 2


def test_no_device_error_flag():
    assert api.device_error() == 0
