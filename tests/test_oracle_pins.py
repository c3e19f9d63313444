"""Pins of the fp64 oracle against things other than itself (no GPU).

Each check ties one oracle routine to a library routine, a closed form from
mathematics, an invariant, a brute force on tiny inputs, or a value the pages
print (fixtures under tests/golden/).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _torch_e4m3(codes: np.ndarray) -> np.ndarray:
    """Library decode of e4m3fn codes (torch CPU)."""
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def _torch_e8m0(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(
        torch.float8_e8m0fnu).to(torch.float64).numpy()


def _all_bf16_finite() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return bits[np.isfinite(f)].astype(np.uint16)


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---- codecs -----------------------------------------------------------------

def test_e4m3_decode_all_256_codes(oracle_mod):
    got = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    want = _torch_e4m3(np.arange(256))
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9
    assert math.copysign(1.0, got[0x80]) == -1.0 and got[0x80] == 0.0


def test_e2m1_decode_all_16_codes(oracle_mod):
    # Every e2m1 value is exact in e4m3: re-encode the bit fields into an e4m3
    # pattern (exponent bias 1 -> 7, mantissa bit -> top mantissa bit) and
    # decode that with torch's fp8 cast.
    got = np.array([oracle_mod.e2m1_value(c) for c in range(16)])
    e4 = []
    for c in range(16):
        s, E, m = c >> 3, (c >> 1) & 3, c & 1
        if E == 0 and m == 0:
            bits = 0
        elif E == 0:  # subnormal 0.5 = 2^-1
            bits = (6 << 3)
        else:
            bits = ((E + 6) << 3) | (m << 2)
        e4.append((s << 7) | bits)
    want = _torch_e4m3(np.array(e4))
    assert np.array_equal(got, want)
    assert sorted(set(np.abs(got))) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e8m0_decode_all_256_codes(oracle_mod):
    got = np.array([oracle_mod.e8m0_value(e) for e in range(256)])
    want = _torch_e8m0(np.arange(256))
    assert np.isnan(got[255]) and np.isnan(want[255])
    assert np.array_equal(got[:255], want[:255])
    assert got[127] == 1.0


def test_rne_e4m3_all_bf16_in_range(oracle_mod):
    bits = _all_bf16_finite()
    v = _bf16_to_f64(bits)
    v = v[np.abs(v) <= 448.0]
    got = np.array([oracle_mod.rne_e4m3(x) for x in v], np.uint8)
    want = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)


def test_rne_e4m3_exact_midpoints(oracle_mod):
    vals = _torch_e4m3(np.arange(0x7F))
    mids = (vals[:-1] + vals[1:]) / 2.0  # exact in fp64 and fp32
    got = np.array([oracle_mod.rne_e4m3(x) for x in mids], np.uint8)
    want = torch.from_numpy(mids.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)
    got_neg = np.array([oracle_mod.rne_e4m3(-x) for x in mids], np.uint8)
    assert np.array_equal(got_neg, want | 0x80)
    # saturation (the oracle's reading; torch would give NaN here)
    assert oracle_mod.rne_e4m3(1e6) == 0x7E and oracle_mod.rne_e4m3(-500.0) == 0xFE
    assert oracle_mod.rne_e4m3(-1e-30) == 0x80 and oracle_mod.rne_e4m3(-0.0) == 0x80


def test_rne_e2m1_against_numpy_round_half_even(oracle_mod):
    rng = np.random.default_rng(0)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[:-1] + grid[1:]) / 2
    v = np.concatenate([rng.uniform(0, 7, 4000), mids, grid])
    for x in v:
        if x >= 6:
            want = 6.0
        elif x < 1:  # subnormal step 0.5
            want = np.round(x * 2) / 2
        else:
            e = math.floor(math.log2(x))
            want = min(6.0, np.round(x / 2.0 ** e * 2) / 2 * 2.0 ** e)
        c = oracle_mod.rne_e2m1(x)
        assert oracle_mod.e2m1_value(c) == want, (x, c, want)
        assert oracle_mod.rne_e2m1(-x) == (c | 8)


def test_e8m0_exponent_is_minimal_for_all_bf16(oracle_mod):
    bits = _all_bf16_finite()
    v = np.abs(_bf16_to_f64(bits))
    v = np.unique(v[v > 0])
    for fmax in (448.0, 6.0):
        for a in v:
            e = oracle_mod.e8m0_for_amax(a, fmax)
            assert 0 <= e <= 254
            hi = math.ldexp(fmax, e - 127)
            lo = math.ldexp(fmax, e - 128)
            assert a <= hi or e == 254
            assert a > lo or e == 0
    assert oracle_mod.e8m0_for_amax(0.0, 448.0) == 0
    # exact boundaries: amax == 448 * 2^j gives k == j
    assert oracle_mod.e8m0_for_amax(448.0, 448.0) == 127
    assert oracle_mod.e8m0_for_amax(448.0 * 2 ** -5, 448.0) == 122
    assert oracle_mod.e8m0_for_amax(np.nextafter(448.0, 1e9), 448.0) == 128


# ---- quantisers ---------------------------------------------------------------

def test_quant_act_e8m0_against_torch_cast(oracle_mod):
    x = synth.bf16_matrix(1, 7, 96, 1.0)
    x[0, :32] = 0  # an all-zero block
    x[1, 5] = 1e-3
    codes, scales = oracle_mod.quant_act_e8m0(x)
    xd = x.to(torch.float64).numpy()
    assert scales.shape == (7, 3) and scales[0, 0] == 0 and (codes[0, :32] == 0).all()
    for m in range(7):
        for b in range(3):
            blk = xd[m, 32 * b:32 * b + 32]
            e = int(scales[m, b])
            amax = np.abs(blk).max()
            if amax > 0:
                # invariant: amax / 2^k in (224, 448]
                r = amax / 2.0 ** (e - 127)
                assert 224 < r <= 448
            want = torch.from_numpy((blk * 2.0 ** (127 - e)).astype(np.float32)).to(
                torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(codes[m, 32 * b:32 * b + 32], want)


def test_quant_act_e8m0_every_bf16_pattern(oracle_mod):
    # all 65,536 bf16 patterns minus non-finite ones, spread over blocks; each
    # block's max is forced so that the scale exponent varies
    bits = _all_bf16_finite()
    pad = (-len(bits)) % 32
    bits = np.concatenate([bits, np.zeros(pad, np.uint16)]).reshape(-1, 32)
    codes, scales = oracle_mod.quant_act_e8m0(bits)
    xd = _bf16_to_f64(bits.reshape(-1)).reshape(bits.shape)
    want = torch.from_numpy(xd * np.ldexp(1.0, 127 - scales.astype(np.int64))).float()
    want = want.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, want)


def test_quant_f32_row_against_torch(oracle_mod):
    x = synth.bf16_matrix(4, 5, 160, 1.0)
    x[2] = 0
    codes, s = oracle_mod.quant_f32_row(x)
    xf = x.float()
    amax = xf.abs().amax(1)
    s_t = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    assert np.array_equal(s, s_t.numpy())
    want = (xf / s_t[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, want)


def test_quant_w_e4m3_32x32_blocks(oracle_mod):
    w = synth.bf16_matrix(9, 64, 96, 0.02)
    codes, scales = oracle_mod.quant_w_e4m3_32x32(w)
    assert scales.shape == (2, 3)
    wd = w.to(torch.float64).numpy()
    for nb in range(2):
        for kb in range(3):
            blk = wd[32 * nb:32 * nb + 32, 32 * kb:32 * kb + 32]
            e = int(scales[nb, kb])
            assert 224 < np.abs(blk).max() / 2.0 ** (e - 127) <= 448
            want = torch.from_numpy((blk * 2.0 ** (127 - e)).astype(np.float32)).to(
                torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(codes[32 * nb:32 * nb + 32, 32 * kb:32 * kb + 32], want)


def test_quant_w_e2m1_packing_and_scale(oracle_mod):
    w = synth.bf16_matrix(10, 6, 64, 0.02)
    packed, scales = oracle_mod.quant_w_e2m1_1x32(w)
    assert packed.shape == (6, 32) and scales.shape == (6, 2)
    wd = w.to(torch.float64).numpy()
    lo = packed & 15
    hi = packed >> 4
    codes = np.empty((6, 64), np.uint8)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    for n in range(6):
        for kb in range(2):
            e = int(scales[n, kb])
            blk = wd[n, 32 * kb:32 * kb + 32]
            assert 3 < np.abs(blk).max() / 2.0 ** (e - 127) <= 6
            for k in range(32):
                c = codes[n, 32 * kb + k]
                v = blk[k] * 2.0 ** (127 - e)
                # nearest grid value: |v - dec(c)| is at most half a grid step
                dec = oracle_mod.e2m1_value(int(c))
                step = 0.5 if abs(v) < 2 else (1.0 if abs(v) < 4 else 2.0)
                assert abs(v - dec) <= step / 2 + 1e-12
                assert (c >> 3) == (1 if math.copysign(1, v) < 0 else 0)


# ---- GEMM ---------------------------------------------------------------------

def _dequant_a(codes, scales, a_fmt, K, oracle_mod=None):
    if a_fmt == 3:  # e2m1 activations, packed like e2m1 weights
        return _dequant_b(codes, scales, 1, codes.shape[0], K, oracle_mod)
    val = _torch_e4m3(codes)
    if a_fmt == 1:
        return val * scales.astype(np.float64)[:, None]
    return val * np.repeat(_torch_e8m0(scales), 32, axis=1)


def _dequant_b(codes, scales, b_fmt, N, K, oracle_mod):
    if b_fmt == 1:  # e2m1 packed, low nibble first; values via the e4m3 re-encode pin
        tab = np.array([oracle_mod.e2m1_value(c) for c in range(16)])
        val = np.empty((N, K))
        val[:, 0::2] = tab[codes & 15]
        val[:, 1::2] = tab[codes >> 4]
        return val * np.repeat(_torch_e8m0(scales), 32, axis=1)
    val = _torch_e4m3(codes)
    if b_fmt == 2:
        return val * scales.astype(np.float64)[:, None]
    s = np.repeat(np.repeat(_torch_e8m0(scales), 32, axis=0), 32, axis=1)
    return val * s


FORMATS = [(0, 0), (0, 1), (1, 2), (3, 1)]  # (3, 1): W4A4, e2m1 on both sides


def _problem(oracle_mod, seed, M, N, K, a_fmt, b_fmt):
    x, w, b = synth.problem(seed, M, N, K)
    a_codes, a_scales = oracle_mod.quant_act(x, a_fmt)
    b_codes, b_scales = oracle_mod.quant_weight(w, b_fmt)
    return a_codes, a_scales, b_codes, b_scales, b


@pytest.mark.parametrize("a_fmt,b_fmt", FORMATS)
def test_gemm_equals_dequantised_matmul(oracle_mod, a_fmt, b_fmt):
    M, N, K = 5, 64, 128
    a, sa, bc, sb, _ = _problem(oracle_mod, 21, M, N, K, a_fmt, b_fmt)
    y, t = oracle_mod.gemm(a, sa, a_fmt, bc, sb, b_fmt, None, 0, M, N, K)
    A = _dequant_a(a, sa, a_fmt, K, oracle_mod)
    B = _dequant_b(bc, sb, b_fmt, N, K, oracle_mod)
    want = A @ B.T
    tt = np.abs(A) @ np.abs(B).T
    # dyadic inputs: every product and partial sum is exact in fp64 except for
    # the fp32 row scales, which matmul applies per term and the oracle once
    if a_fmt == 1:
        assert (np.abs(y - want) <= 1e-13 * tt).all()
    else:
        assert np.array_equal(y, want)
    assert np.allclose(t, tt, rtol=1e-13, atol=0)


def test_gemm_identity_weight_is_exact(oracle_mod):
    M, K = 4, 64
    x = synth.bf16_matrix(3, M, K, 1.0)
    a, sa = oracle_mod.quant_act_e8m0(x)
    eye = np.zeros((K, K), np.uint8)
    eye[np.arange(K), np.arange(K)] = 0x38  # e4m3 1.0
    sb = np.full((K // 32, K // 32), 127, np.uint8)
    y, _ = oracle_mod.gemm(a, sa, 0, eye, sb, 0, None, 0, M, K, K)
    assert np.array_equal(y, _dequant_a(a, sa, 0, K))


def test_gemm_one_hot_x_selects_a_weight_column(oracle_mod):
    N, K = 64, 96
    w = synth.bf16_matrix(4, N, K, 0.02)
    bc, sb = oracle_mod.quant_w_e2m1_1x32(w)
    for k in (0, 33, 95):
        a = np.zeros((1, K), np.uint8)
        a[0, k] = 0x38
        sa = np.full((1, K // 32), 127, np.uint8)
        y, _ = oracle_mod.gemm(a, sa, 0, bc, sb, 1, None, 0, 1, N, K)
        B = _dequant_b(bc, sb, 1, N, K, oracle_mod)
        assert np.array_equal(y[0], B[:, k])


def test_gemm_bumping_one_scale_doubles_that_block(oracle_mod):
    M, N, K = 3, 64, 128
    a, sa, bc, sb, _ = _problem(oracle_mod, 8, M, N, K, 0, 0)
    y0, _, acc0 = oracle_mod.gemm(a, sa, 0, bc, sb, 0, None, 0, M, N, K, want_acc=True)
    sb2 = sb.copy()
    sb2[1, 2] += 1  # W rows 32..63, K block 2
    y1, _, acc1 = oracle_mod.gemm(a, sa, 0, bc, sb2, 0, None, 0, M, N, K, want_acc=True)
    A = _dequant_a(a, sa, 0, K)
    B = _dequant_b(bc, sb, 0, N, K, oracle_mod)
    blk = A[:, 64:96] @ B[:, 64:96].T
    d = acc1 - acc0
    assert np.array_equal(d[:, :32], np.zeros((M, 32)))
    assert np.array_equal(d[:, 32:], blk[:, 32:])
    sa2 = sa.copy()
    sa2[2, 0] += 1
    y2, _ = oracle_mod.gemm(a, sa2, 0, bc, sb, 0, None, 0, M, N, K)
    assert np.array_equal(y2[2] - y0[2], (A[2:3, :32] @ B[:, :32].T)[0])
    assert np.array_equal(y2[:2], y0[:2])


def test_bias_epilogue_is_linear(oracle_mod):
    M, N, K = 4, 32, 64
    a, sa, bc, sb, b = _problem(oracle_mod, 12, M, N, K, 0, 0)
    y0, _ = oracle_mod.gemm(a, sa, 0, bc, sb, 0, None, 0, M, N, K)
    y1, t1 = oracle_mod.gemm(a, sa, 0, bc, sb, 0, b, 1, M, N, K)
    assert np.allclose(y1 - y0, b.numpy().astype(np.float64)[None, :], rtol=0, atol=1e-15)


def test_gelu_and_silu_against_torch(oracle_mod):
    v = np.concatenate([np.linspace(-30, 30, 2001), [0.0, 1.0, -1.0, 1e-8, 88.0]])
    g = np.array([oracle_mod.gelu_tanh(x) for x in v])
    s = np.array([oracle_mod.silu(x) for x in v])
    tv = torch.from_numpy(v)
    assert np.allclose(g, F.gelu(tv, approximate="tanh").numpy(), rtol=1e-13, atol=1e-15)
    assert np.allclose(s, F.silu(tv).numpy(), rtol=1e-13, atol=1e-15)
    assert oracle_mod.gelu_tanh(0.0) == 0.0 and oracle_mod.silu(0.0) == 0.0
    # the tanh form stays within 1e-3 of the erf form of GELU
    erf_gelu = 0.5 * v * (1 + np.array([math.erf(x / math.sqrt(2)) for x in v]))
    assert np.max(np.abs(g - erf_gelu)) < 1e-3


def test_gelu_constants_from_the_page(oracle_mod):
    # tests/golden/gelu_tanh_constants.txt: the constants vit.rs prints
    with open(os.path.join(GOLDEN, "gelu_tanh_constants.txt")) as f:
        rows = dict(l.split()[:2] for l in f if l.strip() and not l.startswith("#"))
    c = float(rows["sqrt_2_over_pi"])
    cub = float(rows["cubic"])
    clamp = float(rows["clamp"])
    assert abs(c - math.sqrt(2 / math.pi)) < 1e-10
    for v in np.linspace(-12, 12, 481):
        u = max(-clamp, min(clamp, c * (v + cub * v ** 3)))
        page = 0.5 * v * (1 + math.tanh(u))
        assert abs(oracle_mod.gelu_tanh(v) - page) <= 1e-9 * max(1, abs(v))


def test_gelu_epilogue_applies_bias_first(oracle_mod):
    M, N, K = 3, 32, 64
    a, sa, bc, sb, b = _problem(oracle_mod, 13, M, N, K, 0, 0)
    _, _, acc = oracle_mod.gemm(a, sa, 0, bc, sb, 0, None, 0, M, N, K, want_acc=True)
    y, _ = oracle_mod.gemm(a, sa, 0, bc, sb, 0, b, 2, M, N, K)
    want = F.gelu(torch.from_numpy(acc + b.numpy().astype(np.float64)[None]), approximate="tanh").numpy()
    assert np.allclose(y, want, rtol=1e-13, atol=1e-16)


def test_swiglu_pairs_gate_rows_with_up_rows(oracle_mod):
    M, N, K = 4, 128, 64
    a, sa, bc, sb, b = _problem(oracle_mod, 14, M, N, K, 0, 1)
    _, _, acc = oracle_mod.gemm(a, sa, 0, bc, sb, 1, None, 0, M, N, K, want_acc=True)
    y, t = oracle_mod.gemm(a, sa, 0, bc, sb, 1, b, 3, M, N, K)
    bb = b.numpy().astype(np.float64)
    g = torch.from_numpy(acc[:, :64] + bb[None, :64])
    u = acc[:, 64:] + bb[None, 64:]
    assert y.shape == (M, 64)
    assert np.allclose(y, F.silu(g).numpy() * u, rtol=1e-13, atol=1e-16)
    assert (t >= 0).all()
    # without bias
    y0, _ = oracle_mod.gemm(a, sa, 0, bc, sb, 1, None, 3, M, N, K)
    assert np.allclose(y0, F.silu(torch.from_numpy(acc[:, :64])).numpy() * acc[:, 64:], rtol=1e-13, atol=1e-16)


# ---- the SwiGLU tolerance term ------------------------------------------------
#
# For SwiGLU the acceptance bound carries the GEMM's error terms through the
# epilogue to first order: |d acc_g| <= 1e-5 T_g and |d acc_u| <= 1e-5 T_u move
# y = silu(g) u by at most |silu'(g)| T_g |u| + |silu(g)| T_u (times 1e-5).
# The checks below tie that term to autograd, to finite differences and to a
# brute-force propagation on dequantised operands; the planted-mistake test
# rebuilds the oracle with a wrong term and shows that they catch it.

def _check_silu_grad(om):
    v = np.concatenate([np.linspace(-30, 30, 1201), [0.0, 1e-8, -1e-8, 5.0, -5.0]])
    got = np.array([om.silu_grad(x) for x in v])
    tv = torch.from_numpy(v).requires_grad_(True)
    F.silu(tv).sum().backward()
    assert np.allclose(got, tv.grad.numpy(), rtol=1e-12, atol=1e-15), "silu' differs from autograd"
    h = 1e-5
    fd = np.array([(om.silu(x + h) - om.silu(x - h)) / (2 * h) for x in v])
    assert np.allclose(got, fd, rtol=1e-7, atol=1e-9), "silu' differs from the central difference"
    assert om.silu_grad(0.0) == 0.5  # sigma(0) (1 + 0) = 1/2


def _dequant_swiglu(om, seed, M, N, K, b_fmt):
    a, sa, bc, sb, bias = _problem(om, seed, M, N, K, 0, b_fmt)
    A = _dequant_a(a, sa, 0, K)
    B = _dequant_b(bc, sb, b_fmt, N, K, om)
    return a, sa, bc, sb, bias, A, B


def _check_swiglu_term(om, b_fmt):
    M, N, K = 4, 128, 96
    a, sa, bc, sb, bias, A, B = _dequant_swiglu(om, 15 + b_fmt, M, N, K, b_fmt)
    y, t = om.gemm(a, sa, 0, bc, sb, b_fmt, bias, 3, M, N, K)
    h = N // 2
    bb = bias.double().numpy()
    g = A @ B[:h].T + bb[None, :h]
    u = A @ B[h:].T + bb[None, h:]
    t_g = np.abs(A) @ np.abs(B[:h]).T
    t_u = np.abs(A) @ np.abs(B[h:]).T
    gt = torch.from_numpy(g).requires_grad_(True)
    s = F.silu(gt)
    s.sum().backward()
    want = np.abs(gt.grad.numpy()) * t_g * np.abs(u) + np.abs(s.detach().numpy()) * t_u
    assert np.allclose(t, want, rtol=1e-12, atol=0), "SwiGLU T differs from the brute-force propagation"


def _check_swiglu_term_is_tight(om):
    # One token.  Perturbing every gate product a_k w_gk by eps |a_k w_gk| with
    # the sign of silu'(g) u moves y by eps |silu'(g)| T_g |u| to first order;
    # the up products, likewise, by eps |silu(g)| T_u.  The two perturbations
    # together reach eps T, and random signs stay inside it.
    M, N, K = 1, 128, 96
    a, sa, bc, sb, bias, A, B = _dequant_swiglu(om, 19, M, N, K, 1)
    y, t = om.gemm(a, sa, 0, bc, sb, 1, bias, 3, M, N, K)
    h = N // 2
    bb = bias.double().numpy()

    def swiglu(Bm):
        g = torch.from_numpy(A @ Bm[:h].T + bb[None, :h])
        return (F.silu(g) * torch.from_numpy(A @ Bm[h:].T + bb[None, h:])).numpy()

    y0 = swiglu(B)
    g0 = A @ B[:h].T + bb[None, :h]
    u0 = A @ B[h:].T + bb[None, h:]
    gt = torch.from_numpy(g0).requires_grad_(True)
    F.silu(gt).sum().backward()
    dg = gt.grad.numpy()[0]
    sg = F.silu(torch.from_numpy(g0)).numpy()[0]
    eps = 1e-7
    # w_nk += eps s sign(a_k) |w_nk| changes a_k w_nk by eps s |a_k w_nk|
    a_sign = np.sign(A[0])[None, :]
    s_gate = np.sign(dg * u0[0])[:, None]
    s_up = np.sign(sg)[:, None]
    Bp = B.copy()
    Bp[:h] += eps * s_gate * a_sign * np.abs(B[:h])
    Bp[h:] += eps * s_up * a_sign * np.abs(B[h:])
    dy = (swiglu(Bp) - y0)[0]
    assert np.allclose(dy, eps * t[0], rtol=1e-4, atol=0), "T is not the first-order bound it should be"
    rng = np.random.default_rng(7)
    for _ in range(3):
        Br = B * (1 + eps * rng.uniform(-1, 1, B.shape))
        assert (np.abs(swiglu(Br) - y0)[0] <= eps * t[0] * (1 + 1e-4)).all()


def test_silu_grad_against_autograd_and_finite_differences(oracle_mod):
    _check_silu_grad(oracle_mod)


@pytest.mark.parametrize("b_fmt", [0, 1])
def test_swiglu_tolerance_term_against_brute_force(oracle_mod, b_fmt):
    _check_swiglu_term(oracle_mod, b_fmt)


def test_swiglu_tolerance_term_is_the_tight_first_order_bound(oracle_mod):
    _check_swiglu_term_is_tight(oracle_mod)


# Mistakes planted in a rebuilt copy of the oracle (never in the oracle the
# other tests use): each must make at least two of the checks above fail.
SWIGLU_TERM_MUTANTS = [
    ("sign flip inside the SiLU derivative",
     "return sig * (1.0 + v * (1.0 - sig));", "return sig * (1.0 - v * (1.0 - sig));"),
    ("|u| dropped from the gate term",
     "t = fabs(dsg) * aabs * fabs(u) + fabs(sg) * u_abs;", "t = fabs(dsg) * aabs + fabs(sg) * u_abs;"),
    ("gate and up error terms swapped",
     "t = fabs(dsg) * aabs * fabs(u) + fabs(sg) * u_abs;", "t = fabs(dsg) * u_abs * fabs(u) + fabs(sg) * aabs;"),
    ("derivative taken as sigma(g)",
     "return sig * (1.0 + v * (1.0 - sig));", "return sig;"),
]


@pytest.mark.parametrize("what,old,new", SWIGLU_TERM_MUTANTS, ids=[m[0] for m in SWIGLU_TERM_MUTANTS])
def test_swiglu_term_checks_catch_planted_mistakes(oracle_mod, tmp_path, what, old, new):
    import subprocess
    src_path = os.path.join(os.path.dirname(oracle_mod.__file__), "mxref.c")
    src = open(src_path).read()
    assert src.count(old) == 1, f"mutation site for '{what}' not found"
    (tmp_path / "mxref.c").write_text(src.replace(old, new))
    so = tmp_path / "_mxref_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-fPIC", "-fopenmp", "-fno-fast-math",
                    "-ffp-contract=off", "-shared", "-o", str(so), str(tmp_path / "mxref.c"), "-lm"], check=True)
    mutant = oracle_mod.load_library(str(so))
    saved = oracle_mod._LIB
    caught = []
    try:
        oracle_mod._LIB = mutant
        for name, check in [("silu_grad", lambda: _check_silu_grad(oracle_mod)),
                            ("term e4m3", lambda: _check_swiglu_term(oracle_mod, 0)),
                            ("term e2m1", lambda: _check_swiglu_term(oracle_mod, 1)),
                            ("tight", lambda: _check_swiglu_term_is_tight(oracle_mod))]:
            try:
                check()
            except AssertionError:
                caught.append(name)
    finally:
        oracle_mod._LIB = saved
    assert len(caught) >= 2, f"planted mistake '{what}' caught only by {caught}"


def test_tolerance_accepts_correct_bf16_roundings_and_no_more(oracle_mod):
    # The bound's first term stands for the bf16 rounding of the output: every
    # correct rounding (torch's cast) of values across bf16's whole range,
    # subnormals included, passes with T = 0; two bf16 steps away fails.
    rng = np.random.default_rng(3)
    n = 20000
    y = np.where(rng.random(n) < 0.5, -1.0, 1.0) * np.exp2(rng.uniform(-140.0, 120.0, n))
    yb = torch.from_numpy(y).to(torch.bfloat16)
    t0 = np.zeros(n)
    assert oracle_mod.within_tolerance(yb.double().numpy(), y, t0).all()
    bits = yb.view(torch.int16).numpy().astype(np.int32)
    far = torch.from_numpy((bits + 2).astype(np.int16)).view(torch.bfloat16).double().numpy()
    normal = np.abs(y) >= 2.0 ** -124
    assert not oracle_mod.within_tolerance(far, y, t0)[normal].any()


def test_page_shapes_fixture(oracle_mod):
    # tests/golden/page_shapes.txt: layouts the pages print.
    path = os.path.join(GOLDEN, "page_shapes.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    seen = set()
    for r in rows:
        kind = r[0]
        seen.add(kind)
        if kind == "scale32x32":
            N, K, sr, sc = map(int, r[1:5])
            # the oracle's scale array for an N x K weight has the printed shape;
            # quantise a 32-row slice and check the column count, rows by formula
            w = synth.bf16_matrix(0, 32, K, 0.02)
            _, s = oracle_mod.quant_w_e4m3_32x32(w)
            assert s.shape[1] == sc and N // 32 == sr
        elif kind == "bytes":
            N, K, bytes_per, total = int(r[1]), int(r[2]), float(r[3]), float(r[4])
            assert abs(N * K * bytes_per / 1e9 - total) < 0.006
    assert {"scale32x32", "bytes"} <= seen


# ---- producers that hand the next GEMM MX codes (fused-quant row) -------------

def _torch_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16_midpoint_distance(v: np.ndarray) -> np.ndarray:
    """Relative distance of each fp64 value to the nearest bf16 rounding
    midpoint (where two correct roundings of a value one ulp away can differ)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    q = np.ldexp(1.0, (np.maximum(e, -126) - 7).astype(np.int64))  # bf16 quantum
    frac = a / q - np.floor(a / q)
    return np.abs(frac - 0.5) * q / np.where(a > 0, a, 1.0)


def test_bf16_rne_against_torch_fp32_cast(oracle_mod):
    # fp32 inputs: torch's float32 -> bfloat16 cast is one RNE rounding.  Random
    # finite patterns, every exact midpoint between neighbouring bf16 values of
    # a sweep of exponents, subnormals, and the overflow threshold.
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 1 << 32, 200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    hi = np.arange(0, 0x7F7F, 97, dtype=np.uint32)
    mids = ((hi << 16) | 0x8000).view(np.float32)  # exactly halfway to the next bf16
    extra = np.array([0.0, -0.0, 1.0, -1.0, 3.3895313892515355e38, 3.3961775292304690e38,
                      np.float32(2.0 ** -133), np.float32(3 * 2.0 ** -134)], np.float32)
    f = np.concatenate([f, mids, -mids, extra])
    got = oracle_mod.round_bf16(f.astype(np.float64))
    want = _torch_bf16_bits(torch.from_numpy(f).to(torch.bfloat16))
    assert np.array_equal(got, want)


def test_bf16_rne_is_nearest_even_for_fp64_inputs(oracle_mod):
    # values that are not fp32 numbers (a detour through fp32 would round
    # twice): the result is a nearest bf16 value, the even one on a tie
    rng = np.random.default_rng(6)
    v = rng.standard_normal(20_000) * np.exp2(rng.integers(-130, 120, 20_000))
    mid = _bf16_to_f64(np.arange(0x3F80, 0x3FA0, dtype=np.uint16)) + 2.0 ** -8  # exact midpoints in [1, 2)
    v = np.concatenate([v, mid, -mid, mid * (1 + 2.0 ** -40), mid * (1 - 2.0 ** -40)])
    got = oracle_mod.round_bf16(v)
    mag = (got & 0x7FFF).astype(np.int64)
    a = np.abs(v)
    d = np.abs(a - _bf16_to_f64(mag.astype(np.uint16)))
    d_up = np.abs(a - _bf16_to_f64((mag + 1).astype(np.uint16)))
    d_dn = np.abs(a - _bf16_to_f64(np.maximum(mag - 1, 0).astype(np.uint16)))
    assert (d <= d_up).all() and (d <= d_dn).all()
    tie = (d == d_up) | ((d == d_dn) & (mag > 0))
    assert tie.sum() >= 64 and (mag[tie] % 2 == 0).all()
    assert np.array_equal(np.signbit(_bf16_to_f64(got)), np.signbit(v))


def test_residual_add_against_torch(oracle_mod):
    # bf16(x + r): torch adds in fp32 (exact for two bf16 values whose
    # exponents differ by <= 16; otherwise the smaller one is below half a
    # bf16 ulp of the larger either way) and rounds once to bf16
    x = synth.bf16_matrix(31, 8, 256, 1.0)
    r = synth.bf16_matrix(32, 8, 256, 1.0)
    r[0] = r[0] * 2.0 ** -20  # far-apart exponents
    r[1] = -x[1]  # exact cancellation -> +0
    got = oracle_mod.add_bf16(x, r)
    want = _torch_bf16_bits((x.float() + r.float()).to(torch.bfloat16))
    assert np.array_equal(got, want)


def test_rmsnorm_against_torch_rms_norm(oracle_mod):
    M, K, eps = 6, 1536, 1e-6
    v = synth.bf16_matrix(33, M, K, 1.0)
    v[1] = v[1] * 2.0 ** 30
    w = synth.bf16_matrix(34, 1, K, 0.5)[0] + 1.0
    got = oracle_mod.rmsnorm_bf16(v, w, eps)
    ref = F.rms_norm(v.double(), (K,), weight=w.double(), eps=eps).numpy()
    want = oracle_mod.round_bf16(ref)
    # torch's fp64 result may differ from the oracle's in the last fp64 bit,
    # which can change the bf16 rounding only right at a midpoint
    diff = got != want
    assert (_bf16_midpoint_distance(ref)[diff] < 1e-12).all()
    assert diff.sum() <= 2


def test_rmsnorm_closed_forms(oracle_mod):
    K = 96
    w = synth.bf16_matrix(35, 1, K, 1.0)[0]
    wb = _torch_bf16_bits(w)
    # a constant row c with eps = 0 normalises to sign(c) exactly: y = sign(c) w
    for c in (3.0, -0.375, 2.0 ** -100):
        row = torch.full((1, K), c, dtype=torch.bfloat16)
        y = oracle_mod.rmsnorm_bf16(row, w, 0.0)[0]
        want = wb if c > 0 else wb ^ np.uint16(0x8000)
        assert np.array_equal(y, want)
    # eps = 0: scaling a row by 2^j leaves the result bit for bit unchanged
    v = synth.bf16_matrix(36, 3, K, 1.0)
    y0 = oracle_mod.rmsnorm_bf16(v, w, 0.0)
    for j in (-40, -3, 5, 60):
        assert np.array_equal(oracle_mod.rmsnorm_bf16(v * 2.0 ** j, w, 0.0), y0)
    # an all-zero row with eps > 0 gives zeros
    z = oracle_mod.rmsnorm_bf16(torch.zeros((1, K), dtype=torch.bfloat16), w, 1e-6)
    assert (_bf16_to_f64(z) == 0).all()


def test_add_rms_quant_is_the_unfused_chain(oracle_mod):
    # against the chain built from library routines: torch's fp32 add and
    # bf16 cast, torch's fp64 rms_norm, and the e4m3 cast of each block
    # scaled by 2^-k with k the minimal exponent (torch float8_e4m3fn)
    M, K, eps = 5, 512, 1e-6
    x = synth.bf16_matrix(37, M, K, 1.0)
    r = synth.bf16_matrix(38, M, K, 1.0)
    w = synth.bf16_matrix(39, 1, K, 0.2)[0] + 1.0
    res, y, codes, scales = oracle_mod.add_rms_quant(x, r, w, eps)
    res_t = (x.float() + r.float()).to(torch.bfloat16)
    assert np.array_equal(res, _torch_bf16_bits(res_t))
    ref = F.rms_norm(res_t.double(), (K,), weight=w.double(), eps=eps).numpy()
    yd = _bf16_to_f64(y)
    assert (np.abs(yd - ref) <= 2.0 ** -8 * np.abs(ref)).all()  # one bf16 rounding
    blocks = yd.reshape(M, K // 32, 32)
    amax = np.abs(blocks).max(-1)
    k = scales.astype(np.int64) - 127
    assert ((amax <= 448.0 * np.exp2(k)) & (amax > 448.0 * np.exp2(k - 1))).all()
    want = torch.from_numpy((blocks * np.exp2(-k)[..., None]).astype(np.float32))
    want = want.to(torch.float8_e4m3fn).view(torch.uint8).numpy().reshape(M, K)
    assert np.array_equal(codes, want)


def test_gemm_swiglu_mxq_is_the_unfused_chain(oracle_mod):
    # tiny SwiGLU problem: brute force (dequantise, fp64 matmul, torch silu)
    # rounded to bf16, then each 32-wide block cast to e4m3 at its minimal
    # E8M0 exponent
    M, N, K = 3, 128, 96
    a, sa, bc, sb, bias = _problem(oracle_mod, 40, M, N, K, 0, 1)
    yb, codes, scales, y, t = oracle_mod.gemm_swiglu_mxq(a, sa, 0, bc, sb, 1, bias, M, N, K)
    A = _dequant_a(a, sa, 0, K)
    B = _dequant_b(bc, sb, 1, N, K, oracle_mod)
    acc = A @ B.T + bias.double().numpy()[None, :]
    g, u = torch.from_numpy(acc[:, :N // 2]), torch.from_numpy(acc[:, N // 2:])
    ref = (F.silu(g) * u).numpy()
    want_y = oracle_mod.round_bf16(ref)
    diff = yb != want_y
    assert (_bf16_midpoint_distance(ref)[diff] < 1e-12).all() and diff.sum() <= 1
    blocks = _bf16_to_f64(yb).reshape(M, N // 64, 32)
    k = scales.astype(np.int64) - 127
    amax = np.abs(blocks).max(-1)
    assert ((amax <= 448.0 * np.exp2(k)) & ((amax > 448.0 * np.exp2(k - 1)) | (amax == 0))).all()
    want = torch.from_numpy((blocks * np.exp2(-k)[..., None]).astype(np.float32))
    want = want.to(torch.float8_e4m3fn).view(torch.uint8).numpy().reshape(M, N // 2)
    assert np.array_equal(codes, want)


# ---- the W4A4 operand and the residual epilogue (next rows) -------------------

def test_e2m1_activation_operand(oracle_mod):
    # activations quantised to e2m1 with the 1 x 32 rule: every block's amax
    # lands in (3, 6] of its scale, each code is the RNE e2m1 neighbour, and
    # the packed bytes put the even k in the low nibble
    M, K = 6, 256
    x = synth.bf16_matrix(41, M, K, 1.0)
    x[2, 32:64] = 0
    packed, scales = oracle_mod.quant_act(x, 3)
    assert packed.shape == (M, K // 2) and scales.shape == (M, K // 32)
    xd = x.double().numpy().reshape(M, K // 32, 32)
    k = scales.astype(np.int64) - 127
    amax = np.abs(xd).max(-1)
    nz = amax > 0
    assert ((amax[nz] <= 6.0 * np.exp2(k[nz])) & (amax[nz] > 3.0 * np.exp2(k[nz]))).all()
    assert scales[2, 1] == 0 and (packed[2, 16:32] == 0).all()
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    q = np.abs(xd) * np.exp2(-k)[..., None]
    lo = packed & 15
    hi = packed >> 4
    codes = np.empty((M, K), np.int64)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    codes = codes.reshape(M, K // 32, 32)
    mag = grid[codes & 7]
    # nearest grid point (ties: the even code)
    d = np.abs(q - mag)
    assert (d <= np.abs(q[..., None] - grid).min(-1)).all()
    tie = np.isclose(np.abs(q[..., None] - grid), d[..., None], rtol=0, atol=0).sum(-1) > 1
    assert ((codes[tie] & 1) == 0).all()  # a tie goes to the even code
    assert np.array_equal((codes >> 3) & 1, np.signbit(xd).astype(np.int64))  # sign kept, zeros too


def test_residual_epilogue_against_brute_force(oracle_mod):
    M, N, K = 4, 96, 128
    a, sa, bc, sb, bias = _problem(oracle_mod, 42, M, N, K, 0, 0)
    res = synth.bf16_matrix(43, M, N, 1.0)
    y, t = oracle_mod.gemm_residual(a, sa, 0, bc, sb, 0, bias, res, M, N, K)
    A = _dequant_a(a, sa, 0, K)
    B = _dequant_b(bc, sb, 0, N, K, oracle_mod)
    want = res.double().numpy() + (A @ B.T + bias.double().numpy()[None, :])
    assert np.allclose(y, want, rtol=1e-14, atol=1e-300)
    # without a residual (all zeros) it is the bias epilogue exactly
    y0, t0 = oracle_mod.gemm_residual(a, sa, 0, bc, sb, 0, bias, torch.zeros((M, N), dtype=torch.bfloat16),
                                      M, N, K)
    yb, tb = oracle_mod.gemm(a, sa, 0, bc, sb, 0, bias, 1, M, N, K)
    assert np.array_equal(y0, yb) and np.array_equal(t0, tb)


def test_grouped_gemm_against_per_expert_brute_force(oracle_mod):
    # tokens sorted by expert (one expert gets none), e2m1 expert weights with
    # 1 x 32 scales, SwiGLU gate_up; each group against its own dequantised
    # matmul, and reordering the experts moves the rows with them
    E, N, K = 4, 128, 96
    counts = [3, 0, 5, 2]
    offs = np.concatenate([[0], np.cumsum(counts)])
    x = synth.bf16_matrix(44, int(offs[-1]), K, 1.0)
    a, sa = oracle_mod.quant_act_e8m0(x)
    bc, sb, bias = [], [], []
    for e in range(E):
        c, s_ = oracle_mod.quant_w_e2m1_1x32(synth.bf16_matrix(45 + e, N, K, 0.05))
        bc.append(c)
        sb.append(s_)
        bias.append(synth.f32_vector(50 + e, N, 0.1))
    y, t = oracle_mod.gemm_grouped(a, sa, 0, bc, sb, 1, bias, 3, offs, N, K)
    assert y.shape == (offs[-1], N // 2)
    for e in range(E):
        r0, r1 = offs[e], offs[e + 1]
        if r1 == r0:
            continue
        A = _dequant_a(a[r0:r1], sa[r0:r1], 0, K)
        B = _dequant_b(bc[e], sb[e], 1, N, K, oracle_mod)
        acc = A @ B.T + bias[e].double().numpy()[None, :]
        g, u = torch.from_numpy(acc[:, :N // 2]), torch.from_numpy(acc[:, N // 2:])
        assert np.allclose(y[r0:r1], (F.silu(g) * u).numpy(), rtol=1e-13, atol=1e-15)
    # swap experts 0 and 2 together with their token rows
    perm = [2, 1, 0, 3]
    rows = np.concatenate([np.arange(offs[e], offs[e + 1]) for e in perm])
    offs2 = np.concatenate([[0], np.cumsum([counts[e] for e in perm])])
    y2, _ = oracle_mod.gemm_grouped(a[rows], sa[rows], 0, [bc[e] for e in perm], [sb[e] for e in perm], 1,
                                    [bias[e] for e in perm], 3, offs2, N, K)
    assert np.array_equal(y2, y[rows])
