"""fp64 CPU oracle for the block-scaled projection GEMM -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  It loads ``_mxref.so`` (built
from ``mxref.c`` by ``make -C oracle``) and never touches the CUDA library.

Every function here marshals numpy / CPU-torch arrays into the C routines, or
chains them; the arithmetic and its citations live in ``mxref.c``, except the
residual epilogue's one fp64 addition (``gemm_residual``, ViT page ``vt_add``:
x += y + b).

Parity status: every routine is pinned by ``tests/test_oracle_pins.py``
(closed forms checked against torch's CPU fp8 casts, invariants, brute force
against a dequantise-then-matmul on tiny shapes, library GELU / SiLU).  The
pages print no worked numeric example for the GEMM itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

A_E8M0_1X32, A_F32_ROW, A_E2M1_1X32 = 0, 1, 3
B_E4M3_32X32, B_E2M1_1X32, B_E4M3_F32_ROW = 0, 1, 2
EPI_NONE, EPI_BIAS, EPI_BIAS_GELU_TANH, EPI_SWIGLU = 0, 1, 2, 3


def build() -> str:
    """Compile ``_mxref.so`` with the system gcc (OpenMP)."""
    subprocess.run(["make", "-s", "-C", _HERE, "CC=gcc"], check=True)
    return os.path.join(_HERE, "_mxref.so")


def _signatures():
    P = ctypes.c_void_p
    I = ctypes.c_int
    D = ctypes.c_double
    U = ctypes.c_uint
    Z = ctypes.c_size_t
    return [
        ("mxr_e4m3_value", D, [U]), ("mxr_e2m1_value", D, [U]), ("mxr_e8m0_value", D, [U]),
        ("mxr_rne_e4m3", U, [D]), ("mxr_rne_e2m1", U, [D]),
        ("mxr_e8m0_for_amax", U, [D, D]),
        ("mxr_quant_act_e8m0", None, [P, I, I, P, P]),
        ("mxr_quant_f32_row", None, [P, I, I, P, P]),
        ("mxr_quant_w_e4m3_32x32", None, [P, I, I, P, P]),
        ("mxr_quant_w_e2m1_1x32", None, [P, I, I, P, P]),
        ("mxr_gemm", None, [P, P, I, P, P, I, P, I, I, I, I, P, P, P]),
        ("mxr_gelu_tanh", D, [D]), ("mxr_silu", D, [D]), ("mxr_silu_grad", D, [D]),
        ("mxr_bf16_rne", U, [D]), ("mxr_round_bf16", None, [P, Z, P]),
        ("mxr_add_bf16", None, [P, P, Z, P]),
        ("mxr_rmsnorm_bf16", None, [P, P, I, I, D, P]),
    ]


def load_library(path: str):
    """ctypes handle of an oracle library built from mxref.c (the tests also
    load copies with a planted mistake, to show that the pins catch it)."""
    L = ctypes.CDLL(path)
    for name, res, args in _signatures():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


def lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(_HERE, "_mxref.so")
        src = os.path.join(_HERE, "mxref.c")
        if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(src):
            build()
        _LIB = load_library(path)
    return _LIB


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x) -> np.ndarray:
    """bf16 tensor (CPU torch) or uint16 array -> contiguous uint16 numpy."""
    if isinstance(x, torch.Tensor):
        assert x.dtype == torch.bfloat16
        return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    return np.ascontiguousarray(x, dtype=np.uint16)


# ---- scalar codecs ----------------------------------------------------------

def e4m3_value(c: int) -> float:
    return lib().mxr_e4m3_value(c)


def e2m1_value(c: int) -> float:
    return lib().mxr_e2m1_value(c)


def e8m0_value(e: int) -> float:
    return lib().mxr_e8m0_value(e)


def rne_e4m3(v: float) -> int:
    return lib().mxr_rne_e4m3(v)


def rne_e2m1(v: float) -> int:
    return lib().mxr_rne_e2m1(v)


def e8m0_for_amax(amax: float, fmax: float) -> int:
    return lib().mxr_e8m0_for_amax(amax, fmax)


# ---- quantisers -------------------------------------------------------------

def quant_act_e8m0(x):
    """bf16 [M, K] -> (codes uint8 [M, K], scales uint8 [M, K/32])."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    codes = np.empty((M, K), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    lib().mxr_quant_act_e8m0(_ptr(xb), M, K, _ptr(codes), _ptr(scales))
    return codes, scales


def quant_f32_row(x):
    """bf16 [R, K] -> (codes uint8 [R, K], fp32 scale per row [R])."""
    xb = _bf16_bits(x)
    R, K = xb.shape
    codes = np.empty((R, K), np.uint8)
    s = np.empty((R,), np.float32)
    lib().mxr_quant_f32_row(_ptr(xb), R, K, _ptr(codes), _ptr(s))
    return codes, s


def quant_w_e4m3_32x32(w):
    """bf16 [N, K] -> (codes uint8 [N, K], scales uint8 [N/32, K/32])."""
    wb = _bf16_bits(w)
    N, K = wb.shape
    codes = np.empty((N, K), np.uint8)
    scales = np.empty((N // 32, K // 32), np.uint8)
    lib().mxr_quant_w_e4m3_32x32(_ptr(wb), N, K, _ptr(codes), _ptr(scales))
    return codes, scales


def quant_w_e2m1_1x32(w):
    """bf16 [N, K] -> (packed uint8 [N, K/2], scales uint8 [N, K/32])."""
    wb = _bf16_bits(w)
    N, K = wb.shape
    packed = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // 32), np.uint8)
    lib().mxr_quant_w_e2m1_1x32(_ptr(wb), N, K, _ptr(packed), _ptr(scales))
    return packed, scales


def quant_weight(w, b_fmt: int):
    if b_fmt == B_E4M3_32X32:
        return quant_w_e4m3_32x32(w)
    if b_fmt == B_E2M1_1X32:
        return quant_w_e2m1_1x32(w)
    if b_fmt == B_E4M3_F32_ROW:
        return quant_f32_row(w)
    raise ValueError(b_fmt)


def quant_act_e2m1(x):
    """bf16 [M, K] -> (packed e2m1 codes uint8 [M, K/2], E8M0 scales [M, K/32]):
    the W4A4 activation operand, by the 1 x 32 e2m1 rule of the weights."""
    return quant_w_e2m1_1x32(x)


def quant_act(x, a_fmt: int):
    if a_fmt == A_E2M1_1X32:
        return quant_act_e2m1(x)
    return quant_act_e8m0(x) if a_fmt == A_E8M0_1X32 else quant_f32_row(x)


# ---- the GEMM ---------------------------------------------------------------

def gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, M, N, K,
         want_acc=False):
    """fp64 y [M, Nout] and tolerance term T [M, Nout] (and optionally the raw
    accumulators [M, N])."""
    a = np.ascontiguousarray(a_codes, np.uint8)
    b = np.ascontiguousarray(b_codes, np.uint8)
    if a_fmt == A_F32_ROW:
        sa = np.ascontiguousarray(a_scales, np.float32)
        sb = np.ascontiguousarray(b_scales, np.float32)
    else:
        sa = np.ascontiguousarray(a_scales, np.uint8)
        sb = np.ascontiguousarray(b_scales, np.uint8)
    bias_np = None if bias is None else np.ascontiguousarray(
        bias.detach().cpu().numpy() if isinstance(bias, torch.Tensor) else bias, np.float32)
    nout = N // 2 if epi == EPI_SWIGLU else N
    y = np.empty((M, nout), np.float64)
    t = np.empty((M, nout), np.float64)
    acc = np.empty((M, N), np.float64) if want_acc else None
    lib().mxr_gemm(_ptr(a), _ptr(sa), a_fmt, _ptr(b), _ptr(sb), b_fmt,
                   None if bias_np is None else _ptr(bias_np), epi, M, N, K,
                   _ptr(y), _ptr(t), None if acc is None else _ptr(acc))
    return (y, t, acc) if want_acc else (y, t)


# ---- producers that emit MX codes (quantisation fused into the step before) ---

def bf16_rne(v: float) -> int:
    """bf16 bits of v rounded once, to nearest even."""
    return lib().mxr_bf16_rne(v)


def round_bf16(v) -> np.ndarray:
    """fp64 array -> bf16 bits (uint16), same shape."""
    v = np.ascontiguousarray(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().mxr_round_bf16(_ptr(v), v.size, _ptr(out))
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def add_bf16(x, r) -> np.ndarray:
    """Residual add bf16(x + r) -> bf16 bits."""
    xb, rb = _bf16_bits(x), _bf16_bits(r)
    assert xb.shape == rb.shape
    out = np.empty(xb.shape, np.uint16)
    lib().mxr_add_bf16(_ptr(xb), _ptr(rb), xb.size, _ptr(out))
    return out


def rmsnorm_bf16(v, w, eps: float) -> np.ndarray:
    """RMSNorm with a plain weight, rows of v [M, K], w [K] -> bf16 bits [M, K]."""
    vb, wb = _bf16_bits(v), _bf16_bits(w)
    M, K = vb.shape
    assert wb.shape == (K,)
    y = np.empty((M, K), np.uint16)
    lib().mxr_rmsnorm_bf16(_ptr(vb), _ptr(wb), M, K, float(eps), _ptr(y))
    return y


def add_rms_quant(x, r, w, eps: float):
    """Residual add, RMSNorm and MX quantisation of the normalised rows, read as
    the unfused chain: (residual_out bf16 bits [M, K], y bf16 bits [M, K],
    codes [M, K], E8M0 scales [M, K/32])."""
    res = add_bf16(x, r)
    y = rmsnorm_bf16(res, w, eps)
    codes, scales = quant_act_e8m0(y)
    return res, y, codes, scales


def gemm_swiglu_mxq(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, M, N, K):
    """The SwiGLU GEMM with its output handed on as MX codes, read as the unfused
    chain: bf16(y) of the SwiGLU epilogue, then the activation quantisation.
    Returns (y bf16 bits [M, N/2], codes [M, N/2], E8M0 scales [M, N/64]) and
    the fp64 y with its tolerance term."""
    y, t = gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, EPI_SWIGLU, M, N, K)
    yb = round_bf16(y)
    codes, scales = quant_act_e8m0(yb)
    return yb, codes, scales, y, t


def gemm_grouped(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, offsets, N, K):
    """Grouped GEMM (routed experts, vLLM DeepSeek-V4 mono runner page, MoE
    weights: w13 [experts, 2 inter, hidden/2] and w2 [experts, hidden, inter/2]
    e2m1 with per-expert 1 x 32 scales): the tokens are sorted by expert, rows
    offsets[g] .. offsets[g+1]-1 of A go through expert g's weights
    b_codes[g] / b_scales[g] (and bias[g] if given), each group by ``gemm``.
    Returns y and T over all rows [offsets[-1], Nout]."""
    G = len(offsets) - 1
    nout = N // 2 if epi == EPI_SWIGLU else N
    M = int(offsets[-1])
    y = np.zeros((M, nout), np.float64)
    t = np.zeros((M, nout), np.float64)
    for g in range(G):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 == r0:
            continue
        yg, tg = gemm(np.ascontiguousarray(a_codes[r0:r1]), np.ascontiguousarray(a_scales[r0:r1]), a_fmt,
                      b_codes[g], b_scales[g], b_fmt, None if bias is None else bias[g], epi, r1 - r0, N, K)
        y[r0:r1], t[r0:r1] = yg, tg
    return y, t


def gemm_residual(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, residual, M, N, K):
    """The residual epilogue out = res + (acc + b) (ViT page, vt_add: x += y + b),
    in fp64 before the one bf16 rounding of the output; the tolerance term is
    the GEMM's (the residual is added exactly).  residual: bf16 [M, N]."""
    y, t = gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias,
                EPI_BIAS if bias is not None else EPI_NONE, M, N, K)
    return bf16_bits_to_f64(_bf16_bits(residual)).reshape(M, N) + y, t


def gelu_tanh(v: float) -> float:
    return lib().mxr_gelu_tanh(v)


def silu(v: float) -> float:
    return lib().mxr_silu(v)


def silu_grad(v: float) -> float:
    """The SiLU derivative the SwiGLU tolerance term uses."""
    return lib().mxr_silu_grad(v)


# Absolute floor of the bf16 output rounding: below bf16's normal range
# (2^-126) its values are 2^-133 apart, so the relative 2^-8 |y| no longer
# bounds the rounding of the output.
BF16_FLOOR = 2.0 ** -133


def tolerance_bound(y_ref, t_ref):
    """2^-8 |y| (the bf16 output rounding, with its subnormal floor) + 1e-5 T
    (fp32 accumulation-order slack)."""
    return 2.0 ** -8 * np.abs(y_ref) + 1e-5 * t_ref + BF16_FLOOR


def within_tolerance(y_gpu, y_ref, t_ref):
    """Acceptance bound |y_gpu - y| <= 2^-8 |y| + 1e-5 T (+ 2^-133 below the
    bf16 normal range), elementwise."""
    y_gpu = np.asarray(y_gpu, np.float64)
    return np.abs(y_gpu - y_ref) <= tolerance_bound(y_ref, t_ref)
