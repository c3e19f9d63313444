"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments before touching CUDA (runs without a GPU)."""
import ctypes
import os
import re

import pytest
import torch

import mxfp4_gemm_transformer_b200 as mxg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxgemm.h")

# fake, well-aligned device addresses: validation rejects before using them
A = 0x10000
P = [A * (i + 1) for i in range(16)]


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(mxg.LIB_PATH):
        from mxfp4_gemm_transformer_b200 import build
        build.build()
    return mxg.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mx_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("mx_quant_act", "mx_gemm", "mx_gemm_workspace_size"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(mxg.EXPORTS) == set(declared_functions())


def test_status_strings(lib):
    for s in range(9):
        assert lib.mx_status_string(s).decode().startswith("MX_")


def gemm(lib, **kw):
    args = dict(a=P[0], sa=P[1], af=0, b=P[2], sb=P[3], bf=0, bias=P[4], epi=1, out=P[5],
                M=16, N=256, K=512, ws=P[6], wsb=256, st=None)
    args.update(kw)
    return lib.mx_gemm(args["a"], args["sa"], args["af"], args["b"], args["sb"], args["bf"], args["bias"],
                       args["epi"], args["out"], args["M"], args["N"], args["K"], args["ws"], args["wsb"],
                       args["st"])


def test_gemm_validation(lib):
    assert gemm(lib, a=None) == mxg.MX_ERR_NULL
    assert gemm(lib, out=None) == mxg.MX_ERR_NULL
    assert gemm(lib, bias=None) == mxg.MX_ERR_NULL            # BIAS needs a bias
    assert gemm(lib, epi=0) == mxg.MX_ERR_FORMAT              # NONE must not get one
    assert gemm(lib, epi=9) == mxg.MX_ERR_FORMAT
    assert gemm(lib, af=1, bf=0) == mxg.MX_ERR_FORMAT         # invalid pairing
    assert gemm(lib, af=0, bf=2) == mxg.MX_ERR_FORMAT
    assert gemm(lib, af=7) == mxg.MX_ERR_FORMAT
    assert gemm(lib, sa=None) == mxg.MX_ERR_NULL               # codes need their scales
    assert gemm(lib, af=2, bf=2) == mxg.MX_ERR_FORMAT          # bf16 activations pair with E8M0 weights
    assert gemm(lib, af=2, a=P[0] + 8) == mxg.MX_ERR_ALIGN     # bf16 x: 16-byte aligned
    assert gemm(lib, M=0) == mxg.MX_ERR_SHAPE
    assert gemm(lib, K=48) == mxg.MX_ERR_SHAPE                # K % 32
    assert gemm(lib, K=16) == mxg.MX_ERR_SHAPE
    assert gemm(lib, N=48) == mxg.MX_ERR_SHAPE                # 32x32 blocks need N % 32
    assert gemm(lib, bf=1, K=160) == mxg.MX_ERR_SHAPE         # e2m1 needs K % 128
    assert gemm(lib, epi=3, bias=None, N=96) == mxg.MX_ERR_SHAPE  # SwiGLU needs N % 64
    assert gemm(lib, a=P[0] + 8) == mxg.MX_ERR_ALIGN
    assert gemm(lib, out=P[5] + 4) == mxg.MX_ERR_ALIGN
    assert gemm(lib, bf=1, b=P[2] + 16) == mxg.MX_ERR_ALIGN   # e2m1 codes need 32 B
    assert gemm(lib, ws=None) == mxg.MX_ERR_WORKSPACE
    assert gemm(lib, wsb=8) == mxg.MX_ERR_WORKSPACE


def test_quant_validation(lib):
    assert lib.mx_quant_act(None, 4, 64, P[1], P[2], 0, None) == mxg.MX_ERR_NULL
    assert lib.mx_quant_act(P[0], 4, 48, P[1], P[2], 0, None) == mxg.MX_ERR_SHAPE
    assert lib.mx_quant_act(P[0], 0, 64, P[1], P[2], 0, None) == mxg.MX_ERR_SHAPE
    assert lib.mx_quant_act(P[0], 4, 64, P[1], P[2], 5, None) == mxg.MX_ERR_FORMAT
    assert lib.mx_quant_act(P[0], 4, 64, P[1], P[2], 2, None) == mxg.MX_ERR_FORMAT  # not an output format
    assert lib.mx_quant_act(P[0] + 2, 4, 64, P[1], P[2], 0, None) == mxg.MX_ERR_ALIGN
    assert lib.mx_quant_act(P[0], 4, 64, P[1], P[2] + 2, 1, None) == mxg.MX_ERR_ALIGN
    assert lib.mx_quant_weight(P[0], 48, 64, P[1], P[2], 0, None) == mxg.MX_ERR_SHAPE
    assert lib.mx_quant_weight(P[0], 64, 64, P[1], P[2], 3, None) == mxg.MX_ERR_FORMAT


def test_residual_epilogue_validation(lib):
    # the residual epilogue takes a bias or none
    assert gemm(lib, epi=4, a=None) == mxg.MX_ERR_NULL
    assert gemm(lib, epi=4, out=P[5] + 4) == mxg.MX_ERR_ALIGN


def test_add_rms_quant_validation(lib):
    f = lib.mx_add_rms_quant
    ok = dict(x=P[0], r=P[1], w=P[2], eps=1e-6, M=4, K=64, y=P[3], c=P[4], s=P[5])

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["x"], a["r"], a["w"], a["eps"], a["M"], a["K"], a["y"], a["c"], a["s"], None)
    assert call(x=None) == mxg.MX_ERR_NULL
    assert call(r=None) == mxg.MX_ERR_NULL
    assert call(w=None) == mxg.MX_ERR_NULL
    assert call(c=None) == mxg.MX_ERR_NULL
    assert call(s=None) == mxg.MX_ERR_NULL
    assert call(K=48) == mxg.MX_ERR_SHAPE
    assert call(K=16416) == mxg.MX_ERR_SHAPE
    assert call(M=0) == mxg.MX_ERR_SHAPE
    assert call(eps=-1.0) == mxg.MX_ERR_SHAPE
    assert call(eps=float("nan")) == mxg.MX_ERR_SHAPE
    assert call(x=P[0] + 8) == mxg.MX_ERR_ALIGN
    assert call(y=P[3] + 2) == mxg.MX_ERR_ALIGN
    if not torch.cuda.is_available():
        assert call(y=None) in (mxg.MX_ERR_CUDA, mxg.MX_ERR_ARCH)  # y_out is optional


def test_grouped_validation(lib):
    def call(offs, **kw):
        a = dict(a=P[0], sa=P[1], af=0, b=P[2], sb=P[3], bf=1, bias=None, epi=0, out=P[5], N=256, K=512, ws=P[6],
                 wsb=256)
        a.update(kw)
        arr = None if offs is None else (ctypes.c_int * len(offs))(*offs)
        return lib.mx_gemm_grouped(a["a"], a["sa"], a["af"], a["b"], a["sb"], a["bf"], a["bias"], a["epi"], a["out"],
                                   0 if offs is None else len(offs) - 1, arr, a["N"], a["K"], a["ws"], a["wsb"], None)
    assert call(None) == mxg.MX_ERR_NULL
    assert call([0]) == mxg.MX_ERR_SHAPE                      # no group
    assert call([1, 4]) == mxg.MX_ERR_SHAPE                   # offsets start at 0
    assert call([0, 5, 3]) == mxg.MX_ERR_SHAPE                # decreasing
    assert call([0] * 258) == mxg.MX_ERR_SHAPE                # more than MX_MAX_GROUPS
    assert call([0, 4], af=1, bf=2) == mxg.MX_ERR_FORMAT      # fp32-row formats are not grouped
    assert call([0, 4], af=2) == mxg.MX_ERR_FORMAT            # nor bf16 activations
    assert call([0, 4], epi=5) == mxg.MX_ERR_FORMAT           # nor the MX-code output
    assert call([0, 4], epi=1) == mxg.MX_ERR_NULL             # BIAS needs a bias
    assert call([0, 4], K=160) == mxg.MX_ERR_SHAPE            # e2m1 needs K % 128
    assert call([0, 4], ws=None) == mxg.MX_ERR_WORKSPACE
    assert call([0, 4], out=P[5] + 4) == mxg.MX_ERR_ALIGN
    if not torch.cuda.is_available():
        assert call([0, 4, 4]) in (mxg.MX_ERR_CUDA, mxg.MX_ERR_ARCH)


def test_workspace_size(lib):
    assert lib.mx_gemm_workspace_size(16, 256, 512, 0, 0, 1) >= 4


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error(lib):
    assert gemm(lib) in (mxg.MX_ERR_CUDA, mxg.MX_ERR_ARCH)
    # bf16 activations need no scales pointer: validation passes, the device check fails
    assert gemm(lib, af=2, sa=None) in (mxg.MX_ERR_CUDA, mxg.MX_ERR_ARCH)
    assert lib.mx_quant_act(P[0], 4, 64, P[1], P[2], 0, None) in (mxg.MX_ERR_CUDA, mxg.MX_ERR_ARCH)


def header_constants():
    """Every MX_* enumerator and #define value of include/mxgemm.h."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    vals = {name: int(v) for name, v in re.findall(r"\b(MX_[A-Z0-9_]+)\s*=\s*(\d+)", src)}
    vals.update({name: int(v) for name, v in re.findall(r"#define\s+(MX_[A-Z0-9_]+)\s+(\d+)u?\b", src)})
    return vals


def test_binding_constants_match_the_header():
    hv = header_constants()
    assert len(hv) > 20
    mine = {n: getattr(mxg, n) for n in dir(mxg) if n.startswith("MX_") and isinstance(getattr(mxg, n), int)}
    assert mine, "the binding exports its constants"
    for name, v in mine.items():
        assert name in hv, f"{name} is not in the header"
        assert v == hv[name], f"{name}: binding {v}, header {hv[name]}"
