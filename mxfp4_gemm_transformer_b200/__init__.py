"""Python binding of libmxgemm.so (block-scaled projection GEMM for B200).

The functions carry the C ABI's names (include/mxgemm.h) and only marshal
arguments: torch tensors give their device pointers, the stream defaults to
torch's current stream, and a non-OK status raises MxError.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback -- if the
library is missing the import of a function fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxgemm.so")

# formats and epilogues (values of the C enums)
MX_A_E4M3_E8M0_1X32, MX_A_E4M3_F32_ROW, MX_A_BF16_E8M0_1X32, MX_A_E2M1_E8M0_1X32 = 0, 1, 2, 3
MX_B_E4M3_E8M0_32X32, MX_B_E2M1_E8M0_1X32, MX_B_E4M3_F32_ROW = 0, 1, 2
MX_EPI_NONE, MX_EPI_BIAS, MX_EPI_BIAS_GELU_TANH, MX_EPI_SWIGLU, MX_EPI_RESIDUAL = 0, 1, 2, 3, 4
MX_EPI_SWIGLU_MXQ = 5

MX_LAUNCH_PDL, MX_LAUNCH_PREFETCH_WEIGHTS, MX_LAUNCH_DETERMINISTIC = 1, 2, 4
MX_TUNE_BM_PAIR = 2  # mx_set_tuning block_m: 256 x 240 tiles over CTA pairs
MX_MAX_GROUPS = 256  # groups one mx_gemm_grouped call takes

MX_OK, MX_ERR_NULL, MX_ERR_SHAPE, MX_ERR_ALIGN, MX_ERR_FORMAT = 0, 1, 2, 3, 4
MX_ERR_WORKSPACE, MX_ERR_ARCH, MX_ERR_CUDA, MX_ERR_TIMEOUT = 5, 6, 7, 8

EXPORTS = ["mx_quant_act", "mx_quant_weight", "mx_add_rms_quant", "mx_gemm_grouped", "mx_gemm_workspace_size", "mx_gemm", "mx_status_string",
           "mx_workspace_status", "mx_debug_watchdog", "mx_set_tuning", "mx_gemm_plan", "mx_gemm_noalloc",
           "mx_debug_set_timeline", "mx_set_launch_flags", "mx_set_decode_tuning", "mx_gemm_plan_info"]

_lib = None


class PlanInfo(ctypes.Structure):
    """Mirror of the C struct mx_plan_info (include/mxgemm.h)."""
    _fields_ = [("kernel", ctypes.c_int), ("block_m", ctypes.c_int), ("block_n", ctypes.c_int),
                ("splits", ctypes.c_int), ("k_reduction", ctypes.c_int), ("grid", ctypes.c_int),
                ("acc_bufs", ctypes.c_int), ("stages", ctypes.c_int), ("tiles", ctypes.c_int),
                ("ws_bytes", ctypes.c_size_t), ("ctas_per_sm", ctypes.c_int), ("act_quant", ctypes.c_int)]


K_REDUCTION = {0: "none", 1: "cluster", 2: "workspace", 3: "workspace-atomic"}


class MxError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load(path: str | None = None):
    """Load (once) and return the ctypes handle of libmxgemm.so."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m mxfp4_gemm_transformer_b200.build`")
    L = ctypes.CDLL(path)
    P, I, U, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
    IP = ctypes.POINTER(ctypes.c_int)
    sig = {
        "mx_quant_act": (I, [P, I, I, P, P, I, P]),
        "mx_quant_weight": (I, [P, I, I, P, P, I, P]),
        "mx_add_rms_quant": (I, [P, P, P, ctypes.c_float, I, I, P, P, P, P]),
        "mx_gemm_workspace_size": (S, [I, I, I, I, I, I]),
        "mx_gemm": (I, [P, P, I, P, P, I, P, I, P, I, I, I, P, S, P]),
        "mx_status_string": (ctypes.c_char_p, [I]),
        "mx_workspace_status": (I, [P, P]),
        "mx_debug_watchdog": (I, [P, S, U, P]),
        "mx_set_tuning": (None, [I, I, I, I]),
        "mx_gemm_plan": (I, [I, I, I, I, I, I, IP, IP, IP, IP]),
        "mx_gemm_noalloc": (I, [P, P, I, P, P, I, P, I, P, I, I, I, P]),
        "mx_gemm_grouped": (I, [P, P, I, P, P, I, P, I, P, I, IP, I, I, P, S, P]),
        "mx_debug_set_timeline": (None, [P, S]),
        "mx_set_launch_flags": (None, [U]),
        "mx_set_decode_tuning": (None, [I, I, I, I, I, I]),
        "mx_gemm_plan_info": (I, [I, I, I, I, I, I, S, ctypes.POINTER(PlanInfo)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != MX_OK:
        raise MxError(status, where)


def status_string(status: int) -> str:
    return load().mx_status_string(status).decode()


def mx_status_string(status: int) -> str:
    return status_string(status)


def mx_quant_act(x, codes, scales, fmt=MX_A_E4M3_E8M0_1X32, stream=None):
    """x bf16 [M, K] -> codes uint8 [M, K] and scales (uint8 [M, K/32] or fp32 [M])."""
    M, K = x.shape
    _check(load().mx_quant_act(_p(x), M, K, _p(codes), _p(scales), fmt, _stream(stream)), "mx_quant_act")


def mx_quant_weight(w, codes, scales, fmt, stream=None):
    """w bf16 [N, K] -> weight codes and scales in the chosen B format."""
    N, K = w.shape
    _check(load().mx_quant_weight(_p(w), N, K, _p(codes), _p(scales), fmt, _stream(stream)), "mx_quant_weight")


def mx_add_rms_quant(x, residual, w, eps, y_out, codes, scales, stream=None):
    """residual <- bf16(x + residual); y = bf16(RMSNorm(residual) * w) into
    y_out (None = not wanted); codes / scales = its 1 x 32 E8M0 quantisation."""
    M, K = x.shape
    _check(load().mx_add_rms_quant(_p(x), _p(residual), _p(w), float(eps), M, K, _p(y_out), _p(codes), _p(scales),
                                   _stream(stream)), "mx_add_rms_quant")


def mx_gemm_workspace_size(M, N, K, a_fmt, b_fmt, epi) -> int:
    return int(load().mx_gemm_workspace_size(M, N, K, a_fmt, b_fmt, epi))


def mx_gemm(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M, N, K, workspace,
            ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().mx_gemm(_p(a_codes), _p(a_scales), a_fmt, _p(b_codes), _p(b_scales), b_fmt, _p(bias), epi,
                          _p(out), M, N, K, _p(workspace), ws_bytes, _stream(stream)), "mx_gemm")


def mx_gemm_grouped(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, offsets, N, K, workspace,
                    ws_bytes=None, stream=None):
    """Grouped GEMM over routed experts: rows offsets[g] .. offsets[g+1]-1 of
    the activations through group g's weights (b_codes / b_scales hold every
    group's rows back to back, bias is [groups, N] or None); offsets is a host
    sequence of groups + 1 ints."""
    offs = [int(o) for o in offsets]
    arr = (ctypes.c_int * len(offs))(*offs)
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().mx_gemm_grouped(_p(a_codes), _p(a_scales), a_fmt, _p(b_codes), _p(b_scales), b_fmt, _p(bias), epi,
                                  _p(out), len(offs) - 1, arr, N, K, _p(workspace), ws_bytes, _stream(stream)),
           "mx_gemm_grouped")


def mx_gemm_noalloc(a_codes, a_scales, a_fmt, b_codes, b_scales, b_fmt, bias, epi, out, M, N, K, stream=None):
    """mx_gemm without a workspace, for callers that cannot allocate device
    memory (see include/mxgemm.h); the library's own scratch is used."""
    _check(load().mx_gemm_noalloc(_p(a_codes), _p(a_scales), a_fmt, _p(b_codes), _p(b_scales), b_fmt, _p(bias),
                                  epi, _p(out), M, N, K, _stream(stream)), "mx_gemm_noalloc")


def mx_gemm_status(*args) -> int:
    """Same as mx_gemm but returns the status code instead of raising."""
    a = list(args)
    return load().mx_gemm(*a)


def mx_workspace_status(workspace, stream=None) -> int:
    return load().mx_workspace_status(_p(workspace), _stream(stream))


def mx_debug_watchdog(workspace, timeout_us: int, stream=None) -> int:
    ws_bytes = workspace.numel() * workspace.element_size()
    return load().mx_debug_watchdog(_p(workspace), ws_bytes, timeout_us, _stream(stream))


def mx_debug_set_timeline(buffer=None):
    """Install a uint64 device tensor as the per-CTA stamp buffer (None = off)."""
    if buffer is None:
        load().mx_debug_set_timeline(None, 0)
    else:
        load().mx_debug_set_timeline(_p(buffer), buffer.numel() * buffer.element_size())


def mx_set_launch_flags(flags: int):
    """Process-wide launch options (MX_LAUNCH_PDL, MX_LAUNCH_PREFETCH_WEIGHTS)."""
    load().mx_set_launch_flags(flags)


def mx_set_tuning(block_n: int = 0, splits: int = 0, max_ctas: int = 0, block_m: int = 0):
    load().mx_set_tuning(block_n, splits, max_ctas, block_m)


DEC_SPLIT_AUTO, DEC_SPLIT_CLUSTER, DEC_SPLIT_STREAM_K, DEC_SPLIT_WHOLE_TILES = 0, 1, 2, 3


def mx_set_decode_tuning(mode: int = 0, ctas: int = 0, ctas_per_sm: int = 0, prefetch_stages: int = 0,
                         split: int = 0, cluster_size: int = 0):
    """Decode kernel choice: 0 automatic, 1 whenever it can run, -1 never;
    ctas = its grid size (0 = one CTA per SM); ctas_per_sm = its shared-memory
    budget (2: two CTAs per SM, 1: one with a deep weight ring, 0: choose);
    prefetch_stages = weight stages a CTA may request before the previous
    kernel completes (with MX_LAUNCH_PREFETCH_WEIGHTS; 0 = its whole ring);
    split = DEC_SPLIT_* (how a tile's K range is shared between CTAs);
    cluster_size = CTAs per cluster (0 = fill the SMs)."""
    load().mx_set_decode_tuning(mode, ctas, ctas_per_sm, prefetch_stages, split, cluster_size)


def mx_gemm_plan_info(M, N, K, a_fmt, b_fmt, epi, ws_bytes=None):
    """The plan mx_gemm would choose with `ws_bytes` of workspace (None = as
    much as its fastest plan wants), as a dict."""
    info = PlanInfo()
    wsb = ctypes.c_size_t(-1).value if ws_bytes is None else ws_bytes
    _check(load().mx_gemm_plan_info(M, N, K, a_fmt, b_fmt, epi, wsb, ctypes.byref(info)), "mx_gemm_plan_info")
    d = {name: getattr(info, name) for name, _ in PlanInfo._fields_}
    d["kernel"] = {1: "decode", 3: "pair"}.get(info.kernel, "tile")
    d["k_reduction"] = K_REDUCTION.get(info.k_reduction, str(info.k_reduction))
    return d


def mx_gemm_plan(M, N, K, a_fmt, b_fmt, epi):
    vals = [ctypes.c_int() for _ in range(4)]
    _check(load().mx_gemm_plan(M, N, K, a_fmt, b_fmt, epi, *[ctypes.byref(v) for v in vals]), "mx_gemm_plan")
    return {"block_n": vals[0].value, "splits": vals[1].value, "grid": vals[2].value, "acc_bufs": vals[3].value}


# ---- allocation helpers (torch is the allocator) ---------------------------------

def act_buffers(M, K, fmt=MX_A_E4M3_E8M0_1X32, device="cuda"):
    if fmt == MX_A_E2M1_E8M0_1X32:
        return (torch.empty(M, K // 2, dtype=torch.uint8, device=device),
                torch.empty(M, K // 32, dtype=torch.uint8, device=device))
    codes = torch.empty(M, K, dtype=torch.uint8, device=device)
    if fmt == MX_A_E4M3_E8M0_1X32:
        scales = torch.empty(M, K // 32, dtype=torch.uint8, device=device)
    else:
        scales = torch.empty(M, dtype=torch.float32, device=device)
    return codes, scales


def weight_buffers(N, K, fmt, device="cuda"):
    if fmt == MX_B_E4M3_E8M0_32X32:
        return (torch.empty(N, K, dtype=torch.uint8, device=device),
                torch.empty(N // 32, K // 32, dtype=torch.uint8, device=device))
    if fmt == MX_B_E2M1_E8M0_1X32:
        return (torch.empty(N, K // 2, dtype=torch.uint8, device=device),
                torch.empty(N, K // 32, dtype=torch.uint8, device=device))
    return (torch.empty(N, K, dtype=torch.uint8, device=device),
            torch.empty(N, dtype=torch.float32, device=device))


def workspace(M=1, N=1, K=32, a_fmt=0, b_fmt=0, epi=0, device="cuda", problems=()):
    """A zero-filled workspace for the problem (M, N, K, a_fmt, b_fmt, epi), or
    for the largest of `problems` (tuples of the same six values) if given.
    The default sizes give the 256-byte minimum."""
    probs = list(problems) or [(M, N, K, a_fmt, b_fmt, epi)]
    n = max(mx_gemm_workspace_size(*pr) for pr in probs)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def out_buffer(M, N, epi, device="cuda"):
    """The output of mx_gemm: bf16 [M, N] ([M, N/2] for SwiGLU); for
    MX_EPI_SWIGLU_MXQ the bytes of e4m3 codes [M, N/2] and E8M0 scales
    [M, N/64] (split it with mxq_views)."""
    if epi == MX_EPI_SWIGLU_MXQ:
        return torch.empty(M * (N // 2) + M * (N // 64), dtype=torch.uint8, device=device)
    return torch.empty(M, N // 2 if epi == MX_EPI_SWIGLU else N, dtype=torch.bfloat16, device=device)


def mxq_views(out, M, N):
    """(codes [M, N/2], scales [M, N/64]) views of an MX_EPI_SWIGLU_MXQ output."""
    nc = M * (N // 2)
    return out[:nc].view(M, N // 2), out[nc:nc + M * (N // 64)].view(M, N // 64)
