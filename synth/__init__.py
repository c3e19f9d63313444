"""Seeded synthetic inputs shared by the oracle checks, the GPU tests and the bench.

This module holds no arithmetic of the block-scaled GEMM itself: it only draws
the bf16 activations, bf16 weights and fp32 biases that both sides are fed.

Generator (counter based, so any row of any matrix can be regenerated alone):

* ``u64(seed, i)`` is output ``i`` (0-based) of SplitMix64 (Steele, Lea and
  Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) whose
  state starts at ``key(seed) = mix64(seed)``: ``mix64(key + (i + 1) * gamma)``
  with ``gamma = 0x9E3779B97F4A7C15`` and the published ``mix64`` finaliser.
* Element ``e`` of a normal stream takes ``r0 = u64(seed, 2e)`` and
  ``r1 = u64(seed, 2e + 1)``; ``u1 = ((r0 >> 11) + 1) 2^-53`` in (0, 1],
  ``u2 = (r1 >> 11) 2^-53`` in [0, 1) and ``z = sqrt(-2 ln u1) cos(2 pi u2)``
  (Box and Muller, 1958), all in fp64.
* A matrix value is ``bf16(fp32(sigma * z))``: fp64 -> fp32 -> bf16, each step
  round-to-nearest-even. Element (r, c) of a rows x cols matrix is stream index
  ``r * cols + c``.

The same code runs on CPU or CUDA tensors (torch int64 arithmetic wraps modulo
2^64; the CPU tests pin it against Python's unbounded integers).
"""
from __future__ import annotations

import math

import torch

_MASK64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def _s64(v: int) -> int:
    """Two's-complement view of a 64-bit unsigned constant as a Python int."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def mix64_int(z: int) -> int:
    """SplitMix64 finaliser on Python ints (the plain reference used by tests)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def u64_int(seed: int, i: int) -> int:
    """Output i of the stream for ``seed`` on Python ints."""
    key = mix64_int(seed)
    return mix64_int(key + (i + 1) * _GAMMA)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor holding 64-bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def u64(seed: int, idx: torch.Tensor) -> torch.Tensor:
    """Stream outputs for int64 counters ``idx`` (bit patterns in int64)."""
    key = _s64(mix64_int(seed))
    return _mix64(key + (idx + 1) * _s64(_GAMMA))


def normal_f64(seed: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """fp64 standard normals for stream elements [start, start + count)."""
    e = torch.arange(start, start + count, dtype=torch.int64, device=device)
    return normal_f64_at(seed, e)


def normal_f64_at(seed: int, e: torch.Tensor) -> torch.Tensor:
    """fp64 standard normals for the stream elements listed in ``e`` (int64)."""
    r0 = u64(seed, 2 * e)
    r1 = u64(seed, 2 * e + 1)
    u1 = (_lsr(r0, 11) + 1).to(torch.float64) * 2.0 ** -53
    u2 = _lsr(r1, 11).to(torch.float64) * 2.0 ** -53
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def bf16_matrix(seed: int, rows: int, cols: int, sigma: float, row0: int = 0,
                nrows: int | None = None, device="cpu",
                chunk: int = 1 << 24) -> torch.Tensor:
    """Rows [row0, row0 + nrows) of the seeded rows x cols bf16 matrix."""
    if nrows is None:
        nrows = rows - row0
    assert 0 <= row0 and row0 + nrows <= rows
    out = torch.empty(nrows * cols, dtype=torch.bfloat16, device=device)
    base = row0 * cols
    total = nrows * cols
    for s in range(0, total, chunk):
        n = min(chunk, total - s)
        z = normal_f64(seed, base + s, n, device) * sigma
        out[s:s + n] = z.to(torch.float32).to(torch.bfloat16)
    return out.view(nrows, cols)


def bf16_rows(seed: int, cols: int, sigma: float, row_ids, device="cpu",
              chunk: int = 1 << 24) -> torch.Tensor:
    """Selected rows (any order) of a seeded matrix with ``cols`` columns."""
    ids = torch.as_tensor([int(r) for r in row_ids], dtype=torch.int64, device=device)
    out = torch.empty(len(ids) * cols, dtype=torch.bfloat16, device=device)
    per = max(1, chunk // cols)
    col = torch.arange(cols, dtype=torch.int64, device=device)
    for i in range(0, len(ids), per):
        r = ids[i:i + per]
        z = normal_f64_at(seed, (r[:, None] * cols + col[None, :]).reshape(-1)) * sigma
        out[i * cols:(i + len(r)) * cols] = z.to(torch.float32).to(torch.bfloat16)
    return out.view(len(ids), cols)


def f32_vector(seed: int, n: int, sigma: float, device="cpu") -> torch.Tensor:
    """Seeded fp32 vector (biases): fp32(sigma * z)."""
    return (normal_f64(seed, 0, n, device) * sigma).to(torch.float32)


# Value distributions of the workloads: activations ~N(0, 1), weights
# ~N(0, 0.02) before quantisation, biases ~N(0, 0.1) in fp32.
X_SIGMA = 1.0
W_SIGMA = 0.02
BIAS_SIGMA = 0.1


def problem(seed: int, M: int, N: int, K: int, device="cpu", with_bias=True):
    """The seeded (x, W, bias) triple: x seed s, W seed s+1, bias seed s+2."""
    x = bf16_matrix(seed, M, K, X_SIGMA, device=device)
    w = bf16_matrix(seed + 1, N, K, W_SIGMA, device=device)
    b = f32_vector(seed + 2, N, BIAS_SIGMA, device=device) if with_bias else None
    return x, w, b
