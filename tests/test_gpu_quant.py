"""Quantisation kernels vs the oracle: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _bits_all_bf16_blocks():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    keep = bits[np.isfinite(f)].astype(np.uint16)
    pad = (-len(keep)) % 32
    return np.concatenate([keep, np.zeros(pad, np.uint16)]).reshape(-1, 32)


def _bf16_tensor(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("M,K", [(16, 512), (1, 7168), (8, 7168), (33, 96), (300, 4096), (16, 5120)])
def test_quant_act_e8m0_bit_exact(mx, M, K):
    x = synth.bf16_matrix(M * 7 + K, M, K, 1.0)
    x[0, :32] = 0
    codes, scales = oracle.quant_act_e8m0(x)
    c, s = mx.act_buffers(M, K)
    mx.mx_quant_act(x.cuda(), c, s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), scales)
    assert np.array_equal(c.cpu().numpy(), codes)


def test_quant_act_every_bf16_pattern(mx):
    bits = _bits_all_bf16_blocks()  # [2048 - ish, 32]: every finite bf16 pattern
    x = _bf16_tensor(bits)
    codes, scales = oracle.quant_act_e8m0(x)
    c, s = mx.act_buffers(bits.shape[0], 32)
    mx.mx_quant_act(x.cuda(), c, s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), scales)
    assert np.array_equal(c.cpu().numpy(), codes)
    # the same patterns as whole rows (a block per 32, with a different max per block)
    x2 = _bf16_tensor(bits.reshape(-1, 256))
    codes2, scales2 = oracle.quant_act_e8m0(x2)
    c2, s2 = mx.act_buffers(x2.shape[0], 256)
    mx.mx_quant_act(x2.cuda(), c2, s2)
    torch.cuda.synchronize()
    assert np.array_equal(c2.cpu().numpy(), codes2) and np.array_equal(s2.cpu().numpy(), scales2)


@pytest.mark.parametrize("M,K", [(16, 5120), (3, 96), (1, 32)])
def test_quant_act_f32_row_bit_exact(mx, M, K):
    x = synth.bf16_matrix(5 + K, M, K, 1.0)
    if M > 1:
        x[1] = 0
    codes, s_ref = oracle.quant_f32_row(x)
    c, s = mx.act_buffers(M, K, mx.MX_A_E4M3_F32_ROW)
    mx.mx_quant_act(x.cuda(), c, s, mx.MX_A_E4M3_F32_ROW)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(c.cpu().numpy(), codes)


@pytest.mark.parametrize("fmt,N,K", [(0, 256, 512), (0, 2048, 7168), (1, 544, 5120), (1, 64, 128),
                                     (2, 300, 5120), (2, 33, 64)])
def test_quant_weight_bit_exact(mx, fmt, N, K):
    w = synth.bf16_matrix(100 + N, N, K, 0.02)
    codes, scales = oracle.quant_weight(w, fmt)
    c, s = mx.weight_buffers(N, K, fmt)
    mx.mx_quant_weight(w.cuda(), c, s, fmt)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), scales)
    assert np.array_equal(c.cpu().numpy(), codes)


def test_quant_weight_e2m1_every_bf16_pattern(mx):
    bits = _bits_all_bf16_blocks()
    rows = bits.reshape(-1, 128)[: (bits.size // 128)]
    w = _bf16_tensor(np.ascontiguousarray(rows))
    codes, scales = oracle.quant_w_e2m1_1x32(w)
    c, s = mx.weight_buffers(w.shape[0], 128, 1)
    mx.mx_quant_weight(w.cuda(), c, s, 1)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), scales)
    assert np.array_equal(c.cpu().numpy(), codes)


@pytest.mark.parametrize("M,K", [(4096, 4096), (4096, 5120)])
def test_quant_act_e8m0_bit_exact_prefill_sizes(mx, M, K):
    # the DiT/ViT MLP and W4A8 gate_up prefill activations: several passes of
    # the kernel's grid-stride loop over the blocks
    x = synth.bf16_matrix(2 if K == 4096 else 3, M, K, synth.X_SIGMA, device="cuda")
    x[M - 1, -32:] = 0
    c, s = mx.act_buffers(M, K)
    mx.mx_quant_act(x, c, s)
    torch.cuda.synchronize()
    codes, scales = oracle.quant_act_e8m0(x.cpu())
    assert np.array_equal(s.cpu().numpy(), scales)
    assert np.array_equal(c.cpu().numpy(), codes)


@pytest.mark.parametrize("fmt,N,K", [(1, 34816, 5120), (0, 34816, 5120), (0, 4096, 4096)])
def test_quant_weight_bit_exact_full_sizes(mx, fmt, N, K):
    # the full gate_up weight as e2m1 and as e4m3 with 32 x 32 blocks (several
    # grid-stride passes of either kernel), and the MLP weight
    seed = 3 if N == 34816 else 2
    w = synth.bf16_matrix(seed + 1, N, K, synth.W_SIGMA, device="cuda")
    c, s = mx.weight_buffers(N, K, fmt)
    mx.mx_quant_weight(w, c, s, fmt)
    torch.cuda.synchronize()
    codes, scales = oracle.quant_weight(w.cpu(), fmt)
    del w
    assert np.array_equal(s.cpu().numpy(), scales)
    assert np.array_equal(c.cpu().numpy(), codes)
