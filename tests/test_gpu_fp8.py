"""GPU parity: FP8 E4M3 block-128 linear and the fused shared-expert FFN."""
import numpy as np
import pytest
import torch

import block_quantized_expert_mxfp4_b200 as qk
import oracle
from block_quantized_expert_mxfp4_b200 import synth, workload
from helpers import assert_parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N", [(8, 4096, 2048), (3, 2048, 4096), (20, 512, 256),
                                   (1, 128, 16), (8, 384, 144)])
def test_fp8_block_linear(M, K, N):
    w = synth.fp8_codes(3, M + K, N * K, "cuda").view(N, K)
    s = synth.scale_codes(3, N + K, ((N + 127) // 128) * (K // 128), 118, 127, "cuda").view(
        (N + 127) // 128, K // 128)
    x = synth.activations(M, M, K)
    y = torch.empty((M, N), device="cuda")
    qk.fp8_block_linear(x.cuda(), w, s, y)
    assert qk.qk_last_device_status() == qk.QK_OK
    yo = oracle.fp8_block_linear(x, w.cpu(), s.cpu(), 128)
    assert_parity(y.cpu().numpy(), yo, what=f"fp8 linear {M}x{K}x{N}")


def test_fp8_block_linear_bf16_out():
    M, K, N = 8, 1024, 512
    w = synth.fp8_codes(4, 1, N * K, "cuda").view(N, K)
    s = synth.scale_codes(4, 2, (N // 128) * (K // 128), 118, 127, "cuda").view(N // 128, K // 128)
    x = synth.activations(4, M, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qk.fp8_block_linear(x.cuda(), w, s, y)
    assert_parity(y.float().cpu().numpy(), oracle.fp8_block_linear(x, w.cpu(), s.cpu()),
                  what="fp8 bf16")


@pytest.mark.parametrize("M", [8, 1, 13])
def test_fp8_shared_expert_accumulates(M):
    H, I = 4096, 2048
    sh = workload.make_fp8_shared(0, 0, H, I)
    x = synth.activations(11, M, H)
    y0 = torch.from_numpy(np.random.default_rng(M).standard_normal((M, H)).astype(np.float32))
    y = y0.cuda().clone()
    ws = torch.empty(qk.fp8_shared_expert_workspace_size(M, H, I), dtype=torch.uint8, device="cuda")
    qk.fp8_shared_expert_forward(x.cuda(), sh.wg, sh.sg, sh.wu, sh.su, sh.wd, sh.sd, y, ws)
    assert qk.qk_last_device_status() == qk.QK_OK
    so = oracle.fp8_swiglu_ffn(x, *(t.cpu() for t in (sh.wg, sh.sg, sh.wu, sh.su, sh.wd, sh.sd)))
    assert_parity((y.cpu() - y0).numpy(), so, what=f"shared expert M={M}")


@pytest.mark.parametrize("M,K,N", [(8, 4096, 2048), (3, 512, 96), (1, 128, 16)])
def test_fp8_block_linear_32x32_tiles(M, K, N):
    """32x32 E8M0 tiles (the DeepSeek-V4.1 layout)."""
    w = synth.fp8_codes(5, M + K, N * K, "cuda").view(N, K)
    s = synth.scale_codes(5, N + K, ((N + 31) // 32) * (K // 32), 118, 127, "cuda").view((N + 31) // 32, K // 32)
    x = synth.activations(M + 1, M, K)
    y = torch.empty((M, N), device="cuda")
    qk.fp8_block_linear(x.cuda(), w, s, y, scale_block=32)
    assert qk.qk_last_device_status() == qk.QK_OK
    yo = oracle.fp8_block_linear(x, w.cpu(), s.cpu(), 32)
    assert_parity(y.cpu().numpy(), yo, what=f"fp8 linear 32x32 {M}x{K}x{N}")


@pytest.mark.parametrize("M", [8, 1])
def test_fp8_shared_expert_32x32_tiles(M):
    H, I = 4096, 2048
    sh = workload.make_fp8_shared(1, 0, H, I, block=32)
    x = synth.activations(12, M, H)
    y = torch.zeros((M, H), device="cuda")
    ws = torch.empty(qk.fp8_shared_expert_workspace_size(M, H, I), dtype=torch.uint8, device="cuda")
    qk.fp8_shared_expert_forward(x.cuda(), sh.wg, sh.sg, sh.wu, sh.su, sh.wd, sh.sd, y, ws, scale_block=32)
    assert qk.qk_last_device_status() == qk.QK_OK
    hs = workload.make_fp8_shared(1, 0, H, I, device="cpu", block=32)
    so = oracle.fp8_swiglu_ffn(x, hs.wg, hs.sg, hs.wu, hs.su, hs.wd, hs.sd, block=32)
    assert_parity(y.cpu().numpy(), so, what=f"shared expert 32x32 M={M}")


@pytest.mark.parametrize("M,block", [(200, 128), (200, 32), (2048, 128)])
def test_fp8_shared_expert_large_m_block_scaled(M, block):
    """From 128 rows the shared expert runs on the block-scaled grouped GEMMs
    (e4m3 weights as stored, tile scales expanded to per-32 codes): 200 rows
    (ragged token tiles: 3 x 64 + 8 for gate/up, 5 x 40 for down) checked
    whole, 2048 rows (the prefill size) on 64 rows spread over every tile;
    the result is added into y."""
    H, I = 4096, 2048
    sh = workload.make_fp8_shared(2, 0, H, I, block=block)
    x = synth.activations(13, M, H)
    y0 = torch.from_numpy(np.random.default_rng(M + block).standard_normal((M, H)).astype(np.float32))
    y = y0.cuda().clone()
    ws = torch.empty(qk.fp8_shared_expert_workspace_size(M, H, I), dtype=torch.uint8, device="cuda")
    qk.fp8_shared_expert_forward(x.cuda(), sh.wg, sh.sg, sh.wu, sh.su, sh.wd, sh.sd, y, ws, scale_block=block)
    assert qk.qk_last_device_status() == qk.QK_OK
    rows = np.arange(M) if M <= 256 else np.unique(np.r_[np.linspace(0, M - 1, 62).round().astype(int), 63, 64])
    hs = workload.make_fp8_shared(2, 0, H, I, device="cpu", block=block)
    so = oracle.fp8_swiglu_ffn(x[rows], hs.wg, hs.sg, hs.wu, hs.su, hs.wd, hs.sd, block=block)
    got = (y.cpu() - y0).numpy()[rows]
    assert_parity(got, so, what=f"shared expert block-scaled M={M} block={block} ({len(rows)} rows)")
