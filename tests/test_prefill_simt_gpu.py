"""GPU parity of the CUDA-core chunkwise prefill (fp32 inputs, and bf16 at chunk sizes the
tensor-core kernel does not take) against the fp64 oracle, through the C ABI."""
import pytest
import torch

from gpu_cases import run_dense, run_varlen

pytestmark = pytest.mark.gpu


def test_tiny_config_fp32_head_major():
    # batch 1, 2 heads, 512 tokens, d = 64, fp32, chunk 64, head-major [B,H,N,d], S0 = 0
    eo, es = run_dense(1, 512, 2, 64, 64, torch.float32, chunk=64, seed=1, head_major=True)
    assert eo <= 1e-4 and es <= 1e-4


@pytest.mark.parametrize("N", [1, 15, 64, 65, 300])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_fp32_ragged_lengths_and_chunks(N, chunk):
    run_dense(2, N, 3, 64, 64, torch.float32, chunk=chunk, seed=N, state=True, g_mean=0.0,
              g_std=2.0)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
def test_fp32_head_widths(dk, dv):
    run_dense(1, 200, 2, dk, dv, torch.float32, chunk=64, seed=dk + dv, state=True)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_bf16_simt_chunks(chunk):
    run_dense(1, 333, 3, 128, 128, torch.bfloat16, chunk=chunk, seed=7, state=True)


def test_bf16_d64():
    run_dense(2, 257, 2, 64, 64, torch.bfloat16, chunk=0, seed=8)


@pytest.mark.parametrize("g_fill", [200.0, -1e4])
def test_degenerate_gates(g_fill):
    # gamma == 1 (causal linear attention) and gamma == 0 (current token only)
    run_dense(1, 150, 2, 64, 64, torch.float32, chunk=32, seed=9, state=True, g_fill=g_fill)


def test_varlen_with_empty_and_ragged_sequences():
    run_varlen([0, 1, 63, 64, 65, 200], 2, 64, 64, torch.float32, chunk=64, seed=10,
               state=True)


def test_varlen_state_aliasing():
    run_varlen([100, 0, 37], 2, 64, 64, torch.float32, chunk=32, seed=11, state=True,
               alias_state=True)


def test_k_scale_and_tau():
    run_dense(1, 100, 2, 64, 64, torch.float32, chunk=64, seed=12, tau=4.0, k_scale=0.125)
