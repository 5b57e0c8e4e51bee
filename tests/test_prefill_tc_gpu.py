"""GPU parity of the tensor-core chunkwise prefill (bf16, d_k = d_v = 128) against the fp64
oracle, through the C ABI: ragged lengths, several spans per chain, batches, layouts, varlen
with empty sequences, degenerate gates, entry states, and sampled heads at full size."""
import numpy as np
import pytest
import torch

import synth_inputs as SI
from gpu_cases import TC_TIGHT, lib, run_dense, run_varlen
from oracle import oracle
from parity import assert_parity

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.mark.parametrize("N", [1, 100, 127, 128, 129, 300, 1000])
def test_ragged_lengths(N):
    run_dense(1, N, 3, 128, 128, BF, seed=N, state=True)


@pytest.mark.parametrize("N", [512 * 3 + 17, 4096])
def test_several_spans_per_chain(N):
    # more chunks than one span holds: the look-back between spans is exercised
    run_dense(1, N, 4, 128, 128, BF, seed=N + 1, state=True)


def test_single_long_chain():
    # one head of 40000 tokens (313 chunks): the span-size model cuts a lone chain into many
    # short spans, so the look-back runs as a long serial chain of flags
    run_dense(1, 40000, 1, 128, 128, BF, seed=41, state=True)


def test_batch_of_sequences():
    run_dense(3, 700, 2, 128, 128, BF, seed=31, state=True)


def test_head_major_layout():
    run_dense(2, 333, 2, 128, 128, BF, seed=32, head_major=True)


@pytest.mark.parametrize("g_fill", [200.0, -1e4])
def test_degenerate_gates(g_fill):
    run_dense(1, 400, 2, 128, 128, BF, seed=33, state=True, g_fill=g_fill)


def test_harsh_gates_and_scales():
    run_dense(1, 900, 2, 128, 128, BF, seed=34, g_mean=0.0, g_std=2.0, tau=4.0, k_scale=0.5,
              state=True)


def test_factored_and_unfactored_chunks_in_one_chain():
    """The kernel factors a chunk's decay mask when the chunk's decay stays within 2^-64 and
    keeps the per-element form otherwise.  Here chunk c has gates -12 when c % 3 == 1 (decay
    about 2^-138 over the chunk: unfactored), -5 when c % 3 == 2 (about 2^-58: factored with
    factors near the limit) and N(2, 1) otherwise, so both forms alternate along each chain and
    across span boundaries."""
    def edit(g):   # [B, N, H]
        n = g.shape[1]
        for c in range((n + 127) // 128):
            if c % 3 == 1:
                g[:, c * 128:(c + 1) * 128] = -12.0
            elif c % 3 == 2:
                g[:, c * 128:(c + 1) * 128] = -5.0
    run_dense(1, 3000, 2, 128, 128, BF, seed=41, state=True, g_edit=edit)


def test_varlen_ragged_with_empty_sequences():
    run_varlen([0, 1, 127, 128, 129, 700, 0, 2000], 3, 128, 128, BF, seed=35, state=True)


def test_varlen_more_than_1024_sequences():
    """1100 packed sequences of 0 to 64 tokens: the span plan's prefix runs over two blocks of
    1024 sequences, and the span size is the one chosen for many short, unequal sequences."""
    rng = np.random.default_rng(37)
    lens = [int(x) for x in rng.integers(0, 65, size=1100)]
    run_varlen(lens, 1, 128, 128, BF, seed=37, state=True)


def test_varlen_state_aliasing():
    run_varlen([1500, 0, 37, 600], 2, 128, 128, BF, seed=36, state=True, alias_state=True)


def test_strided_fused_qkv_and_separate_output():
    """q, k, v as views into one [T, 3, H, d] buffer; o with its own padded row stride."""
    G = lib()
    T, H, d = 777, 2, 128
    inp = SI.gret_inputs(1, T, H, d, dtype=BF, seed=37)
    buf = torch.empty((T, 3, H, d), dtype=BF, device="cuda")
    buf[:, 0] = inp["q"][0].cuda()
    buf[:, 1] = inp["k"][0].cuda()
    buf[:, 2] = inp["v"][0].cuda()
    q, k, v = buf[:, 0], buf[:, 1], buf[:, 2]
    o_store = torch.zeros((T, H + 1, d), dtype=BF, device="cuda")
    o = o_store[:, :H]
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    G.gret_prefill_chunkwise(q, k, v, inp["g"][0].cuda(), cu_seqlens=cu, o=o, state_out=True)
    torch.cuda.synchronize()
    o_ref, _ = oracle.gret_recurrent(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0])
    assert_parity("o", o, o_ref, 1e-2, stored_bf16=True, tight=TC_TIGHT)
    assert torch.count_nonzero(o_store[:, H]) == 0          # the padding column is untouched


def test_workspace_status_ok():
    G = lib()
    inp = SI.gret_inputs(1, 1024, 2, 128, dtype=BF, seed=38, device="cuda")
    need = G.gret_prefill_workspace_size(BF, 1024, 1, 2, 128, 128, 0)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    G.gret_prefill_chunkwise(inp["q"], inp["k"], inp["v"], inp["g"], workspace=ws)
    assert G.gret_workspace_status(ws) == 0


def test_repeated_calls_reuse_workspace():
    """Two calls in a row on one workspace (flags and tickets are reset per call)."""
    G = lib()
    inp = SI.gret_inputs(1, 2000, 3, 128, dtype=BF, seed=39, device="cuda")
    need = G.gret_prefill_workspace_size(BF, 2000, 1, 3, 128, 128, 0)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o1, s1 = G.gret_prefill_chunkwise(inp["q"], inp["k"], inp["v"], inp["g"], workspace=ws,
                                      state_out=True)
    o2, s2 = G.gret_prefill_chunkwise(inp["q"], inp["k"], inp["v"], inp["g"], workspace=ws,
                                      state_out=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)      # deterministic
    assert G.gret_workspace_status(ws) == 0


@pytest.mark.parametrize("N", [1553, 4096])
def test_repeated_multi_span_calls_into_poisoned_output(N):
    """Chains of several spans, called again and again into an output pre-filled with NaN: a
    row that a call fails to write, or an entry state read while another warp overwrites it,
    shows up in one of the repetitions even when it is rare."""
    G = lib()
    H = 3
    inp = SI.gret_inputs(1, N, H, 128, dtype=BF, seed=N + 7, with_state=True)
    o_ref, s_ref = oracle.gret_recurrent(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0],
                                         state_in=inp["s"])
    d = {k: v.cuda() for k, v in inp.items()}
    for _ in range(8):
        o = torch.full((1, N, H, 128), float("nan"), dtype=BF, device="cuda")
        _, s = G.gret_prefill_chunkwise(d["q"], d["k"], d["v"], d["g"], state_in=d["s"],
                                        state_out=True, o=o)
        torch.cuda.synchronize()
        assert_parity("o", o[0], o_ref, 1e-2, stored_bf16=True, tight=TC_TIGHT)
        assert_parity("state", s, s_ref, 1e-2, stored_bf16=False, tight=TC_TIGHT)


def _sampled_heads(B, N, H, seed, heads, g_mean=2.0, g_std=1.0):
    """Full-size run on the GPU; oracle on a subset of heads (heads are independent)."""
    G = lib()
    inp = SI.gret_inputs(B, N, H, 128, dtype=BF, g_mean=g_mean, g_std=g_std, seed=seed,
                         device="cuda")
    o, s = G.gret_prefill_chunkwise(inp["q"], inp["k"], inp["v"], inp["g"], state_out=True)
    torch.cuda.synchronize()
    T = B * N
    hs = list(heads)
    sel = lambda x: x.reshape(T, H, -1)[:, hs].cpu()
    o_ref, s_ref = oracle.gret_recurrent(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]),
                                         inp["g"].reshape(T, H)[:, hs].cpu(),
                                         cu_seqlens=np.arange(B + 1) * N)
    assert_parity("o", sel(o), o_ref, 1e-2, stored_bf16=True, tight=TC_TIGHT)
    assert_parity("state", s[:, hs], s_ref, 1e-2, stored_bf16=False, tight=TC_TIGHT)


def test_prefill_32k_3b_shape_sampled_heads():
    # batch 1, 24 heads, 32768 tokens, d = 128, bf16, g ~ N(2, 1): heads 0, 11, 23 checked
    _sampled_heads(1, 32768, 24, 2, [0, 11, 23])


@pytest.mark.slow
def test_prefill_512k_sampled_head():
    # batch 1, 24 heads, 524288 tokens: 4096 chunks per chain; head 5 checked in full
    _sampled_heads(1, 524288, 24, 3, [5])


def test_varlen_8_sequences_harsh_gates_sampled_heads():
    G = lib()
    lens = SI.varlen_lengths(8, 1024, 65536, seed=5)
    cu = SI.cu_seqlens_of(lens)
    T, H = cu[-1], 24
    inp = SI.gret_inputs(1, T, H, 128, dtype=BF, g_mean=0.0, g_std=2.0, seed=5, device="cuda")
    q, k, v, g = (inp[x][0] for x in ("q", "k", "v", "g"))
    o, s = G.gret_prefill_chunkwise(q, k, v, g, state_out=True,
                                    cu_seqlens=torch.tensor(cu, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    hs = [3, 17]
    o_ref, s_ref = oracle.gret_recurrent(q[:, hs].cpu(), k[:, hs].cpu(), v[:, hs].cpu(),
                                         g[:, hs].cpu(), cu_seqlens=cu)
    assert_parity("o", o[:, hs], o_ref, 1e-2, stored_bf16=True, tight=TC_TIGHT)
    assert_parity("state", s[:, hs], s_ref, 1e-2, stored_bf16=False, tight=TC_TIGHT)
