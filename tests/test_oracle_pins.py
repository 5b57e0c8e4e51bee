"""Pins for the fp64 CPU oracle: each check ties the oracle to something other than itself.

The pages ("YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次", section
"路线二：Multi-Head Gated Retention") define gated retention by its recurrence and by the
unrolled sum with products of gates; section "Prefill 与 Decode 为什么使用两种计算形态" says
the parallel, recurrent and chunkwise forms re-associate one formula.  The pages print no
worked numeric example for gRet, so the pins are closed forms, hand-worked tiny cases,
brute force and invariants, chosen so that a dropped term, a wrong sign or index, or a
transposed operand fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(rng, shape, std=1.0, mean=0.0):
    return rng.standard_normal(shape) * std + mean


def case(seed, T, H, dk, dv, g_mean=2.0, g_std=1.0, state=False, n_seqs=1):
    rng = np.random.default_rng(seed)
    q = rnd(rng, (T, H, dk), 1 / math.sqrt(dk))
    k = rnd(rng, (T, H, dk), 1 / math.sqrt(dk))
    v = rnd(rng, (T, H, dv), 1 / math.sqrt(dv))
    g = rnd(rng, (T, H), g_std, g_mean)
    s0 = rnd(rng, (n_seqs, H, dk, dv)) if state else None
    return q, k, v, g, s0


def close(a, b, tol=1e-12):
    scale = max(1e-300, float(np.max(np.abs(b))))
    return float(np.max(np.abs(a - b))) / scale <= tol


# ---------------------------------------------------------------------------------------------
# gate: log(gamma) = logsigmoid(g) / tau, i.e. gamma = sigmoid(g)^(1/tau)


def test_gate_closed_forms(oracle_mod):
    lg = oracle_mod.log_gamma
    assert lg(0.0, 1.0) == pytest.approx(-math.log(2.0), abs=1e-15)       # sigmoid(0) = 1/2
    assert lg(math.log(3.0), 1.0) == pytest.approx(math.log(0.75), abs=1e-15)  # sigmoid(ln3)=3/4
    assert lg(-1e4, 16.0) == -625.0                                        # exact far tail
    assert math.exp(lg(200.0, 16.0)) == 1.0                                # gamma == 1
    for gv in (-7.0, -1.5, 0.3, 2.0, 9.0):
        for tau in (1.0, 4.0, 16.0):
            # the power form sigmoid(g)^(1/tau), evaluated directly
            want = (1.0 / (1.0 + math.exp(-gv))) ** (1.0 / tau)
            assert math.exp(lg(gv, tau)) == pytest.approx(want, rel=1e-14)


# ---------------------------------------------------------------------------------------------
# hand-worked recurrences (exact rationals, derived by hand in the comments)


def test_handworked_scalar_recurrence(oracle_mod):
    # tau = 1, g = 0 -> gamma = 1/2; dk = dv = 1; S0 = 0
    # S1 = 3*5 = 15            o1 = 1*15 = 15
    # S2 = 15/2 + 4*6 = 31.5   o2 = 2*31.5 = 63
    # S3 = 31.5/2 + 1*2 = 17.75  o3 = -17.75
    q = np.array([1.0, 2.0, -1.0]).reshape(3, 1, 1)
    k = np.array([3.0, 4.0, 1.0]).reshape(3, 1, 1)
    v = np.array([5.0, 6.0, 2.0]).reshape(3, 1, 1)
    g = np.zeros((3, 1))
    o, s = oracle_mod.gret_recurrent(q, k, v, g, tau=1.0)
    assert np.allclose(o.ravel(), [15.0, 63.0, -17.75], rtol=0, atol=1e-13)
    assert s.ravel()[0] == pytest.approx(17.75, abs=1e-13)
    # k_scale = 1/2 with S0 = 0 halves every state and output
    o, s = oracle_mod.gret_recurrent(q, k, v, g, tau=1.0, k_scale=0.5)
    assert np.allclose(o.ravel(), [7.5, 31.5, -8.875], rtol=0, atol=1e-13)


def test_handworked_matrix_recurrence_with_entry_state(oracle_mod):
    # tau = 1, g = ln 3 -> gamma = 3/4; dk = dv = 2; row-vector convention o = q S.
    # S0 = [[1,0],[0,2]]
    # t1: q=[1,1] k=[1,0] v=[0,1]: S1 = 3/4 S0 + k^T v = [[0.75,1],[0,1.5]];  o1 = [0.75, 2.5]
    # t2: q=[2,-1] k=[0,1] v=[1,1]: S2 = 3/4 S1 + [[0,0],[1,1]] = [[0.5625,0.75],[1,2.125]]
    #     o2 = 2*[0.5625,0.75] - [1,2.125] = [0.125, -0.625]
    q = np.array([[1.0, 1.0], [2.0, -1.0]]).reshape(2, 1, 2)
    k = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(2, 1, 2)
    v = np.array([[0.0, 1.0], [1.0, 1.0]]).reshape(2, 1, 2)
    g = np.full((2, 1), math.log(3.0))
    s0 = np.array([[1.0, 0.0], [0.0, 2.0]]).reshape(1, 1, 2, 2)
    o, s = oracle_mod.gret_recurrent(q, k, v, g, tau=1.0, state_in=s0)
    assert np.allclose(o.reshape(2, 2), [[0.75, 2.5], [0.125, -0.625]], atol=1e-14)
    assert np.allclose(s.reshape(2, 2), [[0.5625, 0.75], [1.0, 2.125]], atol=1e-14)
    # the same numbers through the brute-force and chunkwise routes
    o2, s2 = oracle_mod.gret_parallel(q, k, v, g, tau=1.0, state_in=s0)
    o3, s3 = oracle_mod.gret_chunkwise(q, k, v, g, 1, tau=1.0, state_in=s0)
    for a, b in ((o2, o), (s2, s), (o3, o), (s3, s)):
        assert np.allclose(a, b, atol=1e-14)


def test_state_size_matches_page_count(oracle_mod):
    """The page's 3B hand count: 13 Self layers x 24 heads x 128x128 state, bf16 -> 9.75 MiB.

    The oracle is run on one token of one request with the page's head count and widths; the
    state it returns must hold exactly heads x d_k x d_v numbers, so that 13 such states in bf16
    come to the page's figure.  A state of another shape (a missing head axis, d_k x d_k, an
    extra per-token axis) fails the count."""
    with open(os.path.join(GOLDEN, "state_size_3b.json")) as f:
        gold = json.load(f)
    H, dk, dv = gold["heads"], gold["d_k"], gold["d_v"]
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, H, dk))
    k = rng.standard_normal((1, H, dk))
    v = rng.standard_normal((1, H, dv))
    g = rng.standard_normal((1, H))
    _, s = oracle_mod.gret_recurrent(q, k, v, g)
    assert s.shape == (1, H, dk, dv)
    mib = gold["self_layers"] * s[0].size * gold["bytes_per_elem"] / 2**20
    assert mib == pytest.approx(gold["mib_per_request"], abs=0.005)
    # with one token from a zero state the state is exactly the first outer product k^T v
    assert np.allclose(s[0], np.einsum("hi,hj->hij", k[0], v[0]), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# brute-force unrolled form with explicit gate products vs the recurrence


@pytest.mark.parametrize("T,dk,dv", [(1, 4, 4), (7, 4, 8), (33, 8, 4), (64, 16, 16)])
@pytest.mark.parametrize("regime", [(2.0, 1.0), (0.0, 2.0), (-3.0, 3.0)])
@pytest.mark.parametrize("state", [False, True])
def test_parallel_equals_recurrent(oracle_mod, T, dk, dv, regime, state):
    q, k, v, g, s0 = case(11 + T + dk, T, 2, dk, dv, regime[0], regime[1], state)
    o1, s1 = oracle_mod.gret_recurrent(q, k, v, g, tau=16.0, k_scale=0.7, state_in=s0)
    o2, s2 = oracle_mod.gret_parallel(q, k, v, g, tau=16.0, k_scale=0.7, state_in=s0)
    assert close(o1, o2) and close(s1, s2)


def test_parallel_equals_recurrent_varlen_with_empty_sequence(oracle_mod):
    lens = [5, 0, 17, 1]
    cu = np.cumsum([0] + lens)
    q, k, v, g, s0 = case(3, int(cu[-1]), 3, 8, 8, 0.0, 2.0, True, n_seqs=len(lens))
    o1, s1 = oracle_mod.gret_recurrent(q, k, v, g, cu_seqlens=cu, state_in=s0)
    o2, s2 = oracle_mod.gret_parallel(q, k, v, g, cu_seqlens=cu, state_in=s0)
    assert close(o1, o2) and close(s1, s2)
    # an empty sequence passes its entry state through unchanged
    assert np.array_equal(s1[1], s0[1])


# ---------------------------------------------------------------------------------------------
# special gates


def test_gamma_one_is_causal_linear_attention(oracle_mod):
    q, k, v, _, _ = case(5, 40, 2, 8, 8)
    g = np.full((40, 2), 200.0)                     # logsigmoid(200)/16 rounds gamma to 1
    o, s = oracle_mod.gret_recurrent(q, k, v, g)
    for h in range(2):
        A = np.tril(q[:, h] @ k[:, h].T)            # causal (Q K^T) with the diagonal kept
        assert close(o[:, h], A @ v[:, h])
        assert close(s[0, h], k[:, h].T @ v[:, h])


def test_gamma_zero_keeps_current_token(oracle_mod):
    q, k, v, _, s0 = case(6, 25, 2, 8, 4, state=True)
    g = np.full((25, 2), -1e4)                      # gamma = exp(-625): nothing survives
    o, s = oracle_mod.gret_recurrent(q, k, v, g, state_in=s0)
    for h in range(2):
        qk = np.sum(q[:, h] * k[:, h], axis=1)
        assert close(o[:, h], qk[:, None] * v[:, h])
        assert close(s[0, h], np.outer(k[-1, h], v[-1, h]))


# ---------------------------------------------------------------------------------------------
# chunkwise re-association, state carry, decode


@pytest.mark.parametrize("chunk", [1, 2, 3, 16, 32, 64, 128, 256, 512])
def test_chunkwise_equals_recurrent(oracle_mod, chunk):
    lens = [200, 64, 1, 129]
    cu = np.cumsum([0] + lens)
    q, k, v, g, s0 = case(chunk, int(cu[-1]), 2, 8, 16, 0.0, 2.0, True, n_seqs=len(lens))
    o1, s1 = oracle_mod.gret_recurrent(q, k, v, g, cu_seqlens=cu, state_in=s0, k_scale=1.3)
    o2, s2 = oracle_mod.gret_chunkwise(q, k, v, g, chunk, cu_seqlens=cu, state_in=s0,
                                       k_scale=1.3)
    assert close(o1, o2, 1e-11) and close(s1, s2, 1e-11)


def test_split_prefill_equals_one_prefill(oracle_mod):
    q, k, v, g, s0 = case(8, 300, 2, 16, 16, state=True)
    o, s = oracle_mod.gret_recurrent(q, k, v, g, state_in=s0)
    oa, sa = oracle_mod.gret_recurrent(q[:113], k[:113], v[:113], g[:113], state_in=s0)
    ob, sb = oracle_mod.gret_recurrent(q[113:], k[113:], v[113:], g[113:], state_in=sa)
    assert close(np.concatenate([oa, ob]), o) and close(sb, s)


def test_decode_after_prefill_equals_longer_prefill(oracle_mod):
    B, N, H, d = 3, 50, 2, 8
    q, k, v, g, _ = case(9, B * (N + 1), H, d, d)
    cu = np.arange(B + 1) * (N + 1)
    o_full, s_full = oracle_mod.gret_recurrent(q, k, v, g, cu_seqlens=cu)
    # prefill the first N tokens of each sequence, then one decode step per sequence
    keep = np.concatenate([np.arange(b * (N + 1), b * (N + 1) + N) for b in range(B)])
    last = np.array([b * (N + 1) + N for b in range(B)])
    _, s_pre = oracle_mod.gret_recurrent(q[keep], k[keep], v[keep], g[keep],
                                         cu_seqlens=np.arange(B + 1) * N)
    o_dec, s_dec = oracle_mod.gret_decode_step(q[last], k[last], v[last], g[last], s_pre)
    assert close(o_dec, o_full[last]) and close(s_dec, s_full)


def test_linearity(oracle_mod):
    q, k, v, g, _ = case(10, 60, 2, 8, 8)
    rng = np.random.default_rng(1)
    v2 = rnd(rng, v.shape)
    o1, _ = oracle_mod.gret_recurrent(q, k, v, g)
    o2, _ = oracle_mod.gret_recurrent(q, k, v2, g)
    o12, _ = oracle_mod.gret_recurrent(q, k, v + 2.0 * v2, g)
    assert close(o12, o1 + 2.0 * o2)
    o3, _ = oracle_mod.gret_recurrent(-1.5 * q, k, v, g)
    assert close(o3, -1.5 * o1)
    o4, _ = oracle_mod.gret_recurrent(q, k, v, g, k_scale=0.25)
    assert close(o4, 0.25 * o1)


def test_causality(oracle_mod):
    """Changing token t changes no output before t."""
    q, k, v, g, _ = case(12, 40, 1, 8, 8)
    o1, _ = oracle_mod.gret_recurrent(q, k, v, g)
    k2, v2, g2 = k.copy(), v.copy(), g.copy()
    k2[20:] += 1.0
    v2[20:] -= 1.0
    g2[20:] = -5.0
    o2, _ = oracle_mod.gret_recurrent(q, k2, v2, g2)
    assert np.array_equal(o1[:20], o2[:20])
    assert not np.allclose(o1[20:], o2[20:])


# ---------------------------------------------------------------------------------------------
# GroupNorm + swish gate


def test_groupnorm_gate_hand_example(oracle_mod):
    # one head, dv = 4, o = [1,2,3,4]: mean 2.5, biased var 1.25; eps = 0.75 -> 1/sqrt(2)
    # x = [1], w = [ln3]*4 -> z = ln3, swish(z) = ln3 * sigmoid(ln3) = 0.75 ln3
    o = np.array([[1.0, 2.0, 3.0, 4.0]])
    x = np.array([[1.0]])
    w = np.full((1, 4), math.log(3.0))
    y = oracle_mod.groupnorm_gate(o, x, w, H=1, eps=0.75)
    want = np.array([-1.5, -0.5, 0.5, 1.5]) / math.sqrt(2.0) * 0.75 * math.log(3.0)
    assert np.allclose(y.ravel(), want, atol=1e-14)


def test_groupnorm_moments_and_gate(oracle_mod):
    rng = np.random.default_rng(4)
    T, H, dv, D = 6, 3, 16, 10
    o = rnd(rng, (T, H * dv), 2.0, 0.5)
    x = rnd(rng, (T, D))
    w = rnd(rng, (D, H * dv), 0.3)
    eps = 1e-5
    # z by an explicit triple loop (independent of the oracle's loop order)
    z = np.zeros((T, H * dv))
    for t in range(T):
        for c in range(H * dv):
            acc = 0.0
            for e in range(D):
                acc += x[t, e] * w[e, c]
            z[t, c] = acc
    swish = z / (1.0 + np.exp(-z))
    # x*W = 0 on a column would make the ratio undefined; this draw has none
    assert np.min(np.abs(swish)) > 1e-8
    y = oracle_mod.groupnorm_gate(o, x, w, H=H, eps=eps)
    n = y / swish
    for t in range(T):
        for h in range(H):
            seg = n[t, h * dv:(h + 1) * dv]
            var = np.var(o[t, h * dv:(h + 1) * dv])
            assert abs(seg.mean()) < 1e-12
            assert seg.var() == pytest.approx(var / (var + eps), rel=1e-10)
    # affine parameters act per channel after normalisation
    gw, gb = rnd(rng, H * dv, 0.2, 1.0), rnd(rng, H * dv, 0.2)
    ya = oracle_mod.groupnorm_gate(o, x, w, H=H, gn_weight=gw, gn_bias=gb, eps=eps)
    assert np.allclose(ya, (n * gw + gb) * swish, atol=1e-12)
    # a row subset returns exactly those rows
    ys = oracle_mod.groupnorm_gate(o, x, w, H=H, eps=eps, rows=[4, 1])
    assert np.array_equal(ys, y[[4, 1]])


# ---- the layer's input projection and the layer composition


def test_projection_brute_force(oracle_mod):
    """[q | k | v | g] = x W against explicit loops on a tiny case."""
    rng = np.random.default_rng(11)
    T, D, H, d = 3, 5, 2, 3
    F = 3 * H * d + H
    x = rng.standard_normal((T, D))
    w = rng.standard_normal((D, F + 2))              # two padding columns, ignored
    q, k, v, g = oracle_mod.qkvg_projection(x, w, H, d)
    for t in range(T):
        for c in range(F):
            ref = sum(x[t, i] * w[i, c] for i in range(D))
            blk, rem = divmod(c, H * d)
            got = (q, k, v)[blk][t, rem // d, rem % d] if blk < 3 else g[t, c - 3 * H * d]
            assert abs(got - ref) < 1e-12


def test_projection_blocks_one_hot(oracle_mod):
    """W with one 1 per column: each output reads one input column, so the block layout of q, k,
    v (heads of d consecutive columns) and g shows directly."""
    T, D, H, d = 2, 64, 2, 4
    F = 3 * H * d + H
    x = np.arange(T * D, dtype=np.float64).reshape(T, D)
    w = np.zeros((D, F))
    for c in range(F):
        w[(7 * c + 3) % D, c] = 1.0
    q, k, v, g = oracle_mod.qkvg_projection(x, w, H, d)
    for t in range(T):
        for h in range(H):
            for j in range(d):
                for blk, arr in enumerate((q, k, v)):
                    c = blk * H * d + h * d + j
                    assert arr[t, h, j] == x[t, (7 * c + 3) % D]
            c = 3 * H * d + h
            assert g[t, h] == x[t, (7 * c + 3) % D]


def test_layer_with_closed_gates_is_per_token(oracle_mod):
    """gamma == 0 (every gate logit -1e4 through a constant input column): each token attends
    only to itself, o_t = k_scale (q_t . k_t) v_t per head with k_scale = d^-1/2, so the layer is
    GroupNorm(bf16(o_t)) * swish(x_t W_G) token by token, with q, k, v rounded to bf16 first."""
    rng = np.random.default_rng(12)
    T, D, H, d = 6, 64, 2, 4
    F = 3 * H * d + H
    x = rng.standard_normal((T, D)) * 0.5
    x[:, 0] = 1.0
    w = rng.standard_normal((D, F)) * 0.3
    w[:, 3 * H * d:] = 0.0
    w[0, 3 * H * d:] = -1e4
    w_g = rng.standard_normal((D, H * d)) * 0.3
    y, _ = oracle_mod.layer_forward(x, w, w_g, H, d)
    import torch
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()
    z = x @ w
    hd = H * d
    q = bf(z[:, :hd]).reshape(T, H, d)
    k = bf(z[:, hd:2 * hd]).reshape(T, H, d)
    v = bf(z[:, 2 * hd:3 * hd]).reshape(T, H, d)
    o = bf(np.einsum("thj,thj->th", q, k)[:, :, None] * d ** -0.5 * v)
    zg = x @ w_g
    for t in range(T):
        for h in range(H):
            row = o[t, h]
            n = (row - row.mean()) / np.sqrt(row.var() + 1e-5)
            zz = zg[t, h * d:(h + 1) * d]
            ref = n * zz / (1.0 + np.exp(-zz))
            assert np.allclose(y[t, h * d:(h + 1) * d], ref, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# Element-wise (per key channel) gate: the alternative that "路线二：Multi-Head Gated Retention"
# weighs against the head-wise gate.  State row i decays by alpha_t[i] = sigmoid(g_t[i])^(1/tau).

def ew_case(seed, T, H, dk, dv, g_mean=2.0, g_std=1.0, state=False, n_seqs=1):
    rng = np.random.default_rng(seed)
    q, k, v, _, s0 = case(seed, T, H, dk, dv, state=state, n_seqs=n_seqs)
    g = rnd(rng, (T, H, dk), g_std, g_mean)
    return q, k, v, g, s0


def test_ew_equal_channel_gates_is_headwise(oracle_mod):
    """One gate shared by every channel of a head reduces to the head-wise recurrence (a
    separate function of the oracle), across sequences with an entry state."""
    q, k, v, g1, s0 = case(41, 23, 2, 6, 5, g_std=2.0, state=True, n_seqs=3)
    g = np.repeat(g1[:, :, None], 6, axis=2)
    cu = [0, 7, 7, 23]
    o_ew, s_ew = oracle_mod.gret_recurrent_ew(q, k, v, g, k_scale=0.7, cu_seqlens=cu,
                                              state_in=s0)
    o_hw, s_hw = oracle_mod.gret_recurrent(q, k, v, g1, k_scale=0.7, cu_seqlens=cu,
                                           state_in=s0)
    assert close(o_ew, o_hw) and close(s_ew, s_hw)


def test_ew_brute_force_products(oracle_mod):
    """The unrolled per-channel form, with the survival products of each channel formed term by
    term and the gate from its closed form sigmoid(g)^(1/tau):
        O_n[j] = sum_i Q_n[i] ( sum_{m<=n} k_scale K_m[i] V_m[j] prod_{m<l<=n} alpha_l[i]
                                + S_0[i][j] prod_{l<=n} alpha_l[i] )."""
    T, H, dk, dv, tau, ks = 9, 2, 3, 4, 16.0, 0.8
    q, k, v, g, s0 = ew_case(42, T, H, dk, dv, g_mean=0.0, g_std=3.0, state=True)
    alpha = (1.0 / (1.0 + np.exp(-g))) ** (1.0 / tau)
    o_ref = np.zeros((T, H, dv))
    for h in range(H):
        for n in range(T):
            for i in range(dk):
                for j in range(dv):
                    acc = s0[0, h, i, j] * np.prod(alpha[:n + 1, h, i])
                    for m in range(n + 1):
                        acc += ks * k[m, h, i] * v[m, h, j] * np.prod(alpha[m + 1:n + 1, h, i])
                    o_ref[n, h, j] += q[n, h, i] * acc
    o, _ = oracle_mod.gret_recurrent_ew(q, k, v, g, tau=tau, k_scale=ks, state_in=s0)
    assert close(o, o_ref, 1e-12)


def test_ew_one_hot_query_reads_one_decayed_row(oracle_mod):
    """With q = e_c, o_t is row c of the state, which must follow a scalar-gate recurrence with
    channel c's gate and key (d_k != d_v, so a gate applied along the value axis fails)."""
    T, H, dk, dv = 17, 1, 5, 3
    _, k, v, g, s0 = ew_case(43, T, H, dk, dv, g_mean=0.0, g_std=2.0, state=True)
    for c in (0, 3):
        q = np.zeros((T, H, dk))
        q[:, :, c] = 1.0
        o, s = oracle_mod.gret_recurrent_ew(q, k, v, g, state_in=s0)
        o1, s1 = oracle_mod.gret_recurrent(np.ones((T, H, 1)), k[:, :, c:c + 1], v, g[:, :, c],
                                           state_in=s0[:, :, c:c + 1, :])
        assert close(o, o1) and close(s[:, :, c:c + 1, :], s1)


def test_ew_closed_gates_keep_current_token(oracle_mod):
    """alpha == 0 on every channel (g = -1e4): O_n = k_scale (Q_n . K_n) V_n and S_N = K_N^T V_N."""
    q, k, v, _, s0 = ew_case(44, 11, 2, 4, 6, state=True)
    g = np.full((11, 2, 4), -1e4)
    o, s = oracle_mod.gret_recurrent_ew(q, k, v, g, k_scale=0.5, state_in=s0)
    o_ref = 0.5 * np.einsum("thi,thi->th", q, k)[:, :, None] * v
    assert close(o, o_ref)
    assert close(s[0], 0.5 * np.einsum("hi,hj->hij", k[-1], v[-1]))


# ---------------------------------------------------------------------------------------------
# Sliding-window attention ("路线一：滑动窗口注意力"): position i sees positions i-C+1 .. i.

def softmax_rows(s):
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


@pytest.mark.parametrize("window", [1, 3, 7, 40])
def test_swa_explicit_mask(oracle_mod, window):
    """Against the matrix form softmax(scale Q K^T + B) V with the causal window mask B written
    out (0 for i - C < j <= i, -inf elsewhere), per sequence, two sequences packed."""
    rng = np.random.default_rng(50 + window)
    T, H, d, dv = 29, 2, 8, 5
    q, k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d)), \
        rng.standard_normal((T, H, dv))
    cu = [0, 12, T]
    o = oracle_mod.swa(q, k, v, window, scale=0.3, cu_seqlens=cu)
    ref = np.zeros_like(o)
    for a, e in zip(cu[:-1], cu[1:]):
        n = e - a
        i, j = np.arange(n)[:, None], np.arange(n)[None, :]
        B = np.where((j <= i) & (j > i - window), 0.0, -np.inf)
        for h in range(H):
            P = softmax_rows(0.3 * q[a:e, h] @ k[a:e, h].T + B)
            ref[a:e, h] = P @ v[a:e, h]
    assert close(o, ref)


def test_swa_window_one_copies_v(oracle_mod):
    rng = np.random.default_rng(60)
    q, k, v = rng.standard_normal((10, 3, 4)), rng.standard_normal((10, 3, 4)), \
        rng.standard_normal((10, 3, 6))
    assert close(oracle_mod.swa(q, k, v, 1), v)


def test_swa_wide_window_is_causal_attention(oracle_mod):
    """A window at least the sequence length gives plain causal softmax attention, computed
    here row by row with a running prefix (a different route from the mask matrix)."""
    rng = np.random.default_rng(61)
    T, H, d = 17, 2, 6
    q, k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d)), \
        rng.standard_normal((T, H, d))
    o = oracle_mod.swa(q, k, v, 1000)
    ref = np.zeros_like(o)
    for h in range(H):
        for i in range(T):
            w = np.exp(q[i, h] @ k[:i + 1, h].T / np.sqrt(d))
            ref[i, h] = (w / w.sum()) @ v[:i + 1, h]
    assert close(o, ref)


def test_swa_zero_queries_average_the_window(oracle_mod):
    """q = 0: every score is 0, so o_i is the plain mean of v over the window."""
    rng = np.random.default_rng(62)
    T, H, d, C = 23, 1, 4, 5
    k, v = rng.standard_normal((T, H, d)), rng.standard_normal((T, H, 3))
    o = oracle_mod.swa(np.zeros((T, H, d)), k, v, C)
    ref = np.stack([v[max(0, i - C + 1):i + 1].mean(axis=0) for i in range(T)])
    assert close(o, ref)
