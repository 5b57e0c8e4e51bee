"""Guard bands around every output of the ABI: each output tensor is a view into the middle of a
larger buffer whose bytes are first set to a sentinel; after the call the bytes before and after
the view must still hold it (no write out of bounds), and no element of a fully written output
may still hold it (no element left unwritten).  Sizes are ragged on purpose (partial chunks,
partial tiles, partial key windows), where an out-of-bounds write would happen."""
import pytest
import torch

import synth_inputs as SI

pytestmark = pytest.mark.gpu

SENTINEL = 0x7F          # bytes 7f 7f ...: 3.39e38 as bf16 and as fp32
GUARD = 4096             # bytes before and after each output


def lib():
    import gated_retention_linear_b200 as G
    return G


class Guarded:
    def __init__(self, shape, dtype, init=None):
        n = 1
        for s in shape:
            n *= s
        es = torch.empty(0, dtype=dtype).element_size()
        self.g, self.n = GUARD // es, n
        self.buf = torch.empty(2 * self.g + n, dtype=dtype, device="cuda")
        self.buf.view(torch.uint8).fill_(SENTINEL)
        self.t = self.buf[self.g:self.g + n].view(shape)
        if init is not None:
            self.t.copy_(init)

    def check(self, name, all_written=True):
        torch.cuda.synchronize()
        raw = self.buf.view(torch.uint8)
        es = self.buf.element_size()
        head, tail = raw[:self.g * es], raw[(self.g + self.n) * es:]
        assert bool((head == SENTINEL).all()), "%s: written before the output" % name
        assert bool((tail == SENTINEL).all()), "%s: written past the output" % name
        if all_written:
            assert torch.isfinite(self.t).all() and self.t.float().abs().max() < 1e30, \
                "%s: an element was left unwritten" % name


def test_guards_prefill_dense_and_noalloc():
    G = lib()
    B, N, H = 2, 300, 3
    inp = SI.gret_inputs(B, N, H, 128, seed=41, with_state=True, device="cuda")
    for fn in (G.gret_prefill_chunkwise, G.gret_prefill_chunkwise_noalloc):
        o = Guarded((B, N, H, 128), torch.bfloat16)
        s = Guarded((B, H, 128, 128), torch.float32)
        fn(inp["q"], inp["k"], inp["v"], inp["g"], state_in=inp["s"], o=o.t, state_out=s.t)
        o.check("o")
        s.check("state_out")


def test_guards_prefill_varlen():
    G = lib()
    lens = [1, 130, 257, 7]
    T, H = sum(lens), 2
    inp = SI.gret_inputs(1, T, H, 128, seed=42, device="cuda")
    cu = torch.tensor(SI.cu_seqlens_of(lens), dtype=torch.int32, device="cuda")
    o = Guarded((T, H, 128), torch.bfloat16)
    s = Guarded((len(lens), H, 128, 128), torch.float32)
    G.gret_prefill_chunkwise(inp["q"][0], inp["k"][0], inp["v"][0], inp["g"][0], cu_seqlens=cu,
                             o=o.t, state_out=s.t)
    o.check("o")
    s.check("state_out")


def test_guards_decode():
    G = lib()
    B, H = 5, 3
    inp = SI.gret_inputs(B, 1, H, 128, seed=43, with_state=True, device="cuda")
    st = Guarded((B, H, 128, 128), torch.float32, init=inp["s"])
    o = Guarded((B, H, 128), torch.bfloat16)
    G.gret_decode_step(inp["q"][:, 0].contiguous(), inp["k"][:, 0].contiguous(),
                       inp["v"][:, 0].contiguous(), inp["g"][:, 0].contiguous(), st.t, o=o.t)
    st.check("state")
    o.check("o")


def test_guards_groupnorm_gate_and_projection():
    G = lib()
    T, H, D = 300, 2, 128       # one partial pair tile of 256 rows, then 44 rows
    e = SI.epilogue_inputs(T, D, H * 128, seed=44, device="cuda")
    o_in = SI.gret_inputs(1, T, H, 128, seed=45, device="cuda")["q"].reshape(T, H * 128)
    y = Guarded((T, H * 128), torch.bfloat16)
    G.gret_groupnorm_gate(o_in, e["x"], e["w_g"], H, y=y.t)
    y.check("y")
    lay = SI.layer_inputs(T, D, H, seed=46, device="cuda", pad=6)   # rows of 776: 16-byte aligned
    outs = [Guarded((T, H, 128), torch.bfloat16) for _ in range(3)] + \
        [Guarded((T, H), torch.float32)]
    G.gret_qkvg_projection(lay["x"], lay["w_qkvg"], H, out=tuple(t.t for t in outs))
    for name, t in zip("qkvg", outs):
        t.check(name)


def test_guards_elementwise_prefill():
    G = lib()
    B, N, H = 1, 300, 2
    inp = SI.gret_inputs(B, N, H, 128, seed=47, with_state=True, device="cuda")
    g = SI.channel_gates(B, N, H, 128, seed=47, device="cuda")
    o = Guarded((B, N, H, 128), torch.bfloat16)
    s = Guarded((B, H, 128, 128), torch.float32)
    G.gret_prefill_elementwise(inp["q"], inp["k"], inp["v"], g, state_in=inp["s"], o=o.t,
                               state_out=s.t)
    o.check("o")
    s.check("state_out")


def test_guards_sliding_window():
    G = lib()
    B, N, H = 1, 300, 2
    inp = SI.gret_inputs(B, N, H, 128, seed=48, device="cuda")
    o = Guarded((B, N, H, 128), torch.bfloat16)
    G.gret_swa_prefill(inp["q"], inp["k"], inp["v"], window=100, o=o.t)
    o.check("o")
    Bd, W = 3, 64
    dec = SI.gret_inputs(Bd, 1, H, 128, seed=49, device="cuda")
    cache = SI.gret_inputs(Bd, W, H, 128, seed=50, device="cuda")
    kc = Guarded((Bd, H, W, 128), torch.bfloat16, init=cache["k"].transpose(1, 2))
    vc = Guarded((Bd, H, W, 128), torch.bfloat16, init=cache["v"].transpose(1, 2))
    pos = torch.tensor([3, 64, 200], dtype=torch.int32, device="cuda")
    od = Guarded((Bd, H, 128), torch.bfloat16)
    G.gret_swa_decode_step(dec["q"][:, 0].contiguous(), dec["k"][:, 0].contiguous(),
                           dec["v"][:, 0].contiguous(), pos, kc.t, vc.t, o=od.t)
    kc.check("k_cache")
    vc.check("v_cache")
    od.check("o")


def test_guards_layer_forward():
    G = lib()
    T, H, D = 300, 2, 128
    lay = SI.layer_inputs(T, D, H, seed=51, device="cuda", pad=6)
    cu = torch.tensor([0, 100, 300], dtype=torch.int32, device="cuda")
    y = Guarded((T, H * 128), torch.bfloat16)
    s = Guarded((2, H, 128, 128), torch.float32)
    G.gret_layer_forward(lay["x"], lay["w_qkvg"], lay["w_g"], H, cu_seqlens=cu, y=y.t,
                         state_out=s.t)
    y.check("y")
    s.check("state_out")
