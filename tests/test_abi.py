"""C-ABI checks that need no GPU: the library loads, exports every entry point declared in
include/gret.h, names its status codes, and rejects bad arguments on the host before any
launch (so these calls never touch a device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gret.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gret_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    import gated_retention_linear_b200 as G
    lib = ctypes.CDLL(G.LIB_PATH)
    names = declared_functions()
    assert {"gret_prefill_chunkwise", "gret_decode_step", "gret_groupnorm_gate"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    import gated_retention_linear_b200 as G
    for code, name in G.STATUS.items():
        assert G.gret_status_string(code).startswith(name)
    assert G.gret_status_string(99) == "GRET_ERR_UNKNOWN"


def _prefill(lib, **kw):
    a = dict(q=1024, k=1024, sb=0, st=128 * 24, sh=128, v=1024, vsb=0, vst=128 * 24, vsh=128,
             g=1024, tau=16.0, ks=1.0,
             dtype=1, B=1, N=64, H=24, dk=128, dv=128, cu=None, n=0, sin=None, sout=None,
             o=2048, osb=0, ost=128 * 24, osh=128, chunk=0, ws=None, wsb=0, stream=None)
    a.update(kw)
    return lib.gret_prefill_chunkwise(*a.values())


def test_prefill_rejects_bad_arguments_without_launching():
    import gated_retention_linear_b200 as G
    lib = G._lib
    assert _prefill(lib, dk=96) == 1          # unsupported head width
    assert _prefill(lib, H=0) == 1
    assert _prefill(lib, tau=0.0) == 1
    assert _prefill(lib, tau=float("nan")) == 1
    assert _prefill(lib, dtype=7) == 1
    assert _prefill(lib, st=-1) == 1
    assert _prefill(lib, q=None) == 1
    assert _prefill(lib, cu=4096, B=2) == 1   # varlen needs B == 1
    assert _prefill(lib, chunk=48) == 2       # no kernel for this chunk size
    assert _prefill(lib, B=0) == 0            # nothing to do


def test_tensor_core_prefill_checks_workspace_and_alignment():
    import gated_retention_linear_b200 as G
    lib = G._lib
    need = G.gret_prefill_workspace_size(G.GRET_BF16, 32768, 1, 24, 128, 128, 128)
    assert need >= 256
    assert _prefill(lib, chunk=128, ws=None) == 4
    assert _prefill(lib, chunk=128, ws=4096, wsb=need - 1) == 4
    assert _prefill(lib, chunk=128, ws=4096 + 8, wsb=need) == 3      # workspace not 256-aligned
    assert _prefill(lib, chunk=128, ws=4096, wsb=need, q=1032) == 3  # q not 16-byte aligned
    assert _prefill(lib, chunk=128, ws=4096, wsb=need, st=100) == 3  # stride * 2 % 16 != 0


def test_decode_and_epilogue_reject_bad_arguments():
    import gated_retention_linear_b200 as G
    lib = G._lib
    args = [1024, 1024, 1024, 1024, 16.0, 1.0, 1, 64, 24, 128, 128, 4096, 8192, None]
    bad = list(args); bad[9] = 32
    assert lib.gret_decode_step(*bad) == 1
    bad = list(args); bad[11] = 4100                 # state not 16-byte aligned
    assert lib.gret_decode_step(*bad) == 3
    bad = list(args); bad[7] = 0
    assert lib.gret_decode_step(*bad) == 0           # empty batch: nothing launched
    ep = [1024, 2048, 4096, None, None, 1e-5, 100, 24, 128, 3072, 8192, None]
    bad = list(ep); bad[8] = 64
    assert lib.gret_groupnorm_gate(*bad) == 2
    bad = list(ep); bad[9] = 3000
    assert lib.gret_groupnorm_gate(*bad) == 2
    bad = list(ep); bad[6] = 0
    assert lib.gret_groupnorm_gate(*bad) == 0
    bad = list(ep); bad[5] = -1.0
    assert lib.gret_groupnorm_gate(*bad) == 1


def test_projection_rejects_bad_arguments_without_launching():
    import gated_retention_linear_b200 as G
    lib = G._lib

    def call(**kw):
        a = dict(x=1024, w=2048, ldw=3 * 2 * 128 + 2 + 6, T=16, H=2, d=128, D=128, q=4096,
                 k=8192, v=12288, g=16384, stream=None)
        a.update(kw)
        return lib.gret_qkvg_projection(*a.values())
    assert call(ldw=3 * 2 * 128 + 1) == 1     # fewer columns than W_Q, W_K, W_V, W_gamma need
    assert call(H=0) == 1
    assert call(T=-1) == 1
    assert call(d=64, ldw=400) == 2           # only d = 128 has a kernel
    assert call(H=129, ldw=3 * 129 * 128 + 129 + 7) == 2
    assert call(D=96) == 2                    # D must be a multiple of 64
    assert call(T=0) == 0                     # nothing to do
    assert call(x=None) == 1
    assert call(x=1026) == 3                  # not 16-byte aligned
    assert call(ldw=3 * 2 * 128 + 2 + 1) == 3 # rows would not start 16-byte aligned
    assert call(g=16386) == 3


def test_elementwise_prefill_rejects_bad_arguments_without_launching():
    import gated_retention_linear_b200 as G
    lib = G._lib
    # a 256-byte status head, then per (batch, head, range of chunks) one fp32 state slot and
    # one decay row; one 128-token chunk per range while the ranges fill one wave of 148 SMs
    slot = (128 * 128 + 128) * 4
    assert G.gret_prefill_elementwise_workspace_size(1, 64, 1, 128) == 256 + slot
    assert G.gret_prefill_elementwise_workspace_size(1, 129, 2, 128) == 256 + 2 * 2 * slot
    assert G.gret_prefill_elementwise_workspace_size(1, 1000, 4, 128) == 256 + 4 * 8 * slot
    # 256 chunks x 24 heads: ranges of 43 chunks, 6 per head (144 CTAs, one wave)
    assert G.gret_prefill_elementwise_workspace_size(1, 32768, 24, 128) == 256 + 24 * 6 * slot
    assert G.gret_prefill_elementwise_workspace_size(1, 64, 1, 64) == 0
    assert G.gret_prefill_elementwise_workspace_size(65535, 1 << 40, 65535, 128) == 0

    def call(**kw):
        a = dict(q=1024, k=2048, v=4096, g=8192, tau=16.0, ks=1.0, B=1, N=64, H=1, d=128,
                 sin=None, sout=None, o=16384, ws=1 << 20, wsb=1 << 20, stream=None)
        a.update(kw)
        return lib.gret_prefill_elementwise(*a.values())
    assert call(d=64) == 2
    assert call(H=0) == 1
    assert call(tau=0.0) == 1
    assert call(ks=float("inf")) == 1
    assert call(B=0) == 0
    assert call(N=0) == 0                     # no tokens and no state to write
    assert call(q=None) == 1
    assert call(q=1030) == 3
    assert call(sin=1028) == 3
    assert call(wsb=1000) == 4                # workspace smaller than the size query says
    assert call(ws=None) == 4
    assert call(B=65535, H=65535) == 2       # the scan's grid would not fit
    assert call(B=4, H=65535, N=64 << 30) == 2    # token coordinates past 32 bits


def test_swa_rejects_bad_arguments_without_launching():
    import gated_retention_linear_b200 as G
    lib = G._lib

    def call(**kw):
        a = dict(q=1024, k=2048, v=4096, scale=0.088, W=1024, B=1, N=64, H=2, d=128, o=8192,
                 stream=None)
        a.update(kw)
        return lib.gret_swa_prefill(*a.values())
    assert call(W=0) == 1
    assert call(scale=float("nan")) == 1
    assert call(H=0) == 1
    assert call(d=64) == 2
    assert call(B=0) == 0
    assert call(N=0) == 0
    assert call(o=None) == 1
    assert call(v=4100) == 3


def test_layer_forward_rejects_bad_arguments_without_launching():
    import gated_retention_linear_b200 as G
    lib = G._lib
    need = G.gret_layer_workspace_size(300, 1, 2, 128)
    # the prefill's workspace, then q, k, v, o (bf16) and g (fp32), each 256-byte aligned
    up = lambda x: (x + 255) // 256 * 256
    pre = G.gret_prefill_workspace_size(torch_bf16_code(G), 300, 1, 2, 128, 128)
    assert need == up(pre) + 4 * up(300 * 2 * 128 * 2) + up(300 * 2 * 4)
    assert G.gret_layer_workspace_size(300, 1, 2, 64) == 0
    assert G.gret_layer_workspace_size(300, 0, 2, 128) == 0

    def call(**kw):
        a = dict(x=1024, w=2048, ldw=776, wg=4096, gnw=None, gnb=None, eps=1e-5, tau=16.0,
                 ks=1.0, T=300, H=2, d=128, D=128, cu=None, n=1, sin=None, sout=None, y=8192,
                 ws=1 << 20, wsb=need, stream=None)
        a.update(kw)
        return lib.gret_layer_forward(*a.values())
    assert call(d=64) == 2                     # no kernel for d = 64
    assert call(n=2) == 1                      # two sequences need cu_seqlens
    assert call(H=0) == 1
    assert call(wsb=need - 1) == 4             # workspace smaller than the size query says
    assert call(ws=None) == 4
    assert call(ws=(1 << 20) + 8) == 3         # workspace not 16-byte aligned


def torch_bf16_code(G):
    import torch
    return G._dtype_code(torch.empty(0, dtype=torch.bfloat16))


def test_layer_forward_refuses_before_any_launch():
    """Arguments that only the later steps (the prefill, the GroupNorm gate) would refuse are
    refused up front: none of these calls launches anything (no GPU here)."""
    import gated_retention_linear_b200 as G
    lib = G._lib
    need = G.gret_layer_workspace_size(300, 1, 2, 128)

    def call(**kw):
        a = dict(x=1024, w=2048, ldw=776, wg=4096, gnw=None, gnb=None, eps=1e-5, tau=16.0,
                 ks=1.0, T=300, H=2, d=128, D=128, cu=None, n=1, sin=None, sout=None, y=8192,
                 ws=1 << 20, wsb=need, stream=None)
        a.update(kw)
        return lib.gret_layer_forward(*a.values())
    assert call(eps=-1.0) == 1                 # the gate's eps
    assert call(tau=0.0) == 1                  # the prefill's tau
    assert call(ldw=700) == 1                  # narrower than the projection's columns
    assert call(D=96) == 2                     # the GEMMs' K blocks
    assert call(H=3, ldw=3 * 3 * 128 + 3 + 5, wsb=G.gret_layer_workspace_size(300, 1, 3, 128)) == 2
    assert call(ldw=777) == 3                  # rows of W not 16-byte aligned
    assert call(y=8200) == 3
