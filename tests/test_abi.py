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
