"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point the header declares, validates arguments before touching the GPU,
and reports consistent workspace sizes."""
import ctypes
import os
import re

import pytest

from padding_free_moe_b200 import _lib as L
from padding_free_moe_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return L.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "pfmoe.h")).read()
    return re.findall(r"PFMOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(header_functions())
    for fn in ("moe_route", "pft_build", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_backward",
               "rbd_plan"):
        assert fn in names


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in L.SIGNATURES, f"binding lacks {n}"
    assert lib.moe_abi_version() == 2


FAKE = 1 << 20     # an aligned, never-dereferenced pointer value (validation fails before any use)


def test_route_argument_errors(lib):
    def call(**kw):
        a = dict(x=FAKE, wg=FAKE, bias=None, T=4, d=64, E=8, k=2, dtype=L.PFMOE_BF16, logits=FAKE, ids=FAKE,
                 w=FAKE)
        a.update(kw)
        return lib.moe_route(a["x"], a["wg"], a["bias"], a["T"], a["d"], a["E"], a["k"], a["dtype"], a["logits"],
                             a["ids"], a["w"], None, 0, None, None)
    assert call(k=9) == L.PFMOE_ERR_ARG                     # k > E
    assert b"k <= E" in lib.moe_last_error()
    assert call(k=0) == L.PFMOE_ERR_ARG
    assert call(dtype=7) == L.PFMOE_ERR_ARG
    assert call(d=60) == L.PFMOE_ERR_UNSUPPORTED            # BF16 rows must be 16-byte multiples
    assert call(x=None) == L.PFMOE_ERR_ARG
    assert call(x=FAKE + 4) == L.PFMOE_ERR_ARG              # misaligned
    assert call(E=2048, k=2) == L.PFMOE_ERR_UNSUPPORTED
    assert call(k=33, E=64) == L.PFMOE_ERR_UNSUPPORTED
    assert call(T=-1) == L.PFMOE_ERR_ARG


def test_other_argument_errors(lib):
    assert lib.pft_build(FAKE, FAKE, 4, 8, 9, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None,
                         None) == L.PFMOE_ERR_ARG
    ws = lib.pft_build_workspace_size(4, 8, 2)
    assert lib.pft_build(FAKE, FAKE, 4, 8, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 1, None,
                         None) == L.PFMOE_ERR_ARG
    assert b"workspace" in lib.moe_last_error()
    assert lib.moe_dispatch(FAKE, FAKE, 4, 40, 64, L.PFMOE_BF16, FAKE, None, None) == L.PFMOE_ERR_ARG
    assert lib.moe_combine(FAKE, None, FAKE, 4, 2, 64, L.PFMOE_BF16, FAKE, None, None) == L.PFMOE_ERR_ARG
    assert lib.moe_expert_ffn(FAKE, FAKE, FAKE, 8, 4, 64, 60, L.PFMOE_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              FAKE, None, None) == L.PFMOE_ERR_UNSUPPORTED
    # the gathered expert FFN: BF16 only, 16-byte rows, every pointer given
    def gathered(**kw):
        a = dict(x=FAKE, ids=FAKE, N=8, E=4, d=64, h=64, dtype=L.PFMOE_BF16)
        a.update(kw)
        return lib.moe_expert_ffn_gathered(a["x"], a["ids"], FAKE, FAKE, a["N"], a["E"], a["d"], a["h"], a["dtype"],
                                           FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None)
    assert gathered(dtype=L.PFMOE_F32) == L.PFMOE_ERR_UNSUPPORTED
    assert b"BF16" in lib.moe_last_error()
    assert gathered(h=60) == L.PFMOE_ERR_UNSUPPORTED
    assert gathered(ids=None) == L.PFMOE_ERR_ARG
    assert gathered(x=FAKE + 4) == L.PFMOE_ERR_ARG
    assert gathered(N=-1) == L.PFMOE_ERR_ARG
    # RBD map must tile the experts
    assert lib.rbd_plan(FAKE, 4, 2, 12, 4, 2, *([FAKE] * 10), 1 << 20, None, None) == L.PFMOE_ERR_ARG
    assert lib.rbd_plan_workspace_size(4, 2, 12, 4, 2) == 0


def test_wait_selftest_argument_errors(lib):
    assert lib.moe_selftest_wait_timeout(None, 50_000_000, None) == L.PFMOE_ERR_ARG
    assert lib.moe_selftest_wait_timeout(FAKE, 10, None) == L.PFMOE_ERR_ARG          # below 1 ms
    assert lib.moe_selftest_wait_timeout(FAKE, 10 ** 10, None) == L.PFMOE_ERR_ARG    # above 5 s
    assert b"limit_ns" in lib.moe_last_error()


def test_empty_inputs_are_noops(lib):
    # T = 0: nothing to launch for these steps, so they succeed without a GPU.
    assert lib.moe_dispatch(None, None, 0, 2, 64, L.PFMOE_BF16, None, None, None) == L.PFMOE_OK
    assert lib.moe_combine(None, None, None, 0, 2, 64, L.PFMOE_BF16, None, None, None) == L.PFMOE_OK
    assert lib.moe_expert_ffn(None, None, None, 0, 4, 64, 64, L.PFMOE_BF16, None, None, None, None, None, None,
                              None, None, None) == L.PFMOE_OK
    assert lib.moe_expert_ffn_gathered(None, None, None, None, 0, 4, 64, 64, L.PFMOE_BF16, None, None, None, None,
                                       None, None, None, None, None) == L.PFMOE_OK


def test_workspace_sizes(lib):
    for dt, es in ((L.PFMOE_BF16, 2), (L.PFMOE_F32, 4)):
        T, d, E, h, k = 300, 256, 12, 192, 3
        N = T * k
        b = lib.moe_backward_workspace_size(T, d, E, h, k, dt)
        # dO + dH1 + dH3 + dX_pft at least
        assert b >= (2 * N * d + 2 * N * h) * es
        assert b % 256 == 0
        assert lib.moe_backward_workspace_size(T, d, E, h, k, 5) == 0
    assert lib.pft_build_workspace_size(4096, 64, 6) >= 2 * 64 * 4
    assert lib.rbd_plan_workspace_size(8192, 8, 256, 8, 4) > 0
