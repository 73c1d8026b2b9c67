"""pft_build_no_ws: the PFT build for callers that cannot allocate device memory.

Such a caller (for example a process whose device memory is carved out entirely
by another pool, or a fixed C interface that only passes input and output
pointers) gets its scratch from an array built into the library instead of a
workspace argument.  Its results must equal pft_build's exactly, call after
call, although every call reuses the same array and finds the previous call's
contents in it.
"""
import pytest
import torch

from padding_free_moe_b200 import _lib as L
from workloads.generate import make_topk_ids


def _outputs(T, E, k):
    i32 = dict(device="cuda", dtype=torch.int32)
    N = T * k
    return {
        "tpe": torch.full((E,), -1, **i32), "off": torch.full((E + 1,), -1, **i32),
        "tok": torch.full((N,), -1, **i32), "eid": torch.full((N,), -1, **i32),
        "cw": torch.full((N,), -1.0, device="cuda"), "pos": torch.full((T, k), -1, **i32),
        "tiles": torch.full((E + 1,), -1, **i32),
    }


def _run(fn, ids, w, T, E, k, *ws):
    o = _outputs(T, E, k)
    err = torch.zeros(1, device="cuda", dtype=torch.int32)
    fn(ids, w, T, E, k, o["tpe"], o["off"], o["tok"], o["eid"], o["cw"], o["pos"], o["tiles"], *ws, err)
    torch.cuda.synchronize()
    assert int(err) == 0
    return o


@pytest.mark.gpu
def test_pft_build_no_ws_matches_pft_build_twice():
    L.lib()
    # Calls in a row with different shapes and routings: each call sees the previous call's
    # leftovers in the built-in scratch array.  The second and fourth shapes have more than 64
    # chunks of keys, so their chunk counts are scanned per key (the many-chunk path, which
    # also uses the key-total region of the array), and the fourth runs over the first three's
    # leftovers in every region it uses.
    for T, E, k, seed in ((4096, 64, 6, 11), (20000, 1024, 8, 13), (1500, 256, 8, 12), (32768, 256, 8, 14)):
        assert L.pft_build_workspace_size(T, E, k) <= L.PFT_NO_WS_SCRATCH_BYTES
        ids = make_topk_ids(T, E, k, seed=seed, device="cuda")
        w = torch.rand(T, k, device="cuda")
        ws_b = L.pft_build_workspace_size(T, E, k)
        ws = torch.empty(ws_b, device="cuda", dtype=torch.uint8)
        ref = _run(L.pft_build, ids, w, T, E, k, ws, ws_b)
        got = _run(L.pft_build_no_ws, ids, w, T, E, k)
        for name in ref:
            assert torch.equal(ref[name], got[name]), name


@pytest.mark.gpu
def test_pft_build_no_ws_rejects_oversize_shapes():
    T, E, k = 1 << 20, 1024, 8      # needs far more scratch than the built-in array holds
    assert L.pft_build_workspace_size(T, E, k) > L.PFT_NO_WS_SCRATCH_BYTES
    o = _outputs(4, E, 1)           # never written: the call is rejected before any launch
    fake = o["tok"]
    with pytest.raises(L.PFMoEError, match="bytes of scratch"):
        L.pft_build_no_ws(fake, fake, T, E, k, o["tpe"], o["off"], fake, fake, fake, fake, o["tiles"])
