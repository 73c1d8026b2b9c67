"""ctypes binding of libpfmoe.so: the C ABI of include/pfmoe.h, same names.

Argument marshalling only.  Tensors are passed as their device pointers
(``tensor.data_ptr()``), ``None`` as NULL; ``stream`` defaults to torch's
current CUDA stream.  A non-zero status raises :class:`PFMoEError` with the
library's message.  There is no fallback: if the shared library is missing the
first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpfmoe.so")

PFMOE_OK, PFMOE_ERR_ARG, PFMOE_ERR_UNSUPPORTED, PFMOE_ERR_CUDA = 0, 1, 2, 3
PFMOE_F32, PFMOE_BF16 = 0, 1
DEV_BAD_EXPERT_ID, DEV_BAD_POS, DEV_TIMEOUT, DEV_NONFINITE = 1, 2, 4, 8
TILE_ROWS = 128
PFT_NO_WS_SCRATCH_BYTES = 1 << 20

_P = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t

# name -> (restype, argtypes)
SIGNATURES = {
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_abi_version": (_I, []),
    "moe_route_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "moe_route": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _Z, _P, _P]),
    "pft_build_workspace_size": (_Z, [_I, _I, _I]),
    "pft_build": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P, _P]),
    "pft_build_no_ws": (_I, [_P, _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "moe_expert_ffn": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_ffn_gathered": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_combine": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "moe_backward_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "moe_backward": (_I, [_P] * 16 + [_I] * 6 + [_P] * 7 + [_Z, _P, _P]),
    "rbd_plan_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "rbd_plan": (_I, [_P, _I, _I, _I, _I, _I] + [_P] * 10 + [_Z, _P, _P]),
    "moe_profile_enable": (_I, [_I]),
    "moe_profile_reset": (None, []),
    "moe_profile_read": (_I, [_P, _I, _I, _P, _P]),
    "moe_selftest_wait_timeout": (_I, [_P, ctypes.c_ulonglong, _P]),
}


class PFMoEError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


_lib = None


def lib():
    """Load libpfmoe.so (once) and declare its signatures."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m padding_free_moe_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(name: str, rc: int):
    if rc != PFMOE_OK:
        raise PFMoEError(name, rc, lib().moe_last_error().decode(errors="replace"))


def dtype_code(torch_dtype) -> int:
    import torch
    if torch_dtype == torch.bfloat16:
        return PFMOE_BF16
    if torch_dtype == torch.float32:
        return PFMOE_F32
    raise ValueError(f"unsupported dtype {torch_dtype}")


def moe_last_error() -> str:
    return lib().moe_last_error().decode(errors="replace")


def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_route_workspace_size(T, d, E, k, dtype) -> int:
    return lib().moe_route_workspace_size(T, d, E, k, dtype)


def moe_route(x, wg, bias, T, d, E, k, dtype, logits, topk_ids, topk_w, ws=None, ws_bytes=0, err=None, stream=None):
    _check("moe_route", lib().moe_route(_ptr(x), _ptr(wg), _ptr(bias), T, d, E, k, dtype, _ptr(logits),
                                        _ptr(topk_ids), _ptr(topk_w), _ptr(ws), ws_bytes, _ptr(err),
                                        _stream(stream)))


def pft_build_workspace_size(T, E, k) -> int:
    return lib().pft_build_workspace_size(T, E, k)


def pft_build(topk_ids, topk_w, T, E, k, tokens_per_expert, expert_offsets, token_ids, expert_ids, combine_weights,
              pos, tile_offsets, ws, ws_bytes, err=None, stream=None):
    _check("pft_build", lib().pft_build(_ptr(topk_ids), _ptr(topk_w), T, E, k, _ptr(tokens_per_expert),
                                        _ptr(expert_offsets), _ptr(token_ids), _ptr(expert_ids),
                                        _ptr(combine_weights), _ptr(pos), _ptr(tile_offsets), _ptr(ws), ws_bytes,
                                        _ptr(err), _stream(stream)))


def pft_build_no_ws(topk_ids, topk_w, T, E, k, tokens_per_expert, expert_offsets, token_ids, expert_ids,
                    combine_weights, pos, tile_offsets, err=None, stream=None):
    """pft_build without a workspace argument: for callers that cannot allocate device memory,
    the scratch comes from an array built into the library (PFT_NO_WS_SCRATCH_BYTES bytes)."""
    _check("pft_build_no_ws", lib().pft_build_no_ws(
        _ptr(topk_ids), _ptr(topk_w), T, E, k, _ptr(tokens_per_expert), _ptr(expert_offsets), _ptr(token_ids),
        _ptr(expert_ids), _ptr(combine_weights), _ptr(pos), _ptr(tile_offsets), _ptr(err), _stream(stream)))


def moe_dispatch(x, pos, T, k, d, dtype, x_pft, err=None, stream=None):
    _check("moe_dispatch", lib().moe_dispatch(_ptr(x), _ptr(pos), T, k, d, dtype, _ptr(x_pft), _ptr(err),
                                              _stream(stream)))


def moe_expert_ffn(x_pft, expert_offsets, tile_offsets, N, E, d, h, dtype, w1, w3, w2, h1, h3, a, out, err=None,
                   stream=None):
    _check("moe_expert_ffn", lib().moe_expert_ffn(_ptr(x_pft), _ptr(expert_offsets), _ptr(tile_offsets), N, E, d, h,
                                                  dtype, _ptr(w1), _ptr(w3), _ptr(w2), _ptr(h1), _ptr(h3), _ptr(a),
                                                  _ptr(out), _ptr(err), _stream(stream)))


def moe_expert_ffn_gathered(x, token_ids, expert_offsets, tile_offsets, N, E, d, h, dtype, w1, w3, w2, h1, h3, a, out,
                            err=None, stream=None):
    _check("moe_expert_ffn_gathered",
           lib().moe_expert_ffn_gathered(_ptr(x), _ptr(token_ids), _ptr(expert_offsets), _ptr(tile_offsets), N, E, d,
                                         h, dtype, _ptr(w1), _ptr(w3), _ptr(w2), _ptr(h1), _ptr(h3), _ptr(a),
                                         _ptr(out), _ptr(err), _stream(stream)))


def moe_combine(out, pos, topk_w, T, k, d, dtype, y, err=None, stream=None):
    _check("moe_combine", lib().moe_combine(_ptr(out), _ptr(pos), _ptr(topk_w), T, k, d, dtype, _ptr(y), _ptr(err),
                                            _stream(stream)))


def moe_backward_workspace_size(T, d, E, h, k, dtype) -> int:
    return lib().moe_backward_workspace_size(T, d, E, h, k, dtype)


def moe_backward(dy, x, wg, topk_w, topk_ids, pos, expert_offsets, tile_offsets, x_pft, h1, h3, a, out, w1, w3, w2,
                 T, d, E, h, k, dtype, dx, dwg, dw1, dw3, dw2, dlogits, ws, ws_bytes, err=None, stream=None):
    _check("moe_backward", lib().moe_backward(
        _ptr(dy), _ptr(x), _ptr(wg), _ptr(topk_w), _ptr(topk_ids), _ptr(pos), _ptr(expert_offsets),
        _ptr(tile_offsets), _ptr(x_pft), _ptr(h1), _ptr(h3), _ptr(a), _ptr(out), _ptr(w1), _ptr(w3), _ptr(w2),
        T, d, E, h, k, dtype, _ptr(dx), _ptr(dwg), _ptr(dw1), _ptr(dw3), _ptr(dw2), _ptr(dlogits), _ptr(ws),
        ws_bytes, _ptr(err), _stream(stream)))


def rbd_plan_workspace_size(T, k, E, experts_per_device, devices_per_node) -> int:
    return lib().rbd_plan_workspace_size(T, k, E, experts_per_device, devices_per_node)


def rbd_plan(topk_ids, T, k, E, experts_per_device, devices_per_node, pilots_per_node, node_offsets, pilot_token,
             pilot_node, pilot_device, replica_offsets, replica_expert, assign_pilot, counts, ws, ws_bytes, err=None,
             stream=None):
    _check("rbd_plan", lib().rbd_plan(
        _ptr(topk_ids), T, k, E, experts_per_device, devices_per_node, _ptr(pilots_per_node), _ptr(node_offsets),
        _ptr(pilot_token), _ptr(pilot_node), _ptr(pilot_device), _ptr(replica_offsets), _ptr(replica_expert),
        _ptr(assign_pilot), _ptr(counts), _ptr(ws), ws_bytes, _ptr(err), _stream(stream)))


def moe_profile_enable(on: bool):
    lib().moe_profile_enable(1 if on else 0)


def moe_profile_reset():
    lib().moe_profile_reset()


def moe_profile_read(max_entries: int = 64):
    """Synchronise on the recorded events and return {kernel name: (launches, total_ms)}; clears the record."""
    stride = 64
    names = ctypes.create_string_buffer(stride * max_entries)
    ms = (ctypes.c_double * max_entries)()
    cnt = (ctypes.c_int * max_entries)()
    n = lib().moe_profile_read(ctypes.cast(names, _P), stride, max_entries, ctypes.cast(ms, _P),
                               ctypes.cast(cnt, _P))
    if n < 0:
        raise PFMoEError("moe_profile_read", n, moe_last_error())
    out = {}
    for i in range(n):
        nm = names.raw[i * stride:(i + 1) * stride].split(b"\0", 1)[0].decode()
        out[nm] = (cnt[i], ms[i])
    return out


def moe_selftest_wait_timeout(err, limit_ns: int, stream=None):
    """Test support: a one-warp kernel whose bounded mbarrier wait must give up after limit_ns and
    set DEV_TIMEOUT in the device error word `err` (the context stays usable)."""
    _check("moe_selftest_wait_timeout", lib().moe_selftest_wait_timeout(_ptr(err), int(limit_ns), _stream(stream)))

