"""ctypes binding of libmoe.so: argument marshalling only.

Every function here has the name and argument order of the C entry point it
wraps (see include/moe.h); tensors are passed as raw device pointers, ``None``
as NULL, and the stream defaults to torch's current stream.  No arithmetic of
the layer happens in Python: a missing or unloadable library raises at import
of the first call, and there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libmoe.so")

(MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_INDEX_OOB, MOE_ERR_TIMEOUT,
 MOE_ERR_SCRATCH_LIMIT) = range(7)
MOE_DT_F32, MOE_DT_BF16 = 0, 1
MOE_ACT_GELU, MOE_ACT_SWIGLU = 0, 1


class MoeConfig(ctypes.Structure):
    """Mirror of ``moe_config`` (include/moe.h)."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "T", "D", "E", "ep_size", "top_k", "F", "act", "renormalize", "x_dtype",
        "router_dtype", "n_shared", "F_shared")]

    def __repr__(self):
        return "MoeConfig(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class MoeError(RuntimeError):
    def __init__(self, name, status):
        super().__init__(f"{name} failed: {moe_status_string(status)} ({status})")
        self.status = status


class MoeEpPeers(ctypes.Structure):
    """Mirror of ``moe_ep_peers`` (include/moe.h): P, cap and six device pointers to
    device arrays of P device pointers."""
    _fields_ = [("P", ctypes.c_int32), ("cap", ctypes.c_int32),
                ("cnt", ctypes.c_void_p), ("flags", ctypes.c_void_p), ("recv_x", ctypes.c_void_p),
                ("recv_src", ctypes.c_void_p), ("recv_rank", ctypes.c_void_p),
                ("y_back", ctypes.c_void_p)]


_lib = None
_vp, _i32p, _f32p, _cfgp = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(MoeConfig)
_SIGS = {
    "moe_validate_config": (ctypes.c_int, [_cfgp]),
    "moe_workspace_size": (ctypes.c_size_t, [_cfgp]),
    "moe_packed_weights_size": (ctypes.c_size_t, [_cfgp]),
    "moe_prepare_weights": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_route": (ctypes.c_int, [_cfgp, _vp, _f32p, _f32p, _f32p, _i32p, _f32p, _vp, _vp]),
    "moe_preprocess": (ctypes.c_int, [_cfgp, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p, _vp,
                                      _i32p, _vp]),
    "moe_dispatch_permute": (ctypes.c_int, [_cfgp, _vp, _i32p, _vp, _vp]),
    "moe_route_dispatch_is_fused": (ctypes.c_int32, [_cfgp]),
    "moe_route_dispatch": (ctypes.c_int, [_cfgp, _vp, _f32p, _f32p, _f32p, _i32p, _f32p, _i32p, _i32p,
                                          _i32p, _i32p, _i32p, _i32p, _vp, _vp, _i32p, _vp]),
    "moe_expert_ffn": (ctypes.c_int, [_cfgp, _vp, _vp, _i32p, _vp, _vp, _vp, _vp, _vp, _i32p, _vp]),
    "moe_combine_unpermute": (ctypes.c_int, [_cfgp, _vp, _i32p, _f32p, _vp, _vp, _vp, _vp]),
    "moe_forward": (ctypes.c_int, [_cfgp, _vp, _f32p, _f32p, _vp, _f32p, _i32p, _f32p, _i32p, _i32p,
                                   _i32p, _i32p, _i32p, _i32p, _vp, _vp, _vp, _vp, _vp, _vp, _i32p,
                                   _vp]),
    "moe_preprocess_noalloc": (ctypes.c_int, [_cfgp, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p, _i32p,
                                              _i32p, _vp]),
    "moe_shared_ffn": (ctypes.c_int, [_cfgp, _vp, _vp, _vp, _vp, _i32p, _vp]),
    "moe_ep_local_ids": (ctypes.c_int, [_cfgp, _i32p, _i32p, _i32p, _vp]),
    "moe_gather_rows": (ctypes.c_int, [_vp, _i32p, _vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                       _vp]),
    "moe_check_wait_timeout": (ctypes.c_int, [_vp, _i32p, _vp]),
    "moe_mxfp8_quantize": (ctypes.c_int, [_vp, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp]),
    "moe_packed_weights_mxfp8_size": (ctypes.c_size_t, [_cfgp]),
    "moe_workspace_mxfp8_size": (ctypes.c_size_t, [_cfgp]),
    "moe_prepare_weights_mxfp8": (ctypes.c_int, [_cfgp, _vp, _vp, _vp]),
    "moe_expert_ffn_mxfp8": (ctypes.c_int, [_cfgp, _vp, _vp, _i32p, _vp, _vp, _vp, _vp, _vp, _i32p, _vp]),
    "moe_dispatch_mxfp8": (ctypes.c_int, [_cfgp, _vp, _i32p, _i32p, _vp, _vp]),
    "moe_ep_send_counts": (ctypes.c_int, [_cfgp, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, _i32p,
                                          ctypes.c_uint32, _vp]),
    "moe_ep_send_rows": (ctypes.c_int, [_cfgp, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, _vp,
                                        _i32p, _i32p, _i32p, ctypes.c_uint32, _i32p, _i32p, _vp]),
    "moe_ep_recv_layout": (ctypes.c_int, [_cfgp, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, _i32p,
                                          ctypes.c_uint32, _i32p, _vp]),
    "moe_ep_return_rows": (ctypes.c_int, [_cfgp, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, _vp,
                                          _i32p, ctypes.c_uint32, _i32p, _i32p, _vp]),
    "moe_ep_wait_returned": (ctypes.c_int, [_cfgp, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_uint32, _i32p, _vp]),
    "moe_ep_expert_ffn_return": (ctypes.c_int, [_cfgp, _cfgp, ctypes.c_void_p, ctypes.c_int32, _vp, _i32p,
                                                _i32p, _i32p, _vp, _vp, _vp, _vp, ctypes.c_uint32, _i32p,
                                                _i32p, _vp]),
    "moe_router_filter_view": (ctypes.c_int, [_cfgp, ctypes.POINTER(ctypes.c_size_t),
                                              ctypes.POINTER(ctypes.c_int32),
                                              ctypes.POINTER(ctypes.c_size_t),
                                              ctypes.POINTER(ctypes.c_float)]),
    "moe_ipc_handle_bytes": (ctypes.c_int32, []),
    "moe_ipc_export": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint64)]),
    "moe_ipc_import": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_uint64, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_ipc_close": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_uint64]),
    "moe_instr_read": (ctypes.c_int, [ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_abi_version": (ctypes.c_int32, []),
}


ABI_VERSION = 3          # MOE_ABI_VERSION of include/moe.h


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by ``expert_dispatch_fp32_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so not built: {LIB_PATH} is missing "
                              "(run `python -m expert_dispatch_fp32_b200.build`)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        if L.moe_abi_version() != ABI_VERSION:
            raise ImportError(f"{LIB_PATH} has ABI version {L.moe_abi_version()}, this binding expects "
                              f"{ABI_VERSION} (rebuild with `python -m expert_dispatch_fp32_b200.build`)")
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    if st != MOE_OK:
        raise MoeError(name, st)


def moe_check_wait_timeout(barrier, status, stream=None):
    _call("moe_check_wait_timeout", _p(barrier), _p(status), _s(stream))


def moe_ep_send_counts(cfg, peers, rank0, nlocal, counts, epoch, stream=None):
    _call("moe_ep_send_counts", ctypes.byref(cfg), ctypes.addressof(peers), rank0, nlocal, _p(counts),
          epoch, _s(stream))


def moe_ep_send_rows(cfg, peers, rank0, nlocal, x, topk_idx, pos, expert_offsets, epoch, done, status,
                     stream=None):
    _call("moe_ep_send_rows", ctypes.byref(cfg), ctypes.addressof(peers), rank0, nlocal, _p(x),
          _p(topk_idx), _p(pos), _p(expert_offsets), epoch, _p(done), _p(status), _s(stream))


def moe_ep_recv_layout(cfg, peers, rank0, nlocal, local_offsets, epoch, status, stream=None):
    _call("moe_ep_recv_layout", ctypes.byref(cfg), ctypes.addressof(peers), rank0, nlocal,
          _p(local_offsets), epoch, _p(status), _s(stream))


def moe_ep_return_rows(cfg, peers, rank0, nlocal, y_recv, local_offsets, epoch, done, status, stream=None):
    _call("moe_ep_return_rows", ctypes.byref(cfg), ctypes.addressof(peers), rank0, nlocal, _p(y_recv),
          _p(local_offsets), epoch, _p(done), _p(status), _s(stream))


def moe_ep_expert_ffn_return(cfg, local_cfg, peers, rank, recv_x, recv_src, recv_rank, local_offsets,
                             packed, act, y_recv, workspace, epoch, done, status, stream=None):
    _call("moe_ep_expert_ffn_return", ctypes.byref(cfg), ctypes.byref(local_cfg), ctypes.addressof(peers),
          rank, _p(recv_x), _p(recv_src), _p(recv_rank), _p(local_offsets), _p(packed), _p(act), _p(y_recv),
          _p(workspace), epoch, _p(done), _p(status), _s(stream))


def moe_ep_wait_returned(cfg, peers, rank0, nlocal, epoch, status, stream=None):
    _call("moe_ep_wait_returned", ctypes.byref(cfg), ctypes.addressof(peers), rank0, nlocal, epoch,
          _p(status), _s(stream))


def moe_ipc_handle_bytes() -> int:
    return lib().moe_ipc_handle_bytes()


def moe_ipc_export(ptr) -> tuple[bytes, int]:
    """(handle bytes, offset) of the device allocation holding ``ptr`` (a tensor or an
    address)."""
    n = lib().moe_ipc_handle_bytes()
    h = ctypes.create_string_buffer(n)
    off = ctypes.c_uint64(0)
    _call("moe_ipc_export", _p(ptr), h, ctypes.byref(off))
    return h.raw, off.value


def moe_ipc_import(handle: bytes, offset: int) -> int:
    """Device address of another process's buffer (handle and offset from its
    moe_ipc_export)."""
    h = ctypes.create_string_buffer(bytes(handle), len(handle))
    out = ctypes.c_void_p(0)
    _call("moe_ipc_import", h, offset, ctypes.byref(out))
    return int(out.value or 0)


def moe_ipc_close(ptr: int, offset: int) -> None:
    _call("moe_ipc_close", ptr, offset)


INSTR_CTAS, INSTR_SLOTS = 160, 24


def moe_instr_read(kernel: int):
    """Cycle counters of an instrumented library (kernel 0: bf16 GEMMs, 1: MXFP8) as a
    [160, 24] uint64 numpy array; zeroes them on the device."""
    import numpy as np
    buf = (ctypes.c_uint64 * (INSTR_CTAS * INSTR_SLOTS))()
    _call("moe_instr_read", kernel, buf, INSTR_CTAS * INSTR_SLOTS)
    return np.frombuffer(buf, dtype=np.uint64).reshape(INSTR_CTAS, INSTR_SLOTS).copy()


def moe_mxfp8_quantize(x, rows, K, q, scales, stream=None):
    _call("moe_mxfp8_quantize", _p(x), rows, K, _p(q), _p(scales), _s(stream))


def moe_packed_weights_mxfp8_size(cfg) -> int:
    return lib().moe_packed_weights_mxfp8_size(ctypes.byref(cfg))


def moe_workspace_mxfp8_size(cfg) -> int:
    return lib().moe_workspace_mxfp8_size(ctypes.byref(cfg))


def moe_prepare_weights_mxfp8(cfg, packed, packed_mx, stream=None):
    _call("moe_prepare_weights_mxfp8", ctypes.byref(cfg), _p(packed), _p(packed_mx), _s(stream))


def moe_expert_ffn_mxfp8(cfg, x_perm, x, expert_offsets, packed, packed_mx, y_perm, shared_out,
                         workspace, status, stream=None):
    _call("moe_expert_ffn_mxfp8", ctypes.byref(cfg), _p(x_perm), _p(x), _p(expert_offsets), _p(packed),
          _p(packed_mx), _p(y_perm), _p(shared_out), _p(workspace), _p(status), _s(stream))


def moe_dispatch_mxfp8(cfg, x, src, expert_offsets, workspace, stream=None):
    _call("moe_dispatch_mxfp8", ctypes.byref(cfg), _p(x), _p(src), _p(expert_offsets), _p(workspace),
          _s(stream))


def moe_router_filter_view(cfg):
    """(approx_offset, approx_ld, wmax_offset, coef) of the tensor-core router's values
    in the workspace after moe_route, or None when cfg takes another router path."""
    ao, ld, wo, cf = ctypes.c_size_t(), ctypes.c_int32(), ctypes.c_size_t(), ctypes.c_float()
    st = lib().moe_router_filter_view(ctypes.byref(cfg), ctypes.byref(ao), ctypes.byref(ld),
                                      ctypes.byref(wo), ctypes.byref(cf))
    if st == MOE_ERR_UNSUPPORTED:
        return None
    if st != MOE_OK:
        raise MoeError("moe_router_filter_view", st)
    return ao.value, ld.value, wo.value, cf.value


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_validate_config(cfg: MoeConfig) -> int:
    return lib().moe_validate_config(ctypes.byref(cfg))


def moe_workspace_size(cfg: MoeConfig) -> int:
    return lib().moe_workspace_size(ctypes.byref(cfg))


def moe_packed_weights_size(cfg: MoeConfig) -> int:
    return lib().moe_packed_weights_size(ctypes.byref(cfg))


def moe_prepare_weights(cfg, w_gate_up, w_down, ws_gate_up, ws_down, packed, stream=None):
    _call("moe_prepare_weights", ctypes.byref(cfg), _p(w_gate_up), _p(w_down), _p(ws_gate_up),
          _p(ws_down), _p(packed), _s(stream))


def moe_route(cfg, x, w_router, expert_bias, logits_out, topk_idx, topk_w, workspace, stream=None):
    _call("moe_route", ctypes.byref(cfg), _p(x), _p(w_router), _p(expert_bias), _p(logits_out),
          _p(topk_idx), _p(topk_w), _p(workspace), _s(stream))


def moe_preprocess(cfg, topk_idx, counts, expert_offsets, rank_splits, rank_offsets, pos, src,
                   workspace, status, stream=None):
    _call("moe_preprocess", ctypes.byref(cfg), _p(topk_idx), _p(counts), _p(expert_offsets),
          _p(rank_splits), _p(rank_offsets), _p(pos), _p(src), _p(workspace), _p(status), _s(stream))


def moe_preprocess_noalloc(cfg, topk_idx, counts, expert_offsets, rank_splits, rank_offsets, pos,
                           src, status, stream=None):
    """moe_preprocess without a workspace, for callers that cannot allocate device
    memory (a plugin whose host framework owns all device memory, or a loop that
    cannot afford cudaMalloc's implicit synchronisation); scratch is a fixed array
    inside libmoe.so, so overlapping calls on different streams race."""
    _call("moe_preprocess_noalloc", ctypes.byref(cfg), _p(topk_idx), _p(counts), _p(expert_offsets),
          _p(rank_splits), _p(rank_offsets), _p(pos), _p(src), _p(status), _s(stream))


def moe_dispatch_permute(cfg, x, pos, x_perm, stream=None):
    _call("moe_dispatch_permute", ctypes.byref(cfg), _p(x), _p(pos), _p(x_perm), _s(stream))


def moe_route_dispatch(cfg, x, w_router, expert_bias, logits_out, topk_idx, topk_w, counts,
                       expert_offsets, rank_splits, rank_offsets, pos, src, x_perm, workspace, status,
                       stream=None):
    _call("moe_route_dispatch", ctypes.byref(cfg), _p(x), _p(w_router), _p(expert_bias),
          _p(logits_out), _p(topk_idx), _p(topk_w), _p(counts), _p(expert_offsets), _p(rank_splits),
          _p(rank_offsets), _p(pos), _p(src), _p(x_perm), _p(workspace), _p(status), _s(stream))


def moe_route_dispatch_is_fused(cfg) -> bool:
    return bool(lib().moe_route_dispatch_is_fused(ctypes.byref(cfg)))


def moe_expert_ffn(cfg, x_perm, x, expert_offsets, packed, act, y_perm, shared_out, workspace,
                   status, stream=None):
    _call("moe_expert_ffn", ctypes.byref(cfg), _p(x_perm), _p(x), _p(expert_offsets), _p(packed),
          _p(act), _p(y_perm), _p(shared_out), _p(workspace), _p(status), _s(stream))


def moe_shared_ffn(cfg, x, packed, shared_out, workspace, status, stream=None):
    _call("moe_shared_ffn", ctypes.byref(cfg), _p(x), _p(packed), _p(shared_out), _p(workspace),
          _p(status), _s(stream))


def moe_ep_local_ids(cfg, topk_idx, src, ids, stream=None):
    _call("moe_ep_local_ids", ctypes.byref(cfg), _p(topk_idx), _p(src), _p(ids), _s(stream))


def moe_gather_rows(src, index, dst, n, n_src, D, stream=None):
    _call("moe_gather_rows", _p(src), _p(index), _p(dst), n, n_src, D, _s(stream))


def moe_combine_unpermute(cfg, y_perm, pos, topk_w, x, shared_out, out, stream=None):
    _call("moe_combine_unpermute", ctypes.byref(cfg), _p(y_perm), _p(pos), _p(topk_w), _p(x),
          _p(shared_out), _p(out), _s(stream))


def moe_forward(cfg, x, w_router, expert_bias, packed, logits_out, topk_idx, topk_w, counts,
                expert_offsets, rank_splits, rank_offsets, pos, src, x_perm, act, y_perm, shared_out,
                out, workspace, status, stream=None):
    _call("moe_forward", ctypes.byref(cfg), _p(x), _p(w_router), _p(expert_bias), _p(packed),
          _p(logits_out), _p(topk_idx), _p(topk_w), _p(counts), _p(expert_offsets), _p(rank_splits),
          _p(rank_offsets), _p(pos), _p(src), _p(x_perm), _p(act), _p(y_perm), _p(shared_out),
          _p(out), _p(workspace), _p(status), _s(stream))
