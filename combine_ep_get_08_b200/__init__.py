"""Python binding of libep_b200.so (the sm_100a dispatch/combine library).

Argument marshalling only: every function below has the name of the C entry
point it calls (see include/ep.h), turns torch tensors / ints into raw
pointers and the current torch CUDA stream into a ``cudaStream_t``, and
raises :class:`EpError` on a negative return code.  All arithmetic runs in
the library's CUDA kernels; there is no CPU fallback: if the library is
missing every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("EP_B200_LIB", os.path.join(_HERE, "libep_b200.so"))

EP_OK, EP_ERR_ARG, EP_ERR_CUDA, EP_ERR_UNSUPPORTED, EP_ERR_STATE, EP_ERR_DEVICE = 0, -1, -2, -3, -4, -5
EP_DEV_BAD_EXPERT, EP_DEV_WAIT_TIMEOUT, EP_DEV_SLOT_OVERFLOW = 0x1, 0x2, 0x4
EP_SCALES_ROW_MAJOR, EP_SCALES_COL_MAJOR_TMA = 0, 1
EP_IPC_HANDLE_BYTES = 64


class EpError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({status_text(code)}){': ' + detail if detail else ''}")


class ep_config(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("num_ranks", ctypes.c_int32),
                ("num_topk", ctypes.c_int32), ("expert_alignment", ctypes.c_int32)]


class ep_handle_view(ctypes.Structure):
    _fields_ = [("pos", ctypes.c_void_p), ("row_src", ctypes.c_void_p),
                ("row_slot", ctypes.c_void_p), ("row_weight", ctypes.c_void_p),
                ("num_tokens_per_expert", ctypes.c_void_p), ("num_tokens_per_rank", ctypes.c_void_p),
                ("expert_offsets", ctypes.c_void_p), ("rank_offsets", ctypes.c_void_p),
                ("status", ctypes.c_void_p), ("capacity", ctypes.c_int64)]


_lock = threading.Lock()
_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA extension {LIB_PATH} is missing: build it with "
                "`python -m combine_ep_get_08_b200.build_lib` (nvcc, sm_100a). "
                "There is no CPU fallback.")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, I64, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
        CFG = ctypes.POINTER(ep_config)
        sig = {
            "ep_validate_config": ([CFG], ctypes.c_int),
            "ep_capacity_rows": ([CFG], I64),
            "ep_scales_per_row": ([CFG], I32),
            "ep_scale_buffer_floats": ([CFG, I32], I64),
            "ep_set_scale_layout": ([P, I32], ctypes.c_int),
            "ep_handle_create": ([CFG, ctypes.POINTER(P)], ctypes.c_int),
            "ep_handle_destroy": ([P], ctypes.c_int),
            "ep_handle_get_view": ([P, ctypes.POINTER(ep_handle_view)], ctypes.c_int),
            "ep_get_layout": ([P] + [P] * 7 + [P], ctypes.c_int),
            "ep_get_layout_noalloc": ([CFG] + [P] * 13, ctypes.c_int),
            "ep_layout_shape": ([CFG, ctypes.POINTER(I32), ctypes.POINTER(I32), ctypes.POINTER(I64)], ctypes.c_int),
            "ep_dispatch": ([P, P, P, P], ctypes.c_int),
            "ep_layout_dispatch": ([P] * 11, ctypes.c_int),
            "ep_layout_dispatch_fp8": ([P] * 12, ctypes.c_int),
            "ep_dispatch_fp8": ([P, P, P, P, P], ctypes.c_int),
            "ep_combine": ([P, P, P, P, P], ctypes.c_int),
            "ep_copy_routing": ([P, P, P, P, P, P], ctypes.c_int),
            "ep_get_num_rows": ([P, ctypes.POINTER(I32), P], ctypes.c_int),
            "ep_get_status": ([P, ctypes.POINTER(ctypes.c_uint32), P], ctypes.c_int),
            "ep_clear_status": ([P, P], ctypes.c_int),
            "ep_set_wait_limit": ([P, U64, I32], ctypes.c_int),
            "ep_set_sm_limit": ([P, I32], ctypes.c_int),
            "ep_expert_combine": ([P, P, I32, P, I32, P, P, P, P], ctypes.c_int),
            "ep_expert_combine_fp8": ([P, P, P, I32, P, P, I32, P, P, P, P], ctypes.c_int),
            "ep_ll_capacity_rows": ([CFG, I32], I64),
            "ep_ll_scale_buffer_floats": ([CFG, I32, I32], I64),
            "ep_ll_handle_create": ([CFG, I32, ctypes.POINTER(P)], ctypes.c_int),
            "ep_ll_dispatch": ([P] * 6, ctypes.c_int),
            "ep_ll_dispatch_fp8": ([P] * 7, ctypes.c_int),
            "ep_ll_combine": ([P] * 5, ctypes.c_int),
            "ep_dispatch_peer": ([P] * 5, ctypes.c_int),
            "ep_dispatch_peer_fp8": ([P] * 6, ctypes.c_int),
            "ep_combine_peer": ([P] * 6, ctypes.c_int),
            "ep_ipc_get_handle": ([P, P, ctypes.POINTER(I64)], ctypes.c_int),
            "ep_ipc_open_handle": ([P, ctypes.POINTER(P)], ctypes.c_int),
            "ep_ipc_close_handle": ([P], ctypes.c_int),
            "ep_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "ep_last_error": ([], ctypes.c_char_p),
            "ep_launch_count": ([], U64),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def library():
    """The loaded ctypes library (raises if the extension is missing)."""
    return _load()


def status_text(code: int) -> str:
    try:
        return _load().ep_status_string(code).decode()
    except Exception:  # noqa: BLE001 - only used to format an error message
        return "?"


def _check(fn: str, rc: int) -> int:
    if rc < 0:
        detail = _load().ep_last_error().decode() if rc in (EP_ERR_CUDA, EP_ERR_UNSUPPORTED) else ""
        raise EpError(fn, rc, detail)
    return rc


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr() if t.numel() else None
    raise TypeError(f"expected a tensor, an int pointer or None, got {type(t)}")


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_config(num_tokens, hidden, num_experts, num_ranks, num_topk, expert_alignment=1) -> ep_config:
    return ep_config(num_tokens, hidden, num_experts, num_ranks, num_topk, expert_alignment)


def ep_validate_config(cfg: ep_config) -> int:
    return _load().ep_validate_config(ctypes.byref(cfg))


def ep_capacity_rows(cfg: ep_config) -> int:
    return _check("ep_capacity_rows", _load().ep_capacity_rows(ctypes.byref(cfg)))


def ep_scales_per_row(cfg: ep_config) -> int:
    return _check("ep_scales_per_row", _load().ep_scales_per_row(ctypes.byref(cfg)))


def ep_scale_buffer_floats(cfg: ep_config, layout: int = EP_SCALES_ROW_MAJOR) -> int:
    return _check("ep_scale_buffer_floats", _load().ep_scale_buffer_floats(ctypes.byref(cfg), layout))


def ep_set_scale_layout(h: int, layout: int) -> None:
    _check("ep_set_scale_layout", _load().ep_set_scale_layout(h, layout))


def ep_handle_create(cfg: ep_config) -> int:
    out = ctypes.c_void_p()
    _check("ep_handle_create", _load().ep_handle_create(ctypes.byref(cfg), ctypes.byref(out)))
    return out.value


def ep_handle_destroy(h: int) -> None:
    _check("ep_handle_destroy", _load().ep_handle_destroy(h))


def ep_handle_get_view(h: int) -> ep_handle_view:
    v = ep_handle_view()
    _check("ep_handle_get_view", _load().ep_handle_get_view(h, ctypes.byref(v)))
    return v


def ep_get_layout(h: int, topk_idx, topk_weights=None, num_tokens_per_expert=None,
                  num_tokens_per_rank=None, is_token_in_rank=None, expert_offsets=None,
                  rank_offsets=None, stream=None) -> None:
    _check("ep_get_layout", _load().ep_get_layout(
        h, _ptr(topk_idx), _ptr(topk_weights), _ptr(num_tokens_per_expert),
        _ptr(num_tokens_per_rank), _ptr(is_token_in_rank), _ptr(expert_offsets),
        _ptr(rank_offsets), _stream(stream)))


def ep_get_layout_noalloc(cfg: ep_config, topk_idx, topk_weights, pos, row_src, row_slot, row_weight,
                          num_tokens_per_expert, num_tokens_per_rank, is_token_in_rank, expert_offsets,
                          rank_offsets, status, stream=None) -> None:
    """Layout into caller buffers without any allocation (see include/ep.h)."""
    _check("ep_get_layout_noalloc", _load().ep_get_layout_noalloc(
        ctypes.byref(cfg), _ptr(topk_idx), _ptr(topk_weights), _ptr(pos), _ptr(row_src), _ptr(row_slot),
        _ptr(row_weight), _ptr(num_tokens_per_expert), _ptr(num_tokens_per_rank), _ptr(is_token_in_rank),
        _ptr(expert_offsets), _ptr(rank_offsets), _ptr(status), _stream(stream)))


def ep_layout_shape(cfg: ep_config) -> tuple[int, int, int]:
    """(cluster, ctas, noalloc_scratch_bytes) of the layout launch on the current device."""
    cl, ctas, need = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int64()
    _check("ep_layout_shape", _load().ep_layout_shape(ctypes.byref(cfg), ctypes.byref(cl), ctypes.byref(ctas),
                                                      ctypes.byref(need)))
    return cl.value, ctas.value, need.value


def ep_dispatch(h: int, x, recv_x, stream=None) -> None:
    _check("ep_dispatch", _load().ep_dispatch(h, _ptr(x), _ptr(recv_x), _stream(stream)))


def ep_layout_dispatch(h: int, topk_idx, topk_weights, x, recv_x, num_tokens_per_expert=None,
                       num_tokens_per_rank=None, is_token_in_rank=None, expert_offsets=None, rank_offsets=None,
                       stream=None) -> None:
    _check("ep_layout_dispatch", _load().ep_layout_dispatch(
        h, _ptr(topk_idx), _ptr(topk_weights), _ptr(x), _ptr(recv_x), _ptr(num_tokens_per_expert),
        _ptr(num_tokens_per_rank), _ptr(is_token_in_rank), _ptr(expert_offsets), _ptr(rank_offsets),
        _stream(stream)))


def ep_layout_dispatch_fp8(h: int, topk_idx, topk_weights, x, recv_q, recv_scales, num_tokens_per_expert=None,
                           num_tokens_per_rank=None, is_token_in_rank=None, expert_offsets=None,
                           rank_offsets=None, stream=None) -> None:
    _check("ep_layout_dispatch_fp8", _load().ep_layout_dispatch_fp8(
        h, _ptr(topk_idx), _ptr(topk_weights), _ptr(x), _ptr(recv_q), _ptr(recv_scales),
        _ptr(num_tokens_per_expert), _ptr(num_tokens_per_rank), _ptr(is_token_in_rank), _ptr(expert_offsets),
        _ptr(rank_offsets), _stream(stream)))


def ep_dispatch_fp8(h: int, x, recv_q, recv_scales, stream=None) -> None:
    _check("ep_dispatch_fp8", _load().ep_dispatch_fp8(
        h, _ptr(x), _ptr(recv_q), _ptr(recv_scales), _stream(stream)))


def ep_combine(h: int, y, topk_weights, out, stream=None) -> None:
    _check("ep_combine", _load().ep_combine(h, _ptr(y), _ptr(topk_weights), _ptr(out), _stream(stream)))


def ep_dispatch_peer(h: int, x, recv_bases, row0, stream=None) -> None:
    """recv_bases: device int64 tensor of R buffer addresses; row0: device int32 [R]."""
    _check("ep_dispatch_peer", _load().ep_dispatch_peer(h, _ptr(x), _ptr(recv_bases), _ptr(row0), _stream(stream)))


def ep_dispatch_peer_fp8(h: int, x, recv_bases, scale_bases, row0, stream=None) -> None:
    """recv_bases / scale_bases: device int64 tensors of R code / scale buffer addresses."""
    _check("ep_dispatch_peer_fp8", _load().ep_dispatch_peer_fp8(h, _ptr(x), _ptr(recv_bases), _ptr(scale_bases),
                                                                _ptr(row0), _stream(stream)))


def ep_combine_peer(h: int, y_bases, row0, topk_weights, out, stream=None) -> None:
    _check("ep_combine_peer", _load().ep_combine_peer(h, _ptr(y_bases), _ptr(row0), _ptr(topk_weights), _ptr(out),
                                                      _stream(stream)))


def ep_ipc_get_handle(buf) -> tuple[bytes, int]:
    """(handle bytes, byte offset of `buf` inside its allocation)."""
    hd = ctypes.create_string_buffer(EP_IPC_HANDLE_BYTES)
    off = ctypes.c_int64()
    _check("ep_ipc_get_handle", _load().ep_ipc_get_handle(_ptr(buf), hd, ctypes.byref(off)))
    return hd.raw, off.value


def ep_ipc_open_handle(handle: bytes) -> int:
    """Maps another process's allocation; returns its base address."""
    if len(handle) != EP_IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {EP_IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    base = ctypes.c_void_p()
    _check("ep_ipc_open_handle", _load().ep_ipc_open_handle(ctypes.create_string_buffer(handle, len(handle)),
                                                            ctypes.byref(base)))
    return base.value


def ep_ipc_close_handle(base: int) -> None:
    _check("ep_ipc_close_handle", _load().ep_ipc_close_handle(base))


def ep_copy_routing(h: int, pos=None, row_src=None, row_slot=None, row_weight=None, stream=None) -> None:
    _check("ep_copy_routing", _load().ep_copy_routing(
        h, _ptr(pos), _ptr(row_src), _ptr(row_slot), _ptr(row_weight), _stream(stream)))


def ep_get_num_rows(h: int, stream=None) -> int:
    rows = ctypes.c_int32()
    _check("ep_get_num_rows", _load().ep_get_num_rows(h, ctypes.byref(rows), _stream(stream)))
    return rows.value


def ep_get_status(h: int, stream=None) -> int:
    """Device status bits (0 = fine).  Synchronises the stream."""
    bits = ctypes.c_uint32()
    rc = _load().ep_get_status(h, ctypes.byref(bits), _stream(stream))
    if rc not in (EP_OK, EP_ERR_DEVICE):
        _check("ep_get_status", rc)
    return bits.value


def ep_clear_status(h: int, stream=None) -> None:
    _check("ep_clear_status", _load().ep_clear_status(h, _stream(stream)))


def ep_set_sm_limit(h: int, num_sms: int) -> None:
    _check("ep_set_sm_limit", _load().ep_set_sm_limit(h, num_sms))


def ep_set_wait_limit(h: int, limit_ns: int, extra_arrivals: int = 0) -> None:
    _check("ep_set_wait_limit", _load().ep_set_wait_limit(h, limit_ns, extra_arrivals))


def ep_expert_combine(h: int, act, inner: int, w, n_out: int, topk_weights, out_acc, out, stream=None) -> None:
    _check("ep_expert_combine", _load().ep_expert_combine(
        h, _ptr(act), inner, _ptr(w), n_out, _ptr(topk_weights), _ptr(out_acc), _ptr(out), _stream(stream)))


def ep_expert_combine_fp8(h: int, act_q, act_scales, inner: int, w_q, w_scales, n_out: int, topk_weights, out_acc,
                          out, stream=None) -> None:
    _check("ep_expert_combine_fp8", _load().ep_expert_combine_fp8(
        h, _ptr(act_q), _ptr(act_scales), inner, _ptr(w_q), _ptr(w_scales), n_out, _ptr(topk_weights),
        _ptr(out_acc), _ptr(out), _stream(stream)))


def ep_ll_capacity_rows(cfg: ep_config, num_max_dispatch_tokens: int) -> int:
    return _check("ep_ll_capacity_rows", _load().ep_ll_capacity_rows(ctypes.byref(cfg), num_max_dispatch_tokens))


def ep_ll_scale_buffer_floats(cfg: ep_config, num_max_dispatch_tokens: int,
                              layout: int = EP_SCALES_ROW_MAJOR) -> int:
    return _check("ep_ll_scale_buffer_floats",
                  _load().ep_ll_scale_buffer_floats(ctypes.byref(cfg), num_max_dispatch_tokens, layout))


def ep_ll_handle_create(cfg: ep_config, num_max_dispatch_tokens: int) -> int:
    out = ctypes.c_void_p()
    _check("ep_ll_handle_create",
           _load().ep_ll_handle_create(ctypes.byref(cfg), num_max_dispatch_tokens, ctypes.byref(out)))
    return out.value


def ep_ll_dispatch(h: int, topk_idx, x, recv_x, recv_count=None, stream=None) -> None:
    _check("ep_ll_dispatch", _load().ep_ll_dispatch(
        h, _ptr(topk_idx), _ptr(x), _ptr(recv_x), _ptr(recv_count), _stream(stream)))


def ep_ll_dispatch_fp8(h: int, topk_idx, x, recv_q, recv_scales, recv_count=None, stream=None) -> None:
    _check("ep_ll_dispatch_fp8", _load().ep_ll_dispatch_fp8(
        h, _ptr(topk_idx), _ptr(x), _ptr(recv_q), _ptr(recv_scales), _ptr(recv_count), _stream(stream)))


def ep_ll_combine(h: int, y, topk_weights, out, stream=None) -> None:
    _check("ep_ll_combine", _load().ep_ll_combine(h, _ptr(y), _ptr(topk_weights), _ptr(out), _stream(stream)))


def ep_status_string(code: int) -> str:
    return _load().ep_status_string(code).decode()


def ep_last_error() -> str:
    return _load().ep_last_error().decode()


def ep_launch_count() -> int:
    return int(_load().ep_launch_count())
