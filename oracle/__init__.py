"""CPU oracle for the expert-parallel dispatch/combine path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``combine_ep_get_08_b200``) never does: it has no CPU fallback.

The arithmetic lives in ``ep_oracle.c`` (plain C, single-threaded, built with
gcc without fast-math and without FP contraction).  This module only compiles
it and marshals numpy arrays through ctypes.  Each wrapper names the passage
it follows in the docstring of the C function it calls.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(worked example from the lesson14_deepep practice task, brute force against a
sort-based definition, exhaustive E4M3 checks, round-trip and dense-reference
invariants).  None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, BAD_EXPERT, BAD_ARG, SLOT_OVERFLOW = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile ep_oracle.c into liboracle.so next to it (no-op if up to date)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode_array.argtypes = [i64, P, P]
    lib.oracle_e4m3_encode_array.restype = None
    lib.oracle_capacity_rows.argtypes = [i32, i32, i32, i32]
    lib.oracle_capacity_rows.restype = i64
    lib.oracle_layout.argtypes = [i32, i32, i32, i32, i32] + [P] * 11
    lib.oracle_layout.restype = ctypes.c_int
    lib.oracle_ll_layout.argtypes = [i32, i32, i32, i32, P, P, P]
    lib.oracle_ll_layout.restype = ctypes.c_int
    lib.oracle_dispatch_bf16.argtypes = [i32, i32, i32, P, P, P, P]
    lib.oracle_dispatch_bf16.restype = ctypes.c_int
    lib.oracle_dispatch_fp8.argtypes = [i32, i32, i32, P, P, P, P, P]
    lib.oracle_dispatch_fp8.restype = ctypes.c_int
    lib.oracle_expert_combine.argtypes = [i32] * 6 + [P] * 5 + [i32, P, P]
    lib.oracle_expert_combine.restype = ctypes.c_int
    lib.oracle_combine.argtypes = [i32, i32, i32, i32, P, P, P, i32, P, P]
    lib.oracle_combine.restype = ctypes.c_int
    lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_value.restype = ctypes.c_double
    lib.oracle_expert_combine_fp8.argtypes = [i32] * 6 + [P] * 4 + [i64] + [P] * 3 + [i32, P, P]
    lib.oracle_expert_combine_fp8.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


class use_library:
    """Context manager that points this module at another build of the
    oracle's C source (the mutation tests compile deliberately broken copies
    to show that the pins catch them)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self._saved = _load()
        with _lock:
            _lib = _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self._saved


def compile_source(src_text: str, out_path: str) -> str:
    """Compile a variant of ep_oracle.c (given as text) to a shared library."""
    c_path = out_path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    cmd = ["gcc", "-O1", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", out_path, c_path, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def e4m3_encode(v) -> np.ndarray:
    """fp32 values -> OCP E4M3 codes (round to nearest even, saturate at 448)."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(v.size, _ptr(v), _ptr(out))
    return out


def capacity_rows(T: int, E: int, K: int, A: int) -> int:
    return int(_load().oracle_capacity_rows(T, E, K, A))


class Layout:
    """Result of :func:`layout` (numpy arrays; rows = expert_offsets[-1])."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def layout(topk_idx, num_experts: int, num_ranks: int, expert_alignment: int = 1,
           topk_weights=None) -> Layout:
    """Counts, offsets and the stable (token, k) -> row permutation."""
    idx = _c(topk_idx, np.int64)
    T, K = idx.shape
    E, R, A = num_experts, num_ranks, expert_alignment
    cap = max(capacity_rows(T, E, K, A), 0)
    # slack rows past the capacity: a layout that overruns it is reported as
    # an error (BAD_ARG) instead of writing outside the buffer
    room = cap + E + 16
    w = None if topk_weights is None else _c(topk_weights, np.float32)
    out = Layout(
        num_tokens_per_expert=np.zeros(E, np.int32),
        num_tokens_per_rank=np.zeros(R, np.int32),
        is_token_in_rank=np.zeros((T, R), np.uint8),
        expert_offsets=np.zeros(E + 1, np.int32),
        rank_offsets=np.zeros(R + 1, np.int32),
        pos=np.zeros((T, K), np.int32),
        row_src=np.full(room, -7, np.int32),
        row_slot=np.full(room, -7, np.int32),
        row_weight=np.zeros(room, np.float32),
    )
    rc = _load().oracle_layout(
        T, E, R, K, A, _ptr(idx), _ptr(w), _ptr(out.num_tokens_per_expert),
        _ptr(out.num_tokens_per_rank), _ptr(out.is_token_in_rank),
        _ptr(out.expert_offsets), _ptr(out.rank_offsets), _ptr(out.pos),
        _ptr(out.row_src), _ptr(out.row_slot), _ptr(out.row_weight))
    out.status = rc
    if rc == OK and int(out.expert_offsets[-1]) > cap:
        out.status = BAD_ARG
    if out.status == OK:
        rows = int(out.expert_offsets[-1])
        out.rows = rows
        out.row_src = out.row_src[:rows]
        out.row_slot = out.row_slot[:rows]
        out.row_weight = out.row_weight[:rows]
    out.capacity = cap
    return out


def ll_layout(topk_idx, num_experts: int, max_tokens: int) -> Layout:
    """Low-latency static layout: M = max_tokens slots per expert.

    Fields: status (OK, BAD_EXPERT or SLOT_OVERFLOW), recv_count [E],
    pos [T, K] (e*M + slot, or -1), capacity = E*M, and row_src [E*M]
    (token of each used slot, -1 elsewhere) for the dispatch functions."""
    idx = _c(topk_idx, np.int64)
    T, K = idx.shape
    E, M = num_experts, max_tokens
    out = Layout(recv_count=np.zeros(E, np.int32), pos=np.zeros((T, K), np.int32), capacity=E * M)
    out.status = _load().oracle_ll_layout(T, E, K, M, _ptr(idx), _ptr(out.recv_count), _ptr(out.pos))
    if out.status in (OK, SLOT_OVERFLOW):
        src = np.full(E * M, -1, np.int32)
        used = out.pos >= 0
        src[out.pos[used]] = np.nonzero(used)[0].astype(np.int32)
        out.row_src = src
    return out


def dispatch_bf16(x_bits, row_src, sel_rows=None) -> np.ndarray:
    """Received bf16 rows (as uint16 bit patterns) for all or selected rows."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    src = _c(row_src, np.int32)
    sel = None if sel_rows is None else _c(sel_rows, np.int32)
    n = src.shape[0] if sel is None else sel.shape[0]
    out = np.empty((n, H), np.uint16)
    rc = _load().oracle_dispatch_bf16(T, H, n, _ptr(sel), _ptr(src), _ptr(x), _ptr(out))
    if rc != OK:
        raise ValueError(f"oracle_dispatch_bf16 failed ({rc})")
    return out


def dispatch_fp8(x_bits, row_src, sel_rows=None):
    """Received E4M3 codes [n, H] and fp32 scales [n, H/128]."""
    x = _c(x_bits, np.uint16)
    T, H = x.shape
    src = _c(row_src, np.int32)
    sel = None if sel_rows is None else _c(sel_rows, np.int32)
    n = src.shape[0] if sel is None else sel.shape[0]
    q = np.empty((n, H), np.uint8)
    s = np.empty((n, H // 128), np.float32)
    rc = _load().oracle_dispatch_fp8(T, H, n, _ptr(sel), _ptr(src), _ptr(x), _ptr(q), _ptr(s))
    if rc != OK:
        raise ValueError(f"oracle_dispatch_fp8 failed ({rc})")
    return q, s


def combine(y_bits, pos, topk_weights, sel_tokens=None) -> np.ndarray:
    """fp64 weighted sum over k of the received rows, per (selected) token."""
    y = _c(y_bits, np.uint16)
    rows, H = y.shape
    p = _c(pos, np.int32)
    T, K = p.shape
    w = _c(topk_weights, np.float32)
    sel = None if sel_tokens is None else _c(sel_tokens, np.int32)
    n = T if sel is None else sel.shape[0]
    out = np.empty((n, H), np.float64)
    rc = _load().oracle_combine(T, H, K, rows, _ptr(p), _ptr(y), _ptr(w), n, _ptr(sel), _ptr(out))
    if rc != OK:
        raise ValueError(f"oracle_combine failed ({rc})")
    return out


def expert_combine(act_bits, w_bits, topk_idx, pos, topk_weights, sel_tokens=None) -> np.ndarray:
    """fp64 out[t] = sum_k w[t,k] * act[pos[t,k]] @ W[topk_idx[t,k]]^T (see ep_oracle.c)."""
    act = _c(act_bits, np.uint16)
    rows, I = act.shape
    w = _c(w_bits, np.uint16)
    E, N, I2 = w.shape
    assert I2 == I
    idx = _c(topk_idx, np.int64)
    p = _c(pos, np.int32)
    T, K = p.shape
    tw = _c(topk_weights, np.float32)
    sel = None if sel_tokens is None else _c(sel_tokens, np.int32)
    n = T if sel is None else sel.shape[0]
    out = np.empty((n, N), np.float64)
    rc = _load().oracle_expert_combine(T, K, I, N, E, rows, _ptr(idx), _ptr(p), _ptr(act), _ptr(w), _ptr(tw),
                                       n, _ptr(sel), _ptr(out))
    if rc != OK:
        raise ValueError(f"oracle_expert_combine failed ({rc})")
    return out


def e4m3_value(code: int) -> float:
    """Value of one OCP E4M3 code (see ep_oracle.c)."""
    return float(_load().oracle_e4m3_value(int(code) & 0xFF))


def expert_combine_fp8(act_q, act_scale, w_q, w_scale, topk_idx, pos, topk_weights, scale_ld: int = 0,
                       sel_tokens=None) -> np.ndarray:
    """fp64 out[t] = sum_k w[t,k] * A[pos[t,k]] @ W_e^T with A and W_e restored from E4M3 codes and
    their block scales (1x128 for the rows, 128x128 for the expert matrices; see ep_oracle.c).
    act_scale is row-major [rows, I/128] when scale_ld == 0, else column-major with that leading
    dimension."""
    a = _c(act_q, np.uint8)
    rows, I = a.shape
    sa = _c(act_scale, np.float32)
    if scale_ld == 0:
        assert sa.shape == (rows, I // 128)
    else:
        assert sa.size >= (I // 128) * scale_ld and scale_ld >= rows
    w = _c(w_q, np.uint8)
    E, N, I2 = w.shape
    assert I2 == I
    sw = _c(w_scale, np.float32)
    assert sw.shape == (E, N // 128, I // 128)
    idx = _c(topk_idx, np.int64)
    p = _c(pos, np.int32)
    T, K = p.shape
    tw = _c(topk_weights, np.float32)
    sel = None if sel_tokens is None else _c(sel_tokens, np.int32)
    n = T if sel is None else sel.shape[0]
    out = np.empty((n, N), np.float64)
    rc = _load().oracle_expert_combine_fp8(T, K, I, N, E, rows, _ptr(idx), _ptr(p), _ptr(a), _ptr(sa),
                                           int(scale_ld), _ptr(w), _ptr(sw), _ptr(tw), n, _ptr(sel), _ptr(out))
    if rc != OK:
        raise ValueError(f"oracle_expert_combine_fp8 failed ({rc})")
    return out

