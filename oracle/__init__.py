"""fp64 CPU oracle for paged attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and it
never calls the CUDA library: the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, compiled with
gcc on first use); ``brute.py`` is an independent pure-Python brute force used
to pin it on tiny inputs.  Every function here is argument marshalling around
the C entry points.  bf16 tensors are passed as numpy uint16 bit patterns.

Parity pins (see tests/test_oracle_*.py): pure-Python brute force, closed
forms (constant V, zero Q, single key, peaked softmax, a hand-worked two-key
example), torch's fp64 scaled_dot_product_attention on unpaged data,
block-id permutation invariance, shared-vs-private prefix blocks, chunked
prefill invariance, split/merge identity, the KV-write round trip and the
block pack/unpack round trip checked against the gather.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-shared", "-fPIC",
                               "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    """Open a compiled oracle library and declare its entry points."""
    L = ctypes.CDLL(path)
    L.oracle_slot_mapping.argtypes = [_i32p, _i32p, _i32p, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_int32, _i64p]
    L.oracle_slot_mapping.restype = ctypes.c_int
    L.oracle_kv_write.argtypes = [_u16p, _u16p, ctypes.c_int64, _i64p, ctypes.c_int64, _u16p, _u16p,
                                  ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    L.oracle_kv_write.restype = ctypes.c_int
    L.oracle_gather_kv.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_int32, _i32p, ctypes.c_int64, ctypes.c_int32, _u16p]
    L.oracle_gather_kv.restype = ctypes.c_int
    L.oracle_kv_pack.argtypes = [_u16p, _u16p, ctypes.c_int64, ctypes.c_int64, _i32p, ctypes.c_int64, _u16p]
    L.oracle_kv_pack.restype = ctypes.c_int64
    L.oracle_kv_unpack.argtypes = [_u16p, _i32p, ctypes.c_int64, _u16p, _u16p, ctypes.c_int64, ctypes.c_int64]
    L.oracle_kv_unpack.restype = ctypes.c_int64
    L.oracle_attend_dense.argtypes = [_u16p, _u16p, _u16p, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_int64, ctypes.c_double, _f64p, _f64p, _f64p, _f64p]
    L.oracle_attend_dense.restype = None
    L.oracle_merge_states.argtypes = [_f64p, _f64p, ctypes.c_int32, ctypes.c_int32, _f64p, _f64p]
    L.oracle_merge_states.restype = None
    L.oracle_attention.argtypes = [
        _u16p, ctypes.c_int32, _u16p, _u16p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, _i32p, _i32p, _i32p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double,
        ctypes.c_void_p, ctypes.c_int32, _f64p, ctypes.c_void_p, _f64p, ctypes.c_int32]
    L.oracle_attention.restype = ctypes.c_int
    L.oracle_num_cores.restype = ctypes.c_int
    return L


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB)
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_cores() -> int:
    return int(_load().oracle_num_cores())


def slot_mapping(query_start_loc, seq_lens, block_table, block_size: int = 16) -> np.ndarray:
    """int64 [T]: slot of every token of the step (block_table[r][p//bs]*bs + p%bs)."""
    qsl = _c(query_start_loc, np.int32)
    bt = _c(block_table, np.int32)
    out = np.zeros(int(qsl[-1]), dtype=np.int64)
    rc = _load().oracle_slot_mapping(qsl, _c(seq_lens, np.int32), bt, bt.shape[1], len(qsl) - 1,
                                     block_size, out)
    if rc:
        raise ValueError("seq_len < q_len")
    return out


def kv_write(k_new, v_new, slots, k_cache, v_cache, row_stride=None):
    """Return copies of both pools after writing the new rows into their slots.

    k_new/v_new are [T, Hkv, D] arrays, or flat 1-D buffers whose token t
    starts at element t * row_stride (row_stride must then be given).
    """
    kn, vn = _c(k_new, np.uint16), _c(v_new, np.uint16)
    NB, Hkv, bs, D = k_cache.shape
    T = len(slots)
    if row_stride is None:
        assert kn.ndim == 3
        row_stride = Hkv * D
    kc, vc = np.array(k_cache, dtype=np.uint16, copy=True), np.array(v_cache, dtype=np.uint16, copy=True)
    rc = _load().oracle_kv_write(kn.reshape(-1), vn.reshape(-1), row_stride, _c(slots, np.int64), T,
                                 kc.reshape(-1), vc.reshape(-1), NB, Hkv, D, bs)
    if rc:
        raise ValueError("slot beyond the pool")
    return kc, vc


def gather_kv(cache, bt_row, seq_len: int, kv_head: int = -1) -> np.ndarray:
    """Contiguous [L, Hkv, D] (or [L, D] for one head) copy of a request's tokens."""
    c = _c(cache, np.uint16)
    NB, Hkv, bs, D = c.shape
    shape = (seq_len, Hkv, D) if kv_head < 0 else (seq_len, D)
    out = np.zeros(shape, dtype=np.uint16)
    rc = _load().oracle_gather_kv(c.reshape(-1), NB, Hkv, D, bs, _c(bt_row, np.int32), seq_len, kv_head,
                                  out.reshape(-1))
    if rc:
        raise ValueError("block id outside the pool")
    return out


def kv_pack(k_cache, v_cache, block_ids) -> np.ndarray:
    """Staging [n, 2, block_elems] (bf16 bits) of whole blocks block_ids (zeros for ids outside the pool)."""
    kc, vc = _c(k_cache, np.uint16), _c(v_cache, np.uint16)
    NB = kc.shape[0]
    elems = int(np.prod(kc.shape[1:]))
    ids = _c(block_ids, np.int32)
    out = np.zeros((len(ids), 2, elems), dtype=np.uint16)
    _load().oracle_kv_pack(kc.reshape(-1), vc.reshape(-1), NB, elems, ids, len(ids), out.reshape(-1))
    return out


def kv_unpack(staging, block_ids, k_cache, v_cache):
    """Copies of both pools with staging entry i written over block block_ids[i] (ids outside skipped)."""
    kc, vc = np.array(k_cache, dtype=np.uint16, copy=True), np.array(v_cache, dtype=np.uint16, copy=True)
    NB = kc.shape[0]
    elems = int(np.prod(kc.shape[1:]))
    ids = _c(block_ids, np.int32)
    _load().oracle_kv_unpack(_c(staging, np.uint16).reshape(-1), ids, len(ids), kc.reshape(-1), vc.reshape(-1),
                             NB, elems)
    return kc, vc


def attend_dense(q, K, V, scale: float):
    """Attention of one query row q [D] over contiguous keys K, V [n, D] (bf16 bits)."""
    q, K, V = _c(q, np.uint16), _c(K, np.uint16), _c(V, np.uint16)
    n, D = K.shape
    out = np.zeros(D, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    err = np.zeros(1, dtype=np.float64)
    scratch = np.zeros(max(n, 1), dtype=np.float64)
    _load().oracle_attend_dense(q, K.reshape(-1) if n else np.zeros(1, np.uint16),
                                V.reshape(-1) if n else np.zeros(1, np.uint16), n, D, D, scale, out, lse,
                                scratch, err)
    return out, float(lse[0]), float(err[0])


def merge_states(o, lse):
    """Merge per-part states (o [S, D], lse [S]) over disjoint key sets."""
    o = _c(o, np.float64)
    lse = _c(lse, np.float64)
    S, D = o.shape
    out = np.zeros(D, dtype=np.float64)
    lo = np.zeros(1, dtype=np.float64)
    _load().oracle_merge_states(o.reshape(-1), lse, S, D, out, lo)
    return out, float(lo[0])


def attention(q, k_cache, v_cache, query_start_loc, seq_lens, block_table, scale: float,
              token_list=None, nthreads: int = 0):
    """fp64 attention for one step.  Returns (out [T|n, Hq, D], lse [T|n, Hq], max |sum w - 1|)."""
    qb = _c(q, np.uint16)
    T, Hq, D = qb.shape
    kc, vc = _c(k_cache, np.uint16), _c(v_cache, np.uint16)
    NB, Hkv, bs, D2 = kc.shape
    assert D2 == D
    qsl = _c(query_start_loc, np.int32)
    bt = _c(block_table, np.int32)
    if bt.ndim == 1:
        bt = bt.reshape(len(qsl) - 1, -1)
    if token_list is not None:
        tl = _c(token_list, np.int32)
        n = len(tl)
        tl_ptr = tl.ctypes.data
    else:
        tl, n, tl_ptr = None, T, None
    out = np.zeros((n, Hq, D), dtype=np.float64)
    lse = np.zeros((n, Hq), dtype=np.float64)
    err = np.zeros(1, dtype=np.float64)
    rc = _load().oracle_attention(qb.reshape(-1), Hq, kc.reshape(-1), vc.reshape(-1), NB, Hkv, D, bs, qsl,
                                  _c(seq_lens, np.int32), bt.reshape(-1) if bt.size else np.zeros(1, np.int32),
                                  bt.shape[1] if bt.ndim == 2 else 0, len(qsl) - 1, float(scale), tl_ptr,
                                  n, out.reshape(-1), lse.ctypes.data, err, int(nthreads))
    if rc:
        raise ValueError(f"oracle_attention failed ({rc})")
    return out, lse, float(err[0])


def attention_for(layout, k_cache, v_cache, q, scale=None, **kw):
    """attention() with the metadata taken from a workloads.StepLayout."""
    if scale is None:
        scale = 1.0 / np.sqrt(layout.head_dim)
    return attention(q, k_cache, v_cache, layout.query_start_loc, layout.seq_lens, layout.block_table,
                     scale, **kw)
