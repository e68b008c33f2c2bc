"""ctypes binding of libpa_b200.so -- argument marshalling only.

Every function here has the name of a C entry point in include/pa.h minus the
``pa_`` prefix, takes torch CUDA tensors, passes their data pointers and the
current stream to the library, and raises PaError on a non-PA_OK status.  The
prefix-cache functions work on host numpy arrays (they never touch the GPU).
All arithmetic runs in the library's CUDA kernels; there is no fallback: if
the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_b200.so")

PA_OK = 0
STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_WORKSPACE_TOO_SMALL",
                4: "PA_ERR_CUDA"}
DEVICE_BAD_SEQ = 1
DEVICE_BAD_BLOCK = 2
DEVICE_WAIT_TIMEOUT = 4
DEVICE_BAD_SLOT = 8

# every symbol include/pa.h declares
EXPORTED = ("pa_abi_version", "pa_status_string", "pa_kv_write", "pa_build_slot_mapping", "pa_workspace_size",
            "pa_workspace_size_ex", "pa_attention_mixed", "pa_attention_mixed_ex", "pa_attention_mixed_noalloc",
            "pa_attention_decode_fused", "pa_kv_pack", "pa_kv_unpack", "pa_merge_attn_states", "pa_debug_gather_kv",
            "pa_prefix_block_hashes", "pa_prefix_cache_create", "pa_prefix_cache_destroy", "pa_prefix_cache_insert",
            "pa_prefix_cache_remove_block", "pa_prefix_cache_longest_hit", "pa_prefix_cache_size", "pa_kv_write_ex",
            "pa_noalloc_device_status", "pa_attention_mixed_write")
HASH_ALGOS = {"fnv1a64": 0, "sha256": 1}
LAYOUT_HND = 0   # cache [num_blocks, num_kv_heads, 16, head_dim]
LAYOUT_NHD = 1   # cache [num_blocks, 16, num_kv_heads, head_dim]
_LAYOUTS = {"HND": LAYOUT_HND, "NHD": LAYOUT_NHD}
NOALLOC_SCRATCH_BYTES = 64 << 20


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int64), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("layout", ctypes.c_int32)]


class AttnOptions(ctypes.Structure):
    _fields_ = [("kv_split_tokens", ctypes.c_int32), ("decode_max_query_len", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 6), ("side_stream", ctypes.c_void_p), ("fork_event", ctypes.c_void_p),
                ("join_event", ctypes.c_void_p)]


_lib = None
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


def lib():
    """Open libpa_b200.so (built in place by paged_kv_cache_461_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_461_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.pa_abi_version.restype = _i32
        L.pa_status_string.restype = ctypes.c_char_p
        L.pa_status_string.argtypes = [ctypes.c_int]
        L.pa_kv_write.argtypes = [_vp, _vp, _i64, _vp, _i32, _vp, _vp, ctypes.POINTER(CacheDesc), _vp]
        L.pa_kv_write_ex.argtypes = [_vp, _vp, _i64, _vp, _i32, _vp, _vp, ctypes.POINTER(CacheDesc), _vp, _vp]
        L.pa_noalloc_device_status.argtypes = [_vp, _vp]
        L.pa_build_slot_mapping.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp]
        L.pa_workspace_size.argtypes = [_i32, _i32, _i32, ctypes.POINTER(CacheDesc), _i32]
        L.pa_workspace_size.restype = _sz
        L.pa_workspace_size_ex.argtypes = [_i32, _i32, _i32, ctypes.POINTER(CacheDesc), _i32,
                                           ctypes.POINTER(AttnOptions)]
        L.pa_workspace_size_ex.restype = _sz
        attn = [_vp, _i32, _vp, _vp, ctypes.POINTER(CacheDesc), _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                ctypes.c_float, _vp, _vp, _vp, _sz]
        L.pa_attention_mixed.argtypes = attn + [_vp]
        L.pa_attention_mixed_ex.argtypes = attn + [ctypes.POINTER(AttnOptions), _vp]
        L.pa_attention_mixed_noalloc.argtypes = attn[:-2] + [ctypes.POINTER(AttnOptions), _vp]
        L.pa_attention_decode_fused.argtypes = [_vp, _i32, _vp, _vp, _i64, _vp, _vp, ctypes.POINTER(CacheDesc), _vp,
                                                _vp, _vp, _i32, _i32, _i32, _i32, _i32, ctypes.c_float, _vp, _vp,
                                                _vp, _sz, ctypes.POINTER(AttnOptions), _vp]
        L.pa_attention_mixed_write.argtypes = [_vp, _i32, _vp, _vp, _i64, _vp, _vp, _vp, ctypes.POINTER(CacheDesc),
                                               _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, ctypes.c_float, _vp, _vp,
                                               _vp, _sz, ctypes.POINTER(AttnOptions), _vp]
        L.pa_kv_pack.argtypes = [_vp, _vp, ctypes.POINTER(CacheDesc), _vp, _i32, _vp, _vp]
        L.pa_kv_unpack.argtypes = [_vp, _vp, _i32, _vp, _vp, ctypes.POINTER(CacheDesc), _vp]
        L.pa_merge_attn_states.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]
        L.pa_debug_gather_kv.argtypes = [_vp, ctypes.POINTER(CacheDesc), _vp, _i32, _vp, _vp]
        L.pa_prefix_block_hashes.argtypes = [_vp, _i64, _vp, _i32, _vp, ctypes.POINTER(ctypes.c_int64)]
        L.pa_prefix_block_hashes.restype = ctypes.c_int
        L.pa_prefix_cache_create.restype = _vp
        L.pa_prefix_cache_create.argtypes = []
        L.pa_prefix_cache_destroy.argtypes = [_vp]
        L.pa_prefix_cache_destroy.restype = None
        L.pa_prefix_cache_insert.argtypes = [_vp, _vp, _vp, _i32]
        L.pa_prefix_cache_insert.restype = ctypes.c_int
        L.pa_prefix_cache_remove_block.argtypes = [_vp, _i32]
        L.pa_prefix_cache_remove_block.restype = ctypes.c_int
        L.pa_prefix_cache_longest_hit.argtypes = [_vp, _vp, _i32, _vp]
        L.pa_prefix_cache_longest_hit.restype = _i32
        L.pa_prefix_cache_size.argtypes = [_vp]
        L.pa_prefix_cache_size.restype = _i64
        for name in ("pa_kv_write", "pa_kv_write_ex", "pa_noalloc_device_status", "pa_build_slot_mapping", "pa_attention_mixed", "pa_attention_mixed_ex",
                     "pa_attention_mixed_noalloc", "pa_attention_decode_fused", "pa_attention_mixed_write",
                     "pa_kv_pack", "pa_kv_unpack",
                     "pa_merge_attn_states", "pa_debug_gather_kv"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != PA_OK:
        raise PaError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream=None, device: Optional[torch.device] = None):
    """The stream to enqueue on: torch's current stream unless one is given.  The library launches on
    the current CUDA device, so that device (and a given stream's) must be the tensors' device."""
    if device is not None:
        cur = torch.cuda.current_device()
        if device.index != cur:
            raise ValueError(f"the tensors are on {device} but the current CUDA device is cuda:{cur} "
                             f"(call under torch.cuda.device({device.index}))")
    if stream is None:
        stream = torch.cuda.current_stream()
    elif device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def cache_desc(k_cache: torch.Tensor, layout: str = "HND") -> CacheDesc:
    """Descriptor of a cache tensor: HND [NB, Hkv, 16, D] or NHD [NB, 16, Hkv, D]."""
    if layout == "HND":
        NB, Hkv, bs, D = k_cache.shape
    elif layout == "NHD":
        NB, bs, Hkv, D = k_cache.shape
    else:
        raise ValueError(f"unknown cache layout {layout!r}")
    return CacheDesc(NB, Hkv, D, bs, _LAYOUTS[layout])


# Side stream and fork/join events for running a mixed step's prefill kernel beside its decode kernel,
# created with torch (the library creates none) and kept per (device, caller stream, host thread), so
# that calls that may be issued at the same time never share them.
_SIDE = {}
_SIDE_LOCK = threading.Lock()


def _side_resources(stream_ptr: int) -> tuple:
    """(side stream, fork event, join event) for calls on the caller stream stream_ptr from this thread.
    Created on first use: make the first call on a stream before capturing it into a CUDA graph."""
    dev = torch.cuda.current_device()
    key = (dev, stream_ptr, threading.get_ident())
    with _SIDE_LOCK:
        r = _SIDE.get(key)
    if r is None:
        side = torch.cuda.Stream(device=dev, priority=-100)  # maps to the device's highest priority
        fork, join = torch.cuda.Event(), torch.cuda.Event()
        fork.record(side)            # torch creates a CUDA event at its first record
        join.record(side)
        r = (side, fork, join)
        with _SIDE_LOCK:
            r = _SIDE.setdefault(key, r)
    return r


def _may_fork(num_q_heads: int, k_cache: torch.Tensor, layout: str, max_query_len: int,
              decode_max_query_len: int) -> bool:
    """Whether a call can hold both prefill-shaped and decode-shaped requests (only then does the library use a
    side stream): a decode kernel exists and max_query_len reaches past the decode row limit."""
    Hkv = k_cache.shape[1] if layout == "HND" else k_cache.shape[2]
    G = max(1, num_q_heads // max(1, Hkv))
    if decode_max_query_len == -1:
        return False
    cap = decode_max_query_len * G if decode_max_query_len > 0 else (8 if G <= 8 else 16)
    return int(max_query_len) * G > cap


def _opts(kv_split_tokens: int, decode_max_query_len: int = 0, stream_ptr: Optional[int] = None
          ) -> Optional[AttnOptions]:
    """Options of a call; with stream_ptr, also the binding's side stream and events for that caller stream."""
    if not kv_split_tokens and not decode_max_query_len and stream_ptr is None:
        return None
    o = AttnOptions()
    o.kv_split_tokens = int(kv_split_tokens)
    o.decode_max_query_len = int(decode_max_query_len)
    if stream_ptr is not None:
        side, fork, join = _side_resources(stream_ptr)
        o.side_stream, o.fork_event, o.join_event = side.cuda_stream, fork.cuda_event, join.cuda_event
    return o


def _need(t: torch.Tensor, dtype, name: str, shape=None, dense: bool = False, device=None):
    """The library sees raw pointers only, so every tensor is checked here: dtype, then CUDA
    (and the same device as the call's other tensors), then contiguity and shape where the C
    layout has no strides."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor (got {type(t).__name__})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (got {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's other tensors on {device}")
    if dense and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")


def _need_caches(k_cache: torch.Tensor, v_cache: torch.Tensor, device=None):
    _need(k_cache, torch.bfloat16, "k_cache", dense=True, device=device)
    if k_cache.dim() != 4:
        raise ValueError(f"k_cache must be 4-D (got {tuple(k_cache.shape)})")
    _need(v_cache, torch.bfloat16, "v_cache", shape=k_cache.shape, dense=True, device=k_cache.device)


def _need_meta(query_start_loc: torch.Tensor, seq_lens: torch.Tensor, block_table: torch.Tensor, device):
    """query_start_loc int32 [R+1], seq_lens int32 [R], block_table int32 [R, >= blocks] with unit column
    stride (its row stride is passed as bt_stride)."""
    _need(seq_lens, torch.int32, "seq_lens", dense=True, device=device)
    if seq_lens.dim() != 1:
        raise ValueError("seq_lens must be 1-D")
    R = seq_lens.shape[0]
    _need(query_start_loc, torch.int32, "query_start_loc", shape=(R + 1,), dense=True, device=device)
    _need(block_table, torch.int32, "block_table", device=device)
    if block_table.dim() != 2 or block_table.shape[0] != R or (block_table.numel() and block_table.stride(1) != 1):
        raise ValueError("block_table must be int32 [num_seqs, max_blocks] with unit column stride")


def _need_new_rows(k_new: torch.Tensor, v_new: torch.Tensor, d: CacheDesc, device) -> int:
    """k_new/v_new [T, Hkv, D] bf16 whose rows may be strided (views into a fused QKV); returns the row stride."""
    _need(k_new, torch.bfloat16, "k_new", device=device)
    _need(v_new, torch.bfloat16, "v_new", shape=k_new.shape, device=device)
    if k_new.dim() != 3 or tuple(k_new.shape[1:]) != (d.num_kv_heads, d.head_dim):
        raise ValueError(f"k_new must be [T, {d.num_kv_heads}, {d.head_dim}] (got {tuple(k_new.shape)})")
    T = k_new.shape[0]
    if T and (k_new.stride(0) != v_new.stride(0) or k_new.stride(-1) != 1 or k_new.stride(-2) != k_new.shape[-1]
              or v_new.stride(-1) != 1 or v_new.stride(-2) != v_new.shape[-1]):
        raise ValueError("k_new and v_new need the same row stride and contiguous [Hkv, D] rows")
    return k_new.stride(0) if T else k_new.shape[-1] * k_new.shape[-2]


def _need_q_out(q: torch.Tensor, out: Optional[torch.Tensor], lse: Optional[torch.Tensor]):
    _need(q, torch.bfloat16, "q", dense=True)
    if q.dim() != 3:
        raise ValueError(f"q must be [num_tokens, num_q_heads, head_dim] (got {tuple(q.shape)})")
    if out is not None:
        _need(out, torch.bfloat16, "out", shape=q.shape, dense=True, device=q.device)
    if lse is not None:
        _need(lse, torch.float32, "lse", shape=q.shape[:2], dense=True, device=q.device)


# ---------------------------------------------------------------- entry points

def abi_version() -> int:
    return int(lib().pa_abi_version())


def kv_write(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor, k_cache: torch.Tensor,
             v_cache: torch.Tensor, stream=None, layout: str = "HND", status: Optional[torch.Tensor] = None) -> None:
    """pa_kv_write: k_new/v_new [T, Hkv, D] (rows may be strided), slot_mapping int64 [T].
    status (int32 [1] on the device, optional): pa_kv_write_ex ORs DEVICE_BAD_SLOT into it when a slot lies
    outside the pool (the caller clears it)."""
    _need_caches(k_cache, v_cache)
    d = cache_desc(k_cache, layout)
    row_stride = _need_new_rows(k_new, v_new, d, k_cache.device)
    T = k_new.shape[0]
    _need(slot_mapping, torch.int64, "slot_mapping", shape=(T,), dense=True, device=k_cache.device)
    if status is None:
        _check(lib().pa_kv_write(_ptr(k_new), _ptr(v_new), row_stride, _ptr(slot_mapping), T, _ptr(k_cache),
                                 _ptr(v_cache), ctypes.byref(d), _stream(stream, k_cache.device)), "pa_kv_write")
        return
    _need(status, torch.int32, "status", shape=(1,), dense=True, device=k_cache.device)
    _check(lib().pa_kv_write_ex(_ptr(k_new), _ptr(v_new), row_stride, _ptr(slot_mapping), T, _ptr(k_cache),
                                _ptr(v_cache), ctypes.byref(d), _ptr(status), _stream(stream, k_cache.device)),
           "pa_kv_write_ex")


def noalloc_device_status(stream=None) -> int:
    """pa_noalloc_device_status: the PA_DEVICE_* bits of the last pa_attention_mixed_noalloc call on the current
    device, read after the stream has finished the call."""
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = _stream(stream, out.device)
    _check(lib().pa_noalloc_device_status(_ptr(out), st), "pa_noalloc_device_status")
    return int(out.item())


def build_slot_mapping(query_start_loc: torch.Tensor, seq_lens: torch.Tensor, block_table: torch.Tensor,
                       num_tokens: int, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need_meta(query_start_loc, seq_lens, block_table, query_start_loc.device)
    if out is None:
        out = torch.full((num_tokens,), -1, dtype=torch.int64, device=query_start_loc.device)
    _need(out, torch.int64, "out", shape=(num_tokens,), dense=True, device=query_start_loc.device)
    _check(lib().pa_build_slot_mapping(_ptr(query_start_loc), _ptr(seq_lens), _ptr(block_table),
                                       block_table.stride(0), seq_lens.shape[0], num_tokens, _ptr(out),
                                       _stream(stream, query_start_loc.device)), "pa_build_slot_mapping")
    return out


def workspace_size(num_seqs: int, num_tokens: int, num_q_heads: int, k_cache_or_desc, max_seq_len: int,
                   kv_split_tokens: int = 0, decode_max_query_len: int = 0, layout: str = "HND") -> int:
    d = k_cache_or_desc if isinstance(k_cache_or_desc, CacheDesc) else cache_desc(k_cache_or_desc, layout)
    o = _opts(kv_split_tokens, decode_max_query_len)
    return int(lib().pa_workspace_size_ex(num_seqs, num_tokens, num_q_heads, ctypes.byref(d), max_seq_len,
                                          ctypes.byref(o) if o else None))


def alloc_workspace(num_seqs, num_tokens, num_q_heads, k_cache, max_seq_len, kv_split_tokens=0,
                    decode_max_query_len=0, layout: str = "HND") -> torch.Tensor:
    n = workspace_size(num_seqs, num_tokens, num_q_heads, k_cache, max_seq_len, kv_split_tokens, decode_max_query_len,
                       layout)
    if n == 0:
        raise PaError(1, "pa_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=k_cache.device)


def attention_mixed(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, query_start_loc: torch.Tensor,
                    seq_lens: torch.Tensor, block_table: torch.Tensor, max_query_len: int, max_seq_len: int,
                    softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    kv_split_tokens: int = 0, decode_max_query_len: int = 0, stream=None,
                    layout: str = "HND", concurrent: bool = True) -> torch.Tensor:
    """pa_attention_mixed[_ex]: q [T, Hq, D] bf16 -> out [T, Hq, D] bf16 (lse [T, Hq] fp32 if given).
    concurrent: pass the binding's side stream and events for this caller stream, so that a step holding
    both prefill and decode work runs the two kernels side by side (else one after the other)."""
    _need_q_out(q, out, lse)
    _need_caches(k_cache, v_cache, q.device)
    _need_meta(query_start_loc, seq_lens, block_table, q.device)
    T, Hq, D = q.shape
    R = seq_lens.shape[0]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(R, T, Hq, k_cache, max_seq_len, kv_split_tokens, decode_max_query_len, layout)
    _need(workspace, torch.uint8, "workspace", dense=True, device=q.device)
    d = cache_desc(k_cache, layout)
    st = _stream(stream, q.device)
    fork = concurrent and _may_fork(Hq, k_cache, layout, max_query_len, decode_max_query_len)
    o = _opts(kv_split_tokens, decode_max_query_len, (st.value or 0) if fork else None)
    _check(lib().pa_attention_mixed_ex(_ptr(q), Hq, _ptr(k_cache), _ptr(v_cache), ctypes.byref(d),
                                       _ptr(query_start_loc), _ptr(seq_lens), _ptr(block_table),
                                       block_table.stride(0), R, T, int(max_query_len), int(max_seq_len),
                                       float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       ctypes.byref(o) if o else None, st), "pa_attention_mixed")
    return out


def attention_mixed_write(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor,
                          k_cache: torch.Tensor, v_cache: torch.Tensor, query_start_loc: torch.Tensor,
                          seq_lens: torch.Tensor, block_table: torch.Tensor, max_query_len: int, max_seq_len: int,
                          softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                          lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                          kv_split_tokens: int = 0, decode_max_query_len: int = 0, stream=None,
                          layout: str = "HND", concurrent: bool = True) -> torch.Tensor:
    """pa_attention_mixed_write: kv_write(k_new, v_new, slot_mapping) and attention_mixed in one call, the
    write and the step's plan in one launch (k_new/v_new [T, Hkv, D], rows may be strided; slot_mapping
    int64 [T])."""
    _need_q_out(q, out, lse)
    _need_caches(k_cache, v_cache, q.device)
    _need_meta(query_start_loc, seq_lens, block_table, q.device)
    d = cache_desc(k_cache, layout)
    row_stride = _need_new_rows(k_new, v_new, d, q.device)
    T, Hq, D = q.shape
    R = seq_lens.shape[0]
    if k_new.shape[0] != T:
        raise ValueError(f"k_new has {k_new.shape[0]} rows, q has {T} tokens")
    _need(slot_mapping, torch.int64, "slot_mapping", shape=(T,), dense=True, device=q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(R, T, Hq, k_cache, max_seq_len, kv_split_tokens, decode_max_query_len, layout)
    _need(workspace, torch.uint8, "workspace", dense=True, device=q.device)
    st = _stream(stream, q.device)
    fork = concurrent and _may_fork(Hq, k_cache, layout, max_query_len, decode_max_query_len)
    o = _opts(kv_split_tokens, decode_max_query_len, (st.value or 0) if fork else None)
    _check(lib().pa_attention_mixed_write(_ptr(q), Hq, _ptr(k_new), _ptr(v_new), row_stride, _ptr(slot_mapping),
                                          _ptr(k_cache), _ptr(v_cache), ctypes.byref(d), _ptr(query_start_loc),
                                          _ptr(seq_lens), _ptr(block_table), block_table.stride(0), R, T,
                                          int(max_query_len), int(max_seq_len), float(softmax_scale), _ptr(out),
                                          _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          ctypes.byref(o) if o else None, st), "pa_attention_mixed_write")
    return out


def attention_mixed_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                            query_start_loc: torch.Tensor, seq_lens: torch.Tensor, block_table: torch.Tensor,
                            max_query_len: int, max_seq_len: int, softmax_scale: Optional[float] = None,
                            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            kv_split_tokens: int = 0, stream=None, layout: str = "HND",
                            concurrent: bool = True) -> torch.Tensor:
    """pa_attention_mixed_noalloc: like attention_mixed but with the library's built-in scratch
    (for callers that cannot allocate a workspace; calls that overlap on the GPU race on it)."""
    _need_q_out(q, out, lse)
    _need_caches(k_cache, v_cache, q.device)
    _need_meta(query_start_loc, seq_lens, block_table, q.device)
    T, Hq, D = q.shape
    R = seq_lens.shape[0]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    d = cache_desc(k_cache, layout)
    st = _stream(stream, q.device)
    fork = concurrent and _may_fork(Hq, k_cache, layout, max_query_len, 0)
    o = _opts(kv_split_tokens, 0, (st.value or 0) if fork else None)
    _check(lib().pa_attention_mixed_noalloc(_ptr(q), Hq, _ptr(k_cache), _ptr(v_cache), ctypes.byref(d),
                                            _ptr(query_start_loc), _ptr(seq_lens), _ptr(block_table),
                                            block_table.stride(0), R, T, int(max_query_len), int(max_seq_len),
                                            float(softmax_scale), _ptr(out), _ptr(lse),
                                            ctypes.byref(o) if o else None, st),
           "pa_attention_mixed_noalloc")
    return out


def attention_decode_fused(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
                           v_cache: torch.Tensor, query_start_loc: torch.Tensor, seq_lens: torch.Tensor,
                           block_table: torch.Tensor, max_query_len: int, max_seq_len: int,
                           softmax_scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                           kv_split_tokens: int = 0, decode_max_query_len: int = 0, stream=None,
                           layout: str = "HND") -> torch.Tensor:
    """pa_attention_decode_fused: writes k_new/v_new [T, Hkv, D] (rows may be strided) into their
    slots and attends, in the decode kernel; every request must be decode-shaped."""
    _need_q_out(q, out, lse)
    _need_caches(k_cache, v_cache, q.device)
    _need_meta(query_start_loc, seq_lens, block_table, q.device)
    d = cache_desc(k_cache, layout)
    row_stride = _need_new_rows(k_new, v_new, d, q.device)
    T, Hq, D = q.shape
    R = seq_lens.shape[0]
    if k_new.shape[0] != T:
        raise ValueError(f"k_new has {k_new.shape[0]} rows, q has {T} tokens")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(R, T, Hq, k_cache, max_seq_len, kv_split_tokens, decode_max_query_len, layout)
    _need(workspace, torch.uint8, "workspace", dense=True, device=q.device)
    o = _opts(kv_split_tokens, decode_max_query_len)
    _check(lib().pa_attention_decode_fused(_ptr(q), Hq, _ptr(k_new), _ptr(v_new), row_stride, _ptr(k_cache),
                                           _ptr(v_cache), ctypes.byref(d), _ptr(query_start_loc), _ptr(seq_lens),
                                           _ptr(block_table), block_table.stride(0), R, T, int(max_query_len),
                                           int(max_seq_len), float(softmax_scale), _ptr(out), _ptr(lse),
                                           _ptr(workspace), workspace.numel() * workspace.element_size(),
                                           ctypes.byref(o) if o else None, _stream(stream, q.device)),
           "pa_attention_decode_fused")
    return out


def kv_pack(k_cache: torch.Tensor, v_cache: torch.Tensor, block_ids: torch.Tensor,
            staging: Optional[torch.Tensor] = None, stream=None, layout: str = "HND") -> torch.Tensor:
    """pa_kv_pack: whole blocks block_ids (int32) -> staging bf16 [n, 2, block_elems]."""
    _need_caches(k_cache, v_cache)
    _need(block_ids, torch.int32, "block_ids", dense=True, device=k_cache.device)
    d = cache_desc(k_cache, layout)
    n = block_ids.shape[0]
    elems = d.num_kv_heads * d.block_size * d.head_dim
    if staging is None:
        staging = torch.empty((n, 2, elems), dtype=k_cache.dtype, device=k_cache.device)
    _need(staging, torch.bfloat16, "staging", shape=(n, 2, elems), dense=True, device=k_cache.device)
    _check(lib().pa_kv_pack(_ptr(k_cache), _ptr(v_cache), ctypes.byref(d), _ptr(block_ids), n, _ptr(staging),
                            _stream(stream, k_cache.device)), "pa_kv_pack")
    return staging


def kv_unpack(staging: torch.Tensor, block_ids: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              stream=None, layout: str = "HND") -> None:
    """pa_kv_unpack: staging bf16 [n, 2, block_elems] -> whole blocks block_ids of the caches."""
    _need_caches(k_cache, v_cache)
    _need(block_ids, torch.int32, "block_ids", dense=True, device=k_cache.device)
    d = cache_desc(k_cache, layout)
    n = block_ids.shape[0]
    _need(staging, torch.bfloat16, "staging", shape=(n, 2, d.num_kv_heads * d.block_size * d.head_dim), dense=True,
          device=k_cache.device)
    _check(lib().pa_kv_unpack(_ptr(staging), _ptr(block_ids), block_ids.shape[0], _ptr(k_cache), _ptr(v_cache),
                              ctypes.byref(d), _stream(stream, k_cache.device)), "pa_kv_unpack")


def merge_attn_states(part_out: torch.Tensor, part_lse: torch.Tensor, parts_per_row: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, lse_out: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """pa_merge_attn_states: part_out fp32 [N, H, S, D], part_lse fp32 [N, H, S] -> bf16 [N, H, D]."""
    _need(part_out, torch.float32, "part_out", dense=True)
    if part_out.dim() != 4:
        raise ValueError(f"part_out must be [N, H, S, D] (got {tuple(part_out.shape)})")
    N, H, S, D = part_out.shape
    dev = part_out.device
    _need(part_lse, torch.float32, "part_lse", shape=(N, H, S), dense=True, device=dev)
    if parts_per_row is not None:
        _need(parts_per_row, torch.int32, "parts_per_row", shape=(N,), dense=True, device=dev)
    if out is None:
        out = torch.empty((N, H, D), dtype=torch.bfloat16, device=dev)
    _need(out, torch.bfloat16, "out", shape=(N, H, D), dense=True, device=dev)
    if lse_out is not None:
        _need(lse_out, torch.float32, "lse_out", shape=(N, H), dense=True, device=dev)
    _check(lib().pa_merge_attn_states(_ptr(part_out), _ptr(part_lse), _ptr(parts_per_row), N, H, S, D, _ptr(out),
                                      _ptr(lse_out), _stream(stream, dev)), "pa_merge_attn_states")
    return out


def debug_gather_kv(cache: torch.Tensor, bt_row: torch.Tensor, seq_len: int, stream=None,
                    layout: str = "HND") -> torch.Tensor:
    _need(cache, torch.bfloat16, "cache", dense=True)
    _need(bt_row, torch.int32, "bt_row", dense=True, device=cache.device)
    d = cache_desc(cache, layout)
    if bt_row.numel() < (seq_len + d.block_size - 1) // d.block_size:
        raise ValueError("bt_row holds fewer block ids than seq_len needs")
    out = torch.empty((seq_len, d.num_kv_heads, d.head_dim), dtype=cache.dtype, device=cache.device)
    _check(lib().pa_debug_gather_kv(_ptr(cache), ctypes.byref(d), _ptr(bt_row), seq_len, _ptr(out),
                                    _stream(stream, cache.device)), "pa_debug_gather_kv")
    return out


# ---------------------------------------------------------------- prefix caching (host side)

def prefix_block_hashes(token_ids, algo: str = "fnv1a64", root: Optional[bytes] = None):
    """pa_prefix_block_hashes: chained digests of the full 16-token blocks of a host int32 token array,
    as a numpy uint8 array [len(token_ids) // 16, 32]."""
    import numpy as np
    toks = np.ascontiguousarray(token_ids, dtype=np.int32)
    out = np.zeros((len(toks) // 16, 32), dtype=np.uint8)
    n = ctypes.c_int64(0)
    r = None
    if root is not None:
        rb = np.frombuffer(bytes(root), dtype=np.uint8)
        if rb.size != 32:
            raise ValueError("root digest must be 32 bytes")
        r = rb.ctypes.data
    _check(lib().pa_prefix_block_hashes(toks.ctypes.data if len(toks) else None, len(toks), r, HASH_ALGOS[algo],
                                        out.ctypes.data if len(out) else None, ctypes.byref(n)),
           "pa_prefix_block_hashes")
    assert n.value == len(out)
    return out


class PrefixCache:
    """pa_prefix_cache_*: block digest -> physical block id, with the longest cached prefix lookup."""

    def __init__(self):
        self._h = lib().pa_prefix_cache_create()
        if not self._h:
            raise MemoryError("pa_prefix_cache_create")

    def close(self):
        if self._h:
            lib().pa_prefix_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def insert(self, hashes, block_ids) -> None:
        import numpy as np
        h = np.ascontiguousarray(hashes, dtype=np.uint8).reshape(-1, 32)
        b = np.ascontiguousarray(block_ids, dtype=np.int32)
        if len(h) != len(b):
            raise ValueError(f"{len(h)} hashes but {len(b)} block ids")
        _check(lib().pa_prefix_cache_insert(self._h, h.ctypes.data, b.ctypes.data, len(b)), "pa_prefix_cache_insert")

    def remove_block(self, block_id: int) -> None:
        _check(lib().pa_prefix_cache_remove_block(self._h, int(block_id)), "pa_prefix_cache_remove_block")

    def longest_hit(self, hashes):
        import numpy as np
        h = np.ascontiguousarray(hashes, dtype=np.uint8).reshape(-1, 32)
        out = np.zeros(len(h), dtype=np.int32)
        n = lib().pa_prefix_cache_longest_hit(self._h, h.ctypes.data if len(h) else None, len(h),
                                              out.ctypes.data if len(h) else None)
        if n < 0:
            raise PaError(1, "pa_prefix_cache_longest_hit")
        return out[:n]

    def __len__(self):
        return int(lib().pa_prefix_cache_size(self._h))


def read_device_status(workspace: torch.Tensor) -> int:
    """The PA_DEVICE_* bits the last call that used this workspace left (synchronises)."""
    return int(workspace[:4].view(torch.int32).item()) & 0xFFFFFFFF
