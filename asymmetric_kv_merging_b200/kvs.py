"""ctypes binding of libkvs.so -- argument marshalling only.

Every function here turns torch tensors into raw pointers, calls the C entry point
of the same name (declared in include/kvs.h) on the current CUDA stream, and
raises KvsError on a non-OK status. All computation happens in the library's
CUDA kernels. Importing this module fails if the library is missing: there is
no other implementation to fall back to.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvs.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libkvs.so not built ({_LIB_PATH}); run python -m asymmetric_kv_merging_b200.build")
_lib = ctypes.CDLL(_LIB_PATH)

F32, BF16 = 0, 1
OP_SCORE, OP_MERGE, OP_DECODE, OP_PREFILL = 0, 1, 2, 3
SCOPE_HEAD, SCOPE_POOLED = 0, 1
FORM_FULL, FORM_DIAGONAL, FORM_PER_QUERY = 0, 1, 2
FLAG_BAD_LENGTH, FLAG_OUT_CAPACITY, FLAG_INPLACE_SPAN, FLAG_NONFINITE_STATS = 1, 2, 4, 8
FLAG_TIMEOUT, FLAG_BUDGET = 16, 32

STATUS = {0: "KVS_OK", 1: "KVS_ERR_INVALID_ARG", 2: "KVS_ERR_UNSUPPORTED", 3: "KVS_ERR_BUDGET",
          4: "KVS_ERR_WORKSPACE", 5: "KVS_ERR_ALIAS", 6: "KVS_ERR_CUDA"}

EXPORTS = ("kvs_workspace_size", "kvs_score_pairs", "kvs_merge_compact", "kvs_decode_attn",
           "kvs_device_flags", "kvs_status_str", "kvs_version", "kvs_launch_count",
           "kvs_decode_attn_static", "kvs_static_scratch_bytes", "kvs_score_pairs_form",
           "kvs_prefill_chunk", "kvs_plan_rounds", "kvs_static_device_flags",
           "kvs_stream_read")


class CacheDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H_kv", ctypes.c_int32), ("H_q", ctypes.c_int32),
                ("d", ctypes.c_int32), ("T_cap", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class KvsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} "
                         f"({_lib.kvs_status_str(status).decode()})")


_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_P = ctypes.POINTER(CacheDesc)
_lib.kvs_version.restype = _i32
_lib.kvs_launch_count.restype = ctypes.c_int64
_lib.kvs_status_str.restype = ctypes.c_char_p
_lib.kvs_status_str.argtypes = [ctypes.c_int]
_lib.kvs_workspace_size.restype = _sz
_lib.kvs_workspace_size.argtypes = [_P, _i32, _i32]
_lib.kvs_score_pairs.restype = ctypes.c_int
_lib.kvs_score_pairs.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _sz, _vp]
_lib.kvs_score_pairs_form.restype = ctypes.c_int
_lib.kvs_score_pairs_form.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _i32,
                                      _vp, _sz, _vp]
_lib.kvs_prefill_chunk.restype = ctypes.c_int
_lib.kvs_prefill_chunk.argtypes = [_P, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _i32, _i32,
                                   _i32, _i32, ctypes.POINTER(_i32), _vp, _sz, _vp]
_lib.kvs_plan_rounds.restype = ctypes.c_int
_lib.kvs_plan_rounds.argtypes = [_i32, _i32, _i32, _i32, ctypes.POINTER(_i32), _i32,
                                 ctypes.POINTER(_i32)]
_lib.kvs_merge_compact.restype = ctypes.c_int
_lib.kvs_merge_compact.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32,
                                   _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.kvs_decode_attn.restype = ctypes.c_int
_lib.kvs_decode_attn.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.kvs_decode_attn_static.restype = ctypes.c_int
_lib.kvs_decode_attn_static.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.kvs_static_scratch_bytes.restype = _sz
_lib.kvs_device_flags.restype = ctypes.c_int
_lib.kvs_stream_read.restype = ctypes.c_int
_lib.kvs_stream_read.argtypes = [_vp, ctypes.c_int64, _i32, _i32, _vp, _sz, _vp]
_lib.kvs_static_device_flags.restype = ctypes.c_int
_lib.kvs_static_device_flags.argtypes = [ctypes.POINTER(_i32), _i32, _vp]
_lib.kvs_device_flags.argtypes = [_vp, ctypes.POINTER(_i32), _i32, _vp]

if _lib.kvs_version() != 1:
    raise ImportError("libkvs.so version mismatch; rebuild it")


def library_path() -> str:
    return _LIB_PATH


def dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return F32
    if t == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported cache dtype {t}")


def make_desc(B: int, H_kv: int, H_q: int, d: int, T_cap: int, dtype) -> CacheDesc:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return CacheDesc(int(B), int(H_kv), int(H_q), int(d), int(T_cap), int(code))


def desc_of(K: torch.Tensor, H_q: int) -> CacheDesc:
    """Descriptor of a [B, H_kv, T_cap, d] cache tensor."""
    B, H_kv, T_cap, d = K.shape
    return make_desc(B, H_kv, H_q, d, T_cap, K.dtype)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise KvsError(status, where)


def workspace_size(desc: CacheDesc, W: int, op: int) -> int:
    return int(_lib.kvs_workspace_size(ctypes.byref(desc), int(W), int(op)))


def workspace(desc: CacheDesc, W: int = 32, ops=(OP_SCORE, OP_MERGE, OP_DECODE), device=None) -> torch.Tensor:
    """A zero-filled workspace large enough for every op in `ops` (uint8 tensor)."""
    n = max(workspace_size(desc, W, op) for op in ops)
    if n == 0:
        raise ValueError("invalid cache shape for the workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def score_pairs(desc, K, V, logn, lens, cand_begin, n_recent, Q_win, W, score, w_b, ws, stream=None,
                form=None):
    """kvs_score_pairs, or kvs_score_pairs_form when `form` is given."""
    if form is None:
        _check(_lib.kvs_score_pairs(ctypes.byref(desc), _ptr(K), _ptr(V), _ptr(logn), _ptr(lens),
                                    _ptr(cand_begin), int(n_recent), _ptr(Q_win), int(W),
                                    _ptr(score), _ptr(w_b), _ptr(ws), ws.numel(), _stream(stream)),
               "kvs_score_pairs")
        return
    _check(_lib.kvs_score_pairs_form(ctypes.byref(desc), _ptr(K), _ptr(V), _ptr(logn), _ptr(lens),
                                     _ptr(cand_begin), int(n_recent), _ptr(Q_win), int(W),
                                     _ptr(score), _ptr(w_b), int(form), _ptr(ws), ws.numel(),
                                     _stream(stream)),
           "kvs_score_pairs_form")


def merge_compact(desc, K, V, logn, lens, cand_begin, n_recent, score, w_b, target, scope,
                  T_cap_out, K_out, V_out, logn_out, len_out, ws, dbg_selected=None,
                  dbg_out_offset=None, dbg_kmerged=None, stream=None):
    _check(_lib.kvs_merge_compact(ctypes.byref(desc), _ptr(K), _ptr(V), _ptr(logn), _ptr(lens),
                                  _ptr(cand_begin), int(n_recent), _ptr(score), _ptr(w_b),
                                  _ptr(target), int(scope), int(T_cap_out), _ptr(K_out),
                                  _ptr(V_out), _ptr(logn_out), _ptr(len_out), _ptr(dbg_selected),
                                  _ptr(dbg_out_offset), _ptr(dbg_kmerged), _ptr(ws), ws.numel(),
                                  _stream(stream)),
           "kvs_merge_compact")


def decode_attn(desc, q, K, V, logn, lens, out, ws, k_new=None, v_new=None, stream=None):
    _check(_lib.kvs_decode_attn(ctypes.byref(desc), _ptr(q), _ptr(K), _ptr(V), _ptr(logn),
                                _ptr(lens), _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(ws),
                                ws.numel(), _stream(stream)),
           "kvs_decode_attn")


def device_flags(ws: torch.Tensor, clear: bool = False, stream=None) -> int:
    out = _i32(0)
    _check(_lib.kvs_device_flags(_ptr(ws), ctypes.byref(out), int(bool(clear)), _stream(stream)),
           "kvs_device_flags")
    return int(out.value)


def status_str(code: int) -> str:
    return _lib.kvs_status_str(int(code)).decode()


def launch_count() -> int:
    """Kernels launched through the library by this process (host-side count)."""
    return int(_lib.kvs_launch_count())


def decode_attn_static(desc, q, K, V, logn, lens, out, k_new=None, v_new=None, stream=None):
    """kvs_decode_attn on the library's built-in scratch buffer: allocates nothing."""
    _check(_lib.kvs_decode_attn_static(ctypes.byref(desc), _ptr(q), _ptr(K), _ptr(V), _ptr(logn),
                                       _ptr(lens), _ptr(k_new), _ptr(v_new), _ptr(out),
                                       _stream(stream)),
           "kvs_decode_attn_static")


def static_device_flags(clear: bool = False, stream=None) -> int:
    """kvs_static_device_flags: the flag word of the built-in scratch buffer."""
    out = _i32(0)
    _check(_lib.kvs_static_device_flags(ctypes.byref(out), int(bool(clear)), _stream(stream)),
           "kvs_static_device_flags")
    return int(out.value)


def stream_read(buf: torch.Tensor, d: int, ctas: int, ws: torch.Tensor, stream=None):
    """kvs_stream_read: stream a bf16 [rows, d] buffer with the decode's loads (timing
    helper)."""
    _check(_lib.kvs_stream_read(_ptr(buf), buf.numel() // d, int(d), int(ctas), _ptr(ws),
                                ws.numel(), _stream(stream)), "kvs_stream_read")


def static_scratch_bytes() -> int:
    return int(_lib.kvs_static_scratch_bytes())


def prefill_chunk(desc, K, V, logn, lens, L, k_chunk, v_chunk, Q_win, W, budget, sink, ws,
                  form=FORM_FULL, stream=None) -> int:
    """kvs_prefill_chunk: append a [B, H_kv, n, d] chunk at row L of every head and merge
    back to `budget`; returns the new length of every head."""
    n = 0 if k_chunk is None else int(k_chunk.shape[2])
    out = _i32(0)
    _check(_lib.kvs_prefill_chunk(ctypes.byref(desc), _ptr(K), _ptr(V), _ptr(logn), _ptr(lens),
                                  int(L), _ptr(k_chunk), _ptr(v_chunk), n, _ptr(Q_win), int(W),
                                  int(budget), int(sink), int(form), ctypes.byref(out), _ptr(ws),
                                  ws.numel(), _stream(stream)),
           "kvs_prefill_chunk")
    return int(out.value)


def plan_rounds(length: int, target: int, cand_begin: int, n_recent: int, max_lens: int = 64):
    """kvs_plan_rounds: the per-head lengths [len, ..., target] of the merge rounds."""
    buf = (_i32 * int(max_lens))()
    n = _i32(0)
    _check(_lib.kvs_plan_rounds(int(length), int(target), int(cand_begin), int(n_recent), buf,
                                int(max_lens), ctypes.byref(n)), "kvs_plan_rounds")
    return [int(buf[i]) for i in range(n.value + 1)]
