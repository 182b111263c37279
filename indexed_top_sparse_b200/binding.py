"""ctypes binding of liblisa.so: the C entry points under the same names.

Argument marshalling only -- every step of the decode path runs in the
library's CUDA kernels.  Tensors are torch CUDA tensors used as device memory;
streams default to torch's current stream.  There is no fallback: if the
library is missing, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblisa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python indexed_top_sparse_b200/build.py` "
        "(the library has no CPU fallback)"
    )
_lib = ctypes.CDLL(LIB_PATH)

LISA_OK = 0
STATUS_NAMES = {
    0: "LISA_OK",
    1: "LISA_ERR_INVALID_ARG",
    2: "LISA_ERR_UNSUPPORTED",
    3: "LISA_ERR_WORKSPACE",
    4: "LISA_ERR_CUDA",
    5: "LISA_ERR_DEVICE_CHECK",
    6: "LISA_ERR_TIMEOUT",
}
KPROJ_FP32 = 0
KPROJ_FP8_E4M3 = 1
DEVERR_SEQ_LEN, DEVERR_PAGE_ID, DEVERR_INDEX, DEVERR_COUNT = 0x1, 0x2, 0x4, 0x8


class LisaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({lisa_status_string(status)})")


class DecodeDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("idx_dim", ctypes.c_int32),
        ("budget_m", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("seq_lens", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("softmax_scale", ctypes.c_float),
        ("kv_row_stride", ctypes.c_int32),
    ]


class LinearBranch(ctypes.Structure):
    _fields_ = [
        ("S", ctypes.c_void_p),
        ("z", ctypes.c_void_p),
        ("k_new", ctypes.c_void_p),
        ("v_new", ctypes.c_void_p),
        ("gate_logit", ctypes.c_void_p),
    ]


class StageEvents(ctypes.Structure):
    _fields_ = [
        ("start", ctypes.c_void_p),
        ("after_sample", ctypes.c_void_p),
        ("after_stream", ctypes.c_void_p),
        ("after_index", ctypes.c_void_p),
        ("after_attn", ctypes.c_void_p),
        ("end", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_S = ctypes.c_size_t
_I = ctypes.c_int32
_sig = {
    "lisa_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(DecodeDesc)]),
    "lisa_num_splits": (ctypes.c_int32, [ctypes.POINTER(DecodeDesc)]),
    "lisa_workspace_init": (_I, [_P, _S, _P]),
    "lisa_index_score": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _I, _P, _P, _P, _S, _P]),
    "lisa_topm_select": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _P, _S, _P]),
    "lisa_index_topm": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _I, _P, _P, _P, _P, _S, _P]),
    "lisa_sparse_decode_attn": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _P, _P, _P, _P, _P, _S, _P]),
    "lisa_sparse_decode_attn_noalloc": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _P, _P, _P, _P, _P]),
    "lisa_fused_decode": (
        _I,
        [ctypes.POINTER(DecodeDesc), _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P,
         ctypes.POINTER(LinearBranch), _P, _P, _P, _S, ctypes.POINTER(StageEvents), _P],
    ),
    "lisa_append_token": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _S, _P]),
    "lisa_dense_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(DecodeDesc)]),
    "lisa_calibrate_workspace_size": (ctypes.c_size_t, [_I, _I]),
    "lisa_index_score_multi": (_I, [ctypes.POINTER(DecodeDesc), _I, _P, _P, _P, _I, _P, _P, _P, _S, _P]),
    "lisa_workspace_size_multi": (ctypes.c_size_t, [ctypes.POINTER(DecodeDesc), _I]),
    "lisa_index_topm_multi": (_I, [ctypes.POINTER(DecodeDesc), _I, _P, _P, _P, _I, _P, _P, _P, _P, _S, _P]),
    "lisa_calibrate_basis": (_I, [_I, _I, _I, _P, _I, _P, _I, _P, _P, _P, _S, _P]),
    "lisa_dense_decode_attn": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _P, _P, _P, _S, _P]),
    "lisa_gather_kv": (_I, [ctypes.POINTER(DecodeDesc), _P, _P, _P, _P, _P, _P, _S, _P]),
    "lisa_check_device_error": (_I, [_P, ctypes.POINTER(ctypes.c_uint32), _P]),
    "lisa_status_string": (ctypes.c_char_p, [_I]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_sig)


class DevicePtr(int):
    """A raw device address (e.g. the V half of an interleaved K|V pool), passed through as is."""


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if isinstance(t, DevicePtr):
        return ctypes.c_void_p(int(t))
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"expected a torch.Tensor, got {type(t)}")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> Optional[ctypes.c_void_p]:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, where: str):
    if status != LISA_OK:
        raise LisaError(status, where)


def lisa_status_string(status: int) -> str:
    return _lib.lisa_status_string(status).decode()


def make_desc(*, batch, num_q_heads, num_kv_heads, head_dim, idx_dim, budget_m, page_size, max_pages_per_seq,
              max_seq_len, num_pages, seq_lens=None, page_table=None, softmax_scale=0.0,
              kv_row_stride=0) -> DecodeDesc:
    """Fill a lisa_decode_desc.  The desc refers to (does not own) seq_lens/page_table."""
    d = DecodeDesc(
        batch, num_q_heads, num_kv_heads, head_dim, idx_dim, budget_m, page_size, max_pages_per_seq, max_seq_len,
        num_pages, None, None, float(softmax_scale), int(kv_row_stride),
    )
    if seq_lens is not None:
        d.seq_lens = _ptr(seq_lens).value
        d._seq_lens_ref = seq_lens
    if page_table is not None:
        d.page_table = _ptr(page_table).value
        d._page_table_ref = page_table
    return d


def lisa_workspace_size(desc: DecodeDesc) -> int:
    return int(_lib.lisa_workspace_size(ctypes.byref(desc)))


def lisa_num_splits(desc: DecodeDesc) -> int:
    return int(_lib.lisa_num_splits(ctypes.byref(desc)))


def alloc_workspace(desc: DecodeDesc, device, stream=None) -> torch.Tensor:
    """Allocate (with torch) and initialise a workspace for desc."""
    n = lisa_workspace_size(desc)
    if n == 0:
        raise LisaError(1, "lisa_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    lisa_workspace_init(ws, stream)
    return ws


def lisa_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(_lib.lisa_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "lisa_workspace_init")


def lisa_index_score(desc, q, P, kproj_pool, kproj_dtype, kproj_scale, scores, ws, stream=None) -> None:
    _check(
        _lib.lisa_index_score(ctypes.byref(desc), _ptr(q), _ptr(P), _ptr(kproj_pool), kproj_dtype, _ptr(kproj_scale),
                              _ptr(scores), _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_index_score",
    )


def lisa_topm_select(desc, scores, idx, count, ws, stream=None) -> None:
    _check(
        _lib.lisa_topm_select(ctypes.byref(desc), _ptr(scores), _ptr(idx), _ptr(count), _ptr(ws), ws.numel(),
                              _stream(stream)),
        "lisa_topm_select",
    )


def lisa_index_topm(desc, q, P, kproj_pool, kproj_dtype, kproj_scale, idx, count, ws, stream=None) -> None:
    _check(
        _lib.lisa_index_topm(ctypes.byref(desc), _ptr(q), _ptr(P), _ptr(kproj_pool), kproj_dtype, _ptr(kproj_scale),
                             _ptr(idx), _ptr(count), _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_index_topm",
    )


def lisa_sparse_decode_attn(desc, q, k_pool, v_pool, idx, count, out, lse, ws, stream=None) -> None:
    _check(
        _lib.lisa_sparse_decode_attn(ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(idx),
                                     _ptr(count), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_sparse_decode_attn",
    )


def lisa_sparse_decode_attn_noalloc(desc, q, k_pool, v_pool, idx, count, out, lse, stream=None) -> None:
    """Attention over a given index set without a workspace (for callers that cannot allocate).

    The library keeps the scratch in a fixed device array shared by all calls: calls must not overlap
    on the GPU, and the first call on a device must come before any stream capture.
    """
    _check(
        _lib.lisa_sparse_decode_attn_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(idx),
                                             _ptr(count), _ptr(out), _ptr(lse), _stream(stream)),
        "lisa_sparse_decode_attn_noalloc",
    )


def linear_branch(S, z, k_new, v_new, gate_logit) -> LinearBranch:
    lb = LinearBranch(_ptr(S).value, _ptr(z).value, _ptr(k_new).value, _ptr(v_new).value, _ptr(gate_logit).value)
    lb._refs = (S, z, k_new, v_new, gate_logit)
    return lb


def stage_events(start=None, after_index=None, after_attn=None, end=None, stream=None, after_sample=None,
                 after_stream=None) -> StageEvents:
    """Stage events for lisa_fused_decode from torch.cuda.Event objects.

    torch creates the underlying CUDA event lazily, on its first record; each event is
    recorded once here so that it exists (the library re-records it at its stage).
    """

    def h(e):
        if e is None:
            return None
        if e.cuda_event == 0:
            e.record(stream if stream is not None else torch.cuda.current_stream())
        return e.cuda_event

    ev = StageEvents(h(start), h(after_sample), h(after_stream), h(after_index), h(after_attn), h(end))
    ev._refs = (start, after_sample, after_stream, after_index, after_attn, end)
    return ev


def lisa_fused_decode(desc, q, P, kproj_pool, kproj_dtype, kproj_scale, k_pool, v_pool, reuse_idx, reuse_count,
                      idx_out, count_out, lin: Optional[LinearBranch], out, lse, ws,
                      events: Optional[StageEvents] = None, stream=None) -> None:
    _check(
        _lib.lisa_fused_decode(
            ctypes.byref(desc), _ptr(q), _ptr(P), _ptr(kproj_pool), kproj_dtype, _ptr(kproj_scale), _ptr(k_pool),
            _ptr(v_pool), _ptr(reuse_idx), _ptr(reuse_count), _ptr(idx_out), _ptr(count_out),
            None if lin is None else ctypes.byref(lin), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
            None if events is None else ctypes.byref(events), _stream(stream),
        ),
        "lisa_fused_decode",
    )


def lisa_append_token(desc, positions, k_new, v_new, P, kproj_pool, kproj_dtype, kproj_scale, k_pool, v_pool, ws,
                      stream=None) -> None:
    _check(
        _lib.lisa_append_token(
            ctypes.byref(desc), _ptr(positions), _ptr(k_new), _ptr(v_new), _ptr(P), _ptr(kproj_pool), kproj_dtype,
            _ptr(kproj_scale), _ptr(k_pool), _ptr(v_pool), _ptr(ws), ws.numel(), _stream(stream),
        ),
        "lisa_append_token",
    )


def lisa_index_score_multi(desc, num_tokens, q, P, kproj_pool, kproj_dtype, kproj_scale, scores, ws,
                           stream=None) -> None:
    _check(
        _lib.lisa_index_score_multi(ctypes.byref(desc), num_tokens, _ptr(q), _ptr(P), _ptr(kproj_pool), kproj_dtype,
                                    _ptr(kproj_scale), _ptr(scores), _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_index_score_multi",
    )


def lisa_workspace_size_multi(desc, num_tokens: int) -> int:
    return int(_lib.lisa_workspace_size_multi(ctypes.byref(desc), num_tokens))


def alloc_workspace_multi(desc: DecodeDesc, num_tokens: int, device, stream=None) -> torch.Tensor:
    """Allocate (with torch) and initialise a workspace for lisa_index_topm_multi."""
    n = lisa_workspace_size_multi(desc, num_tokens)
    if n == 0:
        raise LisaError(1, "lisa_workspace_size_multi")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    lisa_workspace_init(ws, stream)
    return ws


def lisa_index_topm_multi(desc, num_tokens, q, P, kproj_pool, kproj_dtype, kproj_scale, idx, count, ws,
                          stream=None) -> None:
    _check(
        _lib.lisa_index_topm_multi(ctypes.byref(desc), num_tokens, _ptr(q), _ptr(P), _ptr(kproj_pool), kproj_dtype,
                                   _ptr(kproj_scale), _ptr(idx), _ptr(count), _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_index_topm_multi",
    )


def lisa_calibrate_workspace_size(num_kv_heads: int, head_dim: int) -> int:
    return int(_lib.lisa_calibrate_workspace_size(num_kv_heads, head_dim))


def lisa_calibrate_basis(q_samples, k_samples, P_out, eigvals_out=None, ws=None, stream=None) -> None:
    """q_samples [Hkv][nq][d], k_samples [Hkv][nk][d] bf16; P_out [Hkv][r][d] fp32; eigvals [Hkv][r]."""
    Hkv, nq, d = q_samples.shape
    nk = k_samples.shape[1]
    r = P_out.shape[1]
    if ws is None:
        ws = torch.zeros(lisa_calibrate_workspace_size(Hkv, d), dtype=torch.uint8, device=q_samples.device)
    _check(
        _lib.lisa_calibrate_basis(Hkv, d, r, _ptr(q_samples), nq, _ptr(k_samples), nk, _ptr(P_out), _ptr(eigvals_out),
                                  _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_calibrate_basis",
    )


def lisa_dense_workspace_size(desc: DecodeDesc) -> int:
    return int(_lib.lisa_dense_workspace_size(ctypes.byref(desc)))


def alloc_dense_workspace(desc: DecodeDesc, device, stream=None) -> torch.Tensor:
    """Allocate (with torch) and initialise a workspace for lisa_dense_decode_attn."""
    n = lisa_dense_workspace_size(desc)
    if n == 0:
        raise LisaError(1, "lisa_dense_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    lisa_workspace_init(ws, stream)
    return ws


def lisa_dense_decode_attn(desc, q, k_pool, v_pool, out, lse, ws, stream=None) -> None:
    _check(
        _lib.lisa_dense_decode_attn(ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(out), _ptr(lse),
                                    _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_dense_decode_attn",
    )


def lisa_gather_kv(desc, idx, count, k_pool, v_pool, gathered, ws, stream=None) -> None:
    _check(
        _lib.lisa_gather_kv(ctypes.byref(desc), _ptr(idx), _ptr(count), _ptr(k_pool), _ptr(v_pool), _ptr(gathered),
                            _ptr(ws), ws.numel(), _stream(stream)),
        "lisa_gather_kv",
    )


def lisa_check_device_error(ws: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the workspace error word; returns the bits (0 = clean)."""
    flags = ctypes.c_uint32(0)
    st = _lib.lisa_check_device_error(_ptr(ws), ctypes.byref(flags), _stream(stream))
    if st not in (LISA_OK, 5):
        raise LisaError(st, "lisa_check_device_error")
    return int(flags.value)
