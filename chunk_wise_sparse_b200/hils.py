"""Python binding of ``libhils.so`` (the C ABI declared in include/hils.h).

Argument marshalling only: every step of the HiLS forward pass runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhils.so")

BF16, FP32 = 0, 1
CHUNK = 64
STATUS_NAMES = {0: "HILS_OK", 1: "HILS_ERR_INVALID_ARGUMENT", 2: "HILS_ERR_UNSUPPORTED", 3: "HILS_ERR_CUDA",
                4: "HILS_ERR_WORKSPACE_TOO_SMALL", 5: "HILS_ERR_DEVICE_TIMEOUT", 6: "HILS_ERR_DEVICE_BOUNDS"}
EXPORTS = ("hils_landmark_summary", "hils_kprime_mma_bytes", "hils_select", "hils_prefill_workspace_bytes",
           "hils_attn_prefill",
           "hils_decode_workspace_bytes", "hils_attn_decode", "hils_attn_decode_fixed_scratch",
           "hils_landmark_summary_paged", "hils_attn_decode_paged", "hils_query_calibrate", "hils_attn_decode_qcal",
           "hils_attn_backward_workspace_bytes", "hils_attn_backward",
           "hils_get_status", "hils_selftest_bounded_wait", "hils_strerror", "hils_kernel_launches")
DECODE_FIXED_SCRATCH_BYTES = 16 << 20


class HilsError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} failed: {STATUS_NAMES.get(status, status)} ({strerror(status)})")
        self.status = status


class hils_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads_q", ctypes.c_int32), ("heads_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("chunk", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("seqlen", ctypes.c_int64), ("dtype", ctypes.c_int32), ("window", ctypes.c_int32)]


_lib = None


def lib():
    """Load libhils.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m chunk_wise_sparse_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        D = ctypes.POINTER(hils_dims)
        L.hils_landmark_summary.argtypes = [D, P, P, I64, I64, P, P, P, P]
        L.hils_kprime_mma_bytes.argtypes = [D]
        L.hils_kprime_mma_bytes.restype = SZ
        L.hils_select.argtypes = [D, P, P, P, P, P, I64, P, P, P]
        L.hils_prefill_workspace_bytes.argtypes = [D]
        L.hils_prefill_workspace_bytes.restype = SZ
        L.hils_attn_prefill.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_decode_workspace_bytes.argtypes = [D]
        L.hils_decode_workspace_bytes.restype = SZ
        L.hils_attn_decode.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_attn_decode_fixed_scratch.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P]
        L.hils_landmark_summary_paged.argtypes = [D, P, P, I64, P, I64, I64, P, P, P, P]
        L.hils_attn_decode_paged.argtypes = [D, P, P, P, P, I64, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_query_calibrate.argtypes = [D, P, I64, P, P, ctypes.c_int32, P, P]
        L.hils_attn_decode_qcal.argtypes = [D, P, P, P, P, P, I64, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_attn_backward_workspace_bytes.argtypes = [D]
        L.hils_attn_backward_workspace_bytes.restype = SZ
        L.hils_attn_backward.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.hils_get_status.argtypes = [ctypes.POINTER(ctypes.c_int32), P]
        L.hils_selftest_bounded_wait.argtypes = [ctypes.c_int32, P]
        L.hils_strerror.argtypes = [ctypes.c_int]
        L.hils_strerror.restype = ctypes.c_char_p
        L.hils_kernel_launches.restype = ctypes.c_uint64
        for name in EXPORTS:
            getattr(L, name).restype = getattr(L, name).restype or ctypes.c_int
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().hils_strerror(int(status)).decode()


def _ptr(t):
    """Device address of a tensor argument (a raw int is passed as is).  Every
    buffer the library reads or writes is dense device memory of the current
    GPU in the layout its header states: a host tensor, one on another GPU or
    a strided view is refused here, before any call."""
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device} but the current device is cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got strides {t.stride()} for shape {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(call, rc):
    if rc != 0:
        raise HilsError(call, rc)


def make_dims(batch, heads_q, heads_kv, head_dim, seqlen, topk, dtype, chunk=CHUNK, window=0) -> hils_dims:
    """window: local window in tokens (0 = the own chunk alone; else a multiple
    of the chunk, at most 16 chunks)."""
    if isinstance(dtype, torch.dtype):
        dtype = BF16 if dtype == torch.bfloat16 else FP32 if dtype == torch.float32 else -1
    return hils_dims(batch, heads_q, heads_kv, head_dim, chunk, topk, seqlen, dtype, window)


def dims_for(q, k, topk, window=0) -> hils_dims:
    """Dims of a prefill from q [B,Hq,N,d] and k [B,Hkv,N,d]."""
    B, Hq, N, d = q.shape
    return make_dims(B, Hq, k.shape[1], d, N, topk, q.dtype, window=window)


# ---------------------------------------------------------------------------
# The C entry points, one Python function each (same names).

def hils_landmark_summary(dims, k, lq, chunk_begin, chunk_end, kprime, bprime, kprime_mma=None, stream=None):
    _check("hils_landmark_summary",
           lib().hils_landmark_summary(ctypes.byref(dims), _ptr(k), _ptr(lq), int(chunk_begin), int(chunk_end),
                                       _ptr(kprime), _ptr(bprime), _ptr(kprime_mma), _stream(stream)))


def hils_kprime_mma_bytes(dims) -> int:
    return int(lib().hils_kprime_mma_bytes(ctypes.byref(dims)))


def hils_select(dims, q, kprime, bprime, kprime_mma, row_pos, n_rows, ids, scores=None, stream=None):
    """row_pos None (n_rows 0): every position; else a device int64 tensor of
    n_rows query positions, ids / scores [B, Hq, n_rows, K]."""
    _check("hils_select", lib().hils_select(ctypes.byref(dims), _ptr(q), _ptr(kprime), _ptr(bprime),
                                            _ptr(kprime_mma), _ptr(row_pos), int(n_rows), _ptr(ids), _ptr(scores),
                                            _stream(stream)))


def hils_prefill_workspace_bytes(dims) -> int:
    return int(lib().hils_prefill_workspace_bytes(ctypes.byref(dims)))


def hils_attn_prefill(dims, q, k, v, kprime, bprime, kprime_mma, ids, scores, o, lse_own=None, workspace=None,
                      workspace_bytes=None, stream=None):
    """scores None: the chunk scores of the kept ids are recomputed from q and
    the summaries (kprime_mma for bf16, kprime and bprime for fp32)."""
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("hils_attn_prefill", lib().hils_attn_prefill(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(kprime),
                                                        _ptr(bprime), _ptr(kprime_mma), _ptr(ids), _ptr(scores),
                                                        _ptr(o), _ptr(lse_own), _ptr(workspace),
                                                        int(workspace_bytes), _stream(stream)))


def prefill_workspace(dims, device):
    """A device workspace for hils_attn_prefill (None when none is needed)."""
    n = hils_prefill_workspace_bytes(dims)
    return torch.empty((n,), dtype=torch.uint8, device=device) if n else None


def hils_decode_workspace_bytes(dims) -> int:
    return int(lib().hils_decode_workspace_bytes(ctypes.byref(dims)))


def hils_attn_decode(dims, q, k_cache, v_cache, kprime, bprime, kprime_mma, seqlens, o, ids_out, scores_out,
                     workspace, workspace_bytes=None, stream=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check("hils_attn_decode",
           lib().hils_attn_decode(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(kprime),
                                  _ptr(bprime), _ptr(kprime_mma), _ptr(seqlens), _ptr(o), _ptr(ids_out),
                                  _ptr(scores_out), _ptr(workspace), int(workspace_bytes), _stream(stream)))


def hils_attn_decode_fixed_scratch(dims, q, k_cache, v_cache, kprime, bprime, kprime_mma, seqlens, o, ids_out,
                                   scores_out, stream=None):
    """hils_attn_decode without a workspace, for callers that cannot allocate
    device memory (a host engine that owns all device memory, or a decode loop
    that must not pay cudaMalloc's implicit synchronisation).  Scratch is the
    library's fixed 16 MiB device array; overlapping calls race on it."""
    _check("hils_attn_decode_fixed_scratch",
           lib().hils_attn_decode_fixed_scratch(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                                _ptr(kprime), _ptr(bprime), _ptr(kprime_mma), _ptr(seqlens),
                                                _ptr(o), _ptr(ids_out), _ptr(scores_out), _stream(stream)))


def hils_landmark_summary_paged(dims, k_pages, page_table, n_pages, lq, chunk_begin, chunk_end, kprime, bprime,
                                kprime_mma=None, stream=None):
    _check("hils_landmark_summary_paged",
           lib().hils_landmark_summary_paged(ctypes.byref(dims), _ptr(k_pages), _ptr(page_table), int(n_pages),
                                             _ptr(lq), int(chunk_begin), int(chunk_end), _ptr(kprime), _ptr(bprime),
                                             _ptr(kprime_mma), _stream(stream)))


def hils_attn_decode_paged(dims, q, k_pages, v_pages, page_table, n_pages, kprime, bprime, kprime_mma, seqlens, o,
                           ids_out, scores_out, workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("hils_attn_decode_paged",
           lib().hils_attn_decode_paged(ctypes.byref(dims), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table),
                                        int(n_pages), _ptr(kprime), _ptr(bprime), _ptr(kprime_mma), _ptr(seqlens),
                                        _ptr(o), _ptr(ids_out), _ptr(scores_out), _ptr(workspace), int(nbytes),
                                        _stream(stream)))


def hils_query_calibrate(dims, q, n_pos, w_down, w_up, rank, q_hat, stream=None):
    _check("hils_query_calibrate",
           lib().hils_query_calibrate(ctypes.byref(dims), _ptr(q), int(n_pos), _ptr(w_down), _ptr(w_up), int(rank),
                                      _ptr(q_hat), _stream(stream)))


def hils_attn_decode_qcal(dims, q, q_score, k_cache, v_cache, page_table, n_pages, kprime, bprime, kprime_mma,
                          seqlens, o, ids_out, scores_out, workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("hils_attn_decode_qcal",
           lib().hils_attn_decode_qcal(ctypes.byref(dims), _ptr(q), _ptr(q_score), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(page_table), int(n_pages), _ptr(kprime), _ptr(bprime), _ptr(kprime_mma),
                                       _ptr(seqlens), _ptr(o), _ptr(ids_out), _ptr(scores_out), _ptr(workspace),
                                       int(nbytes), _stream(stream)))


def hils_attn_backward_workspace_bytes(dims) -> int:
    return int(lib().hils_attn_backward_workspace_bytes(ctypes.byref(dims)))


def hils_attn_backward(dims, q, q_score, k, v, lq, kprime, ids, scores, lse_own, o, d_o, dq, dq_score, dk, dv, dlq,
                       workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else workspace_bytes
    _check("hils_attn_backward",
           lib().hils_attn_backward(ctypes.byref(dims), _ptr(q), _ptr(q_score), _ptr(k), _ptr(v), _ptr(lq),
                                    _ptr(kprime), _ptr(ids), _ptr(scores), _ptr(lse_own), _ptr(o), _ptr(d_o),
                                    _ptr(dq), _ptr(dq_score), _ptr(dk), _ptr(dv), _ptr(dlq), _ptr(workspace),
                                    int(nbytes), _stream(stream)))


def hils_get_status(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("hils_get_status", lib().hils_get_status(ctypes.byref(v), _stream(stream)))
    return int(v.value)


def hils_selftest_bounded_wait(limit_ms: int = 50, stream=None):
    _check("hils_selftest_bounded_wait", lib().hils_selftest_bounded_wait(int(limit_ms), _stream(stream)))


def hils_kernel_launches() -> int:
    return int(lib().hils_kernel_launches())


# ---------------------------------------------------------------------------
# Convenience layer: allocate outputs with torch and chain the calls.

class Summary:
    """Landmark summaries of one KV sequence set: fp32 k', b' and the bf16
    scoring operand (bf16 only)."""

    def __init__(self, dims, device):
        B, H, nc, d = dims.batch, dims.heads_kv, dims.seqlen // CHUNK, dims.head_dim
        self.kprime = torch.empty((B, H, nc, d), dtype=torch.float32, device=device)
        self.bprime = torch.empty((B, H, nc), dtype=torch.float32, device=device)
        self.kprime_mma = None
        if dims.dtype == BF16:
            n = hils_kprime_mma_bytes(dims)
            self.kprime_mma = torch.empty((n // 2,), dtype=torch.bfloat16, device=device)


def landmark_summary(k, lq, topk=1, chunk_begin=0, chunk_end=None, out: Summary | None = None, stream=None):
    B, H, N, d = k.shape
    dims = make_dims(B, H, H, d, N, topk, k.dtype)
    out = out or Summary(dims, k.device)
    chunk_end = N // CHUNK if chunk_end is None else chunk_end
    hils_landmark_summary(dims, k, lq, chunk_begin, chunk_end, out.kprime, out.bprime, out.kprime_mma, stream)
    return out


def select(q, summ: Summary, heads_kv, topk, stream=None, window=0, row_pos=None, with_scores=True):
    """ids (and scores, or None) of every position, or of the positions in
    row_pos (a device int64 tensor): [B, Hq, rows, K]."""
    B, Hq, N, d = q.shape
    dims = make_dims(B, Hq, heads_kv, d, N, topk, q.dtype, window=window)
    n_rows = N if row_pos is None else row_pos.numel()
    ids = torch.empty((B, Hq, n_rows, topk), dtype=torch.int32, device=q.device)
    scores = torch.empty((B, Hq, n_rows, topk), dtype=torch.float32, device=q.device) if with_scores else None
    hils_select(dims, q, summ.kprime, summ.bprime, summ.kprime_mma, row_pos, 0 if row_pos is None else n_rows, ids,
                scores, stream)
    return ids, scores


def prefill(q, k, v, lq, topk, stream=None, return_all=False, window=0, scores_buffer=True):
    """Full HiLS prefill: summary -> select -> sparse attention.  Returns O
    (and, with return_all, the summary, ids, scores and the local branch's
    log-sum-exp).  scores_buffer False: the selection writes no scores and
    the attention recomputes them."""
    dims = dims_for(q, k, topk, window)
    summ = landmark_summary(k, lq, topk, stream=stream)
    ids, scores = select(q, summ, k.shape[1], topk, stream, window, with_scores=scores_buffer)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    hils_attn_prefill(dims, q, k, v, summ.kprime, summ.bprime, summ.kprime_mma, ids, scores, o, lse,
                      prefill_workspace(dims, q.device), stream=stream)
    if return_all:
        return o, dict(summary=summ, ids=ids, scores=scores, lse_own=lse)
    return o


def query_calibrate(q, w_down, w_up, out=None, stream=None):
    """Q-Cal: q^ = q + W_up (W_down q) per query head, for q [B,Hq,N,d] (a
    prefill) or [B,Hq,d] (a decode step); w_down [Hq,r,d], w_up [Hq,d,r]."""
    n_pos = q.shape[2] if q.dim() == 4 else 1
    B, Hq, d = q.shape[0], q.shape[1], q.shape[-1]
    Hq_w, r, _ = w_down.shape
    dims = make_dims(B, Hq, Hq, d, CHUNK, 1, q.dtype)
    out = torch.empty_like(q) if out is None else out
    hils_query_calibrate(dims, q, n_pos, w_down, w_up, r, out, stream)
    return out


def prefill_qcal(q, k, v, lq, topk, w_down, w_up, stream=None, return_all=False, window=0):
    """HiLS prefill with Q-Cal: summary -> calibrate -> select on q^ ->
    sparse attention with q."""
    dims = dims_for(q, k, topk, window)
    summ = landmark_summary(k, lq, topk, stream=stream)
    q_hat = query_calibrate(q, w_down, w_up, stream=stream)
    ids, scores = select(q_hat, summ, k.shape[1], topk, stream, window)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    hils_attn_prefill(dims, q, k, v, summ.kprime, summ.bprime, summ.kprime_mma, ids, scores, o, lse,
                      prefill_workspace(dims, q.device), stream=stream)
    if return_all:
        return o, dict(summary=summ, ids=ids, scores=scores, lse_own=lse, q_hat=q_hat)
    return o


def decode_step_qcal(q, q_score, k_cache, v_cache, summ: Summary, seqlens, topk, workspace=None, stream=None,
                     window=0):
    """One decode step with a separate scoring query q_score [B,Hq,d]."""
    B, Hq, d = q.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    dims = make_dims(B, Hq, Hkv, d, cap, topk, q.dtype, window=window)
    if workspace is None:
        workspace = torch.empty((hils_decode_workspace_bytes(dims),), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    ids = torch.empty((B, Hq, topk), dtype=torch.int32, device=q.device)
    scores = torch.empty((B, Hq, topk), dtype=torch.float32, device=q.device)
    hils_attn_decode_qcal(dims, q, q_score, k_cache, v_cache, None, 0, summ.kprime, summ.bprime, summ.kprime_mma,
                          seqlens, o, ids, scores, workspace, stream=stream)
    return o, ids, scores


def backward(q, k, v, lq, aux, o, d_o, topk, q_score=None, window=0, stream=None):
    """Gradients (fp32) of a prefill made by prefill()/prefill_qcal() with
    return_all=True: returns dict(dq, dq_score (with q_score), dk, dv, dlq)."""
    dims = dims_for(q, k, topk, window)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    f32 = dict(dtype=torch.float32, device=q.device)
    g = dict(dq=torch.empty((B, Hq, N, d), **f32), dk=torch.empty((B, Hkv, N, d), **f32),
             dv=torch.empty((B, Hkv, N, d), **f32), dlq=torch.empty((B, Hkv, N // CHUNK, d), **f32))
    g["dq_score"] = torch.empty((B, Hq, N, d), **f32) if q_score is not None else None
    ws = torch.empty((hils_attn_backward_workspace_bytes(dims),), dtype=torch.uint8, device=q.device)
    hils_attn_backward(dims, q, q_score, k, v, lq, aux["summary"].kprime, aux["ids"], aux["scores"], aux["lse_own"], o,
                       d_o, g["dq"], g["dq_score"], g["dk"], g["dv"], g["dlq"], ws, stream=stream)
    return g


def decode_step(q, k_cache, v_cache, summ: Summary, seqlens, topk, workspace=None, stream=None, window=0):
    """One decode step for q [B,Hq,d] against caches [B,Hkv,cap,d]."""
    B, Hq, d = q.shape
    Hkv, cap = k_cache.shape[1], k_cache.shape[2]
    dims = make_dims(B, Hq, Hkv, d, cap, topk, q.dtype, window=window)
    if workspace is None:
        workspace = torch.empty((hils_decode_workspace_bytes(dims),), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    ids = torch.empty((B, Hq, topk), dtype=torch.int32, device=q.device)
    scores = torch.empty((B, Hq, topk), dtype=torch.float32, device=q.device)
    hils_attn_decode(dims, q, k_cache, v_cache, summ.kprime, summ.bprime, summ.kprime_mma, seqlens, o, ids, scores,
                     workspace, stream=stream)
    return o, ids, scores
