"""ctypes front end of the fp64 HiLS oracle (``hils_oracle.c``).

TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The product path (the CUDA library
and its binding) never imports it.

The C source is compiled on first use (or by ``build()``) with
``gcc -O3 -fopenmp -ffp-contract=off`` -- no fast-math, no FMA contraction --
into ``oracle/_build/``.  A hash of the source and of the compiler flags
names the library, so a stale build is never loaded.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hils_oracle.c")
_FLAGS = ["-O3", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11"]
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("B", "Hq", "Hkv", "N", "d", "C", "K", "W")]


def _lib_path() -> str:
    with open(_SRC, "rb") as f:
        h = hashlib.sha1(f.read() + " ".join(_FLAGS).encode()).hexdigest()[:12]
    return os.path.join(_HERE, "_build", f"libhils_oracle_{h}.so")


def build() -> str:
    path = _lib_path()
    if not os.path.exists(path):
        os.makedirs(os.path.dirname(path), exist_ok=True)
        tmp = path + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_FLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, path)
    return path


def _load():
    global _lib
    if _lib is None:
        # HILS_ORACLE_LIB lets the mutation tests load a deliberately broken
        # copy of the oracle and check that the pins reject it.
        lib = ctypes.CDLL(os.environ.get("HILS_ORACLE_LIB") or build())
        P = ctypes.c_void_p
        lib.hils_oracle_summary.argtypes = [P, P, P, ctypes.c_int64, ctypes.c_int64, P, P]
        lib.hils_oracle_scores.argtypes = [P, P, P, ctypes.c_int64, P, P, P, P, P]
        lib.hils_oracle_select.argtypes = [P, P, P, ctypes.c_int64, P, P, P, P, P, P, P]
        lib.hils_oracle_attend.argtypes = [P, P, P, P, P, ctypes.c_int64, P, P, P, P, P, P,
                                           ctypes.c_int64, ctypes.c_int, P, P]
        lib.hils_oracle_qcal.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P, P, P, P, P]
        lib.hils_oracle_backward.argtypes = [P, P, P, P, P, P, P, ctypes.c_int64, P, P, P, P, P, P]
        lib.hils_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().hils_oracle_max_threads())


def _dims(B, Hq, Hkv, N, d, C, K, W=0):
    return _Dims(B, Hq, Hkv, N, d, C, K, W)


def _p(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


class Rows:
    """Explicit query rows: batch, query head, position and query vector."""

    def __init__(self, b, hq, pos, q):
        self.b = np.ascontiguousarray(b, dtype=np.int32)
        self.hq = np.ascontiguousarray(hq, dtype=np.int32)
        self.pos = np.ascontiguousarray(pos, dtype=np.int64)
        self.q = _f32(q)
        assert self.q.ndim == 2 and self.q.shape[0] == len(self.b)

    def __len__(self):
        return len(self.b)

    @staticmethod
    def from_prefill(Q: np.ndarray, flat_rows: np.ndarray) -> "Rows":
        """Rows of a prefill: Q is [B,Hq,N,d], flat ids enumerate (b, hq, i)."""
        B, Hq, N, d = Q.shape
        flat = np.asarray(flat_rows, dtype=np.int64)
        b, rem = np.divmod(flat, Hq * N)
        hq, i = np.divmod(rem, N)
        return Rows(b, hq, i, Q[b, hq, i, :])

    @staticmethod
    def from_decode(q: np.ndarray, seqlens: np.ndarray) -> "Rows":
        """Decode rows: q is [B,Hq,d]; each query sits at position seqlen-1."""
        B, Hq, d = q.shape
        b = np.repeat(np.arange(B), Hq)
        hq = np.tile(np.arange(Hq), B)
        pos = np.asarray(seqlens, dtype=np.int64)[b] - 1
        return Rows(b, hq, pos, q.reshape(B * Hq, d))


class Oracle:
    """fp64 oracle bound to one set of sizes (K/V arrays have N token slots)."""

    def __init__(self, B, Hq, Hkv, N, d, C, K, W=0):
        """W: local window in tokens, a multiple of C (0 or C: the own chunk alone)."""
        assert Hq % Hkv == 0 and N % C == 0 and W % C == 0
        self.B, self.Hq, self.Hkv, self.N, self.d, self.C, self.K, self.W = B, Hq, Hkv, N, d, C, K, W
        self.nc = N // C
        self._d = _dims(B, Hq, Hkv, N, d, C, K, W)
        self._lib = _load()

    @staticmethod
    def for_workload(w, K=None) -> "Oracle":
        return Oracle(w.B, w.Hq, w.Hkv, w.N, w.d, w.C, w.K if K is None else K, w.window)

    def summary(self, Kt, LQ, chunk_begin=0, chunk_end=None):
        """Compressed keys kp [B,Hkv,nc,d] and entropy biases bp [B,Hkv,nc]."""
        Kt, LQ = _f32(Kt), _f32(LQ)
        assert Kt.shape == (self.B, self.Hkv, self.N, self.d)
        assert LQ.shape == (self.B, self.Hkv, self.nc, self.d)
        chunk_end = self.nc if chunk_end is None else chunk_end
        kp = np.zeros((self.B, self.Hkv, self.nc, self.d), np.float64)
        bp = np.zeros((self.B, self.Hkv, self.nc), np.float64)
        self._lib.hils_oracle_summary(ctypes.byref(self._d), _p(Kt), _p(LQ), chunk_begin, chunk_end,
                                      _p(kp), _p(bp))
        return kp, bp

    def _kb(self, kp, bp):
        kp = np.ascontiguousarray(kp, dtype=np.float64)
        bp = np.ascontiguousarray(bp, dtype=np.float64)
        assert kp.shape == (self.B, self.Hkv, self.nc, self.d) and bp.shape == (self.B, self.Hkv, self.nc)
        return kp, bp

    def scores(self, kp, bp, rows: Rows):
        """All candidate scores [n_rows, nc] (-inf where c >= floor(pos/C))."""
        kp, bp = self._kb(kp, bp)
        out = np.empty((len(rows), self.nc), np.float64)
        self._lib.hils_oracle_scores(ctypes.byref(self._d), _p(kp), _p(bp), len(rows), _p(rows.b),
                                     _p(rows.hq), _p(rows.pos), _p(rows.q), _p(out))
        return out

    def select(self, kp, bp, rows: Rows):
        """(ids [n,K] ascending, -1 padded; their scores; gap K-th vs (K+1)-th)."""
        kp, bp = self._kb(kp, bp)
        n = len(rows)
        ids = np.empty((n, self.K), np.int32)
        sel = np.empty((n, self.K), np.float64)
        gap = np.empty((n,), np.float64)
        self._lib.hils_oracle_select(ctypes.byref(self._d), _p(kp), _p(bp), n, _p(rows.b), _p(rows.hq),
                                     _p(rows.pos), _p(rows.q), _p(ids), _p(sel), _p(gap))
        return ids, sel, gap

    def attend(self, Kt, Vt, kp, bp, rows: Rows, ids, score_mode=0, qscore=None):
        """Fused output O [n,d] and local-branch log-sum-exp [n] for given ids.
        qscore [n,d] (optional): the scoring query of each row (Q-Cal), used
        for the chunk scores in the fusion; rows.q attends."""
        Kt, Vt = _f32(Kt), _f32(Vt)
        assert Kt.shape == (self.B, self.Hkv, self.N, self.d) and Vt.shape == Kt.shape
        kp, bp = self._kb(kp, bp)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        n = len(rows)
        assert ids.shape[0] == n
        O = np.empty((n, self.d), np.float64)
        lse = np.empty((n,), np.float64)
        if qscore is not None:
            qscore = _f32(qscore)
            assert qscore.shape == rows.q.shape
        self._lib.hils_oracle_attend(ctypes.byref(self._d), _p(Kt), _p(Vt), _p(kp), _p(bp), n,
                                     _p(rows.b), _p(rows.hq), _p(rows.pos), _p(rows.q), _p(qscore), _p(ids),
                                     ids.shape[1], int(score_mode), _p(O), _p(lse))
        return O, lse

    def backward(self, Q, Kt, Vt, LQ, ids, dO, Qs=None):
        """Gradients of <dO, O> for a fixed selection ids [B,Hq,N,Kids]: dQ
        (attention query, plus the scoring-query part unless Qs is given),
        dQs (the scoring query's, when Qs is given), dK, dV, dLQ (double)."""
        Q, Kt, Vt, LQ, dO = _f32(Q), _f32(Kt), _f32(Vt), _f32(LQ), _f32(dO)
        B, Hq, Hkv, N, d, nc = self.B, self.Hq, self.Hkv, self.N, self.d, self.nc
        assert Q.shape == (B, Hq, N, d) and dO.shape == Q.shape
        assert Kt.shape == (B, Hkv, N, d) and Vt.shape == Kt.shape and LQ.shape == (B, Hkv, nc, d)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        assert ids.shape[:3] == (B, Hq, N)
        if Qs is not None:
            Qs = _f32(Qs)
            assert Qs.shape == Q.shape
        dQ = np.empty((B, Hq, N, d))
        dQs = np.empty((B, Hq, N, d)) if Qs is not None else None
        dK, dV = np.empty((B, Hkv, N, d)), np.empty((B, Hkv, N, d))
        dLQ = np.empty((B, Hkv, nc, d))
        self._lib.hils_oracle_backward(ctypes.byref(self._d), _p(Q), _p(Qs), _p(Kt), _p(Vt), _p(LQ), _p(ids),
                                       ids.shape[3], _p(dO), _p(dQ), _p(dQs), _p(dK), _p(dV), _p(dLQ))
        return dict(dQ=dQ, dQs=dQs, dK=dK, dV=dV, dLQ=dLQ)

    def prefill_rows(self, Q, Kt, Vt, kp, bp, flat_rows):
        """Select + attend for the given flat rows of a prefill."""
        rows = Rows.from_prefill(_f32(Q), flat_rows)
        ids, sel, gap = self.select(kp, bp, rows)
        O, lse = self.attend(Kt, Vt, kp, bp, rows, ids)
        return dict(ids=ids, sel=sel, gap=gap, O=O, lse_own=lse, rows=rows)

    def decode(self, q, Kc, Vc, kp, bp, seqlens):
        """One decode step: each (b, hq) query at position seqlen-1."""
        rows = Rows.from_decode(_f32(q), seqlens)
        ids, sel, gap = self.select(kp, bp, rows)
        O, lse = self.attend(Kc, Vc, kp, bp, rows, ids)
        B, Hq, d = q.shape
        return dict(ids=ids.reshape(B, Hq, -1), sel=sel.reshape(B, Hq, -1), gap=gap.reshape(B, Hq),
                    O=O.reshape(B, Hq, d), lse_own=lse.reshape(B, Hq), rows=rows)


def qcal(q: np.ndarray, hq: np.ndarray, w_down: np.ndarray, w_up: np.ndarray) -> np.ndarray:
    """Q-Cal (aitrends.kr article, section "방법론" and glossary entry
    "저계수 쿼리 보정"): q^ = q + W_up (W_down q) per row with the projections
    of the row's query head.  q [n,d], hq [n], w_down [Hq,r,d], w_up [Hq,d,r];
    returns q^ [n,d] in double."""
    q, w_down, w_up = _f32(q), _f32(w_down), _f32(w_up)
    hq = np.ascontiguousarray(hq, dtype=np.int32)
    n, d = q.shape
    Hq, r, d2 = w_down.shape
    assert d2 == d and w_up.shape == (Hq, d, r) and len(hq) == n and r <= 256
    assert n == 0 or (hq.min() >= 0 and hq.max() < Hq)
    out = np.empty((n, d), np.float64)
    _load().hils_oracle_qcal(n, d, r, _p(hq), _p(q), _p(w_down), _p(w_up), _p(out))
    return out


def gather_pages(pages: np.ndarray, table: np.ndarray) -> np.ndarray:
    """The contiguous cache [B, Hkv, nc*C, d] that a chunk-paged pool
    [n_pages, Hkv, C, d] and a page table [B, nc] describe: logical chunk c of
    sequence b is page table[b, c] (aitrends.kr article, section "기술 상세":
    chunk-unit KV paging).  Every paged call is defined as the contiguous call
    on this cache."""
    B, nc = table.shape
    n_pages, H, C, d = pages.shape
    out = np.empty((B, H, nc * C, d), dtype=pages.dtype)
    for b in range(B):
        for c in range(nc):
            out[b, :, c * C:(c + 1) * C, :] = pages[int(table[b, c])]
    return out
