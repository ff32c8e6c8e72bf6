"""Seeded synthetic inputs for HiLS attention (shared by the oracle tests, the
GPU parity tests and the benchmark).

This module holds no arithmetic of the method itself: it only draws the
tensors (queries, keys, values, landmark queries), plants "needle" chunks and
rounds to bf16.  Every consumer -- the CUDA path and the fp64 oracle -- reads
the same arrays produced here.

Workload shapes follow the model sizes the HiLS paper benchmarks ("Hierarchical
Sparse Attention Done Right: Toward Infinite Context Modeling", aitrends.kr
article, sections "기술 상세" (chunk size 64, top-K) and "주요 결과" (345M / 7B
models, 512K context)).  Values are i.i.d. N(0, 1); no dataset is involved.

Recipe (fixed, deterministic):
  * float32 ``standard_normal`` draws (numpy PCG64) for Q, K, V, LQ, each in
    its row-major layout (Q [B,Hq,N,d] -- or [B,Hq,d] for a decode-only
    workload --, K and V [B,Hkv,N,d], LQ [B,Hkv,N/C,d]).  Tensor t (0 Q, 1 K,
    2 V, 3 LQ) is filled in blocks of 2^22 consecutive elements; block j is
    drawn from ``default_rng(SeedSequence([seed, t, j]))`` (so blocks can be
    drawn in parallel).  The needle picks use
    ``default_rng(SeedSequence([seed, 4]))``.
  * Needles: a needle chunk has all of its keys shifted by
    ``+1.5 * unit(mean query of a later 256-query block)``.  The direction is
    computed per (batch, kv head) from the fp32 draws of the queries of the
    G query heads that share that kv head, and the shift is applied in fp32
    before rounding.  The needle chunk index is shared by all (batch, kv head).
      - "per_block" mode: every 256-query block except the first gets one
        needle, drawn uniformly (without replacement) among the chunks that
        end at or before the block start.
      - "random" mode: ``n`` distinct needle chunks are drawn among the
        chunks that have at least one later block; each picks its block
        uniformly among the blocks that start at or after the chunk's end.
  * bf16 workloads round every tensor from fp32 with round-to-nearest-even.
  * Oracle sample rows: ``default_rng(seed + 1000).choice`` of distinct flat
    row ids over (b, hq, i), sorted.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

QUERY_BLOCK = 256
NEEDLE_SHIFT = 1.5
DRAW_BLOCK = 1 << 22


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    C: int
    K: int
    seed: int
    dtype: str          # "fp32" or "bf16"
    needles: int
    needle_mode: str    # "per_block", "random" or "none"
    kind: str           # "prefill", "decode" or "prefill+decode"
    sample_rows: int    # rows the oracle checks (0 = all rows)
    paged: bool = False  # decode: the KV cache in chunk pages (page_table)
    window: int = 0      # local window in tokens (0: the own chunk alone)
    qcal: int = 0        # Q-Cal rank (0: no query calibration)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nc(self) -> int:
        return self.N // self.C


# The workloads, named for what they are.
WORKLOADS = {
    "tiny-fp32-1k": Workload("tiny-fp32-1k", 1, 1, 1, 64, 1024, 64, 3, 0,
                             "fp32", 3, "per_block", "prefill", 0),
    "prefill-32k-h16-d64": Workload("prefill-32k-h16-d64", 1, 16, 16, 64, 32768, 64, 16, 1,
                                    "bf16", 32, "random", "prefill", 4096),
    "decode-128k-b8-gqa4-d128": Workload("decode-128k-b8-gqa4-d128", 8, 32, 8, 128, 131072, 64, 32, 2,
                                         "bf16", 0, "none", "decode", 0),
    # the same decode step with the KV cache in chunk pages drawn in random order
    "decode-128k-b8-gqa4-d128-paged": Workload("decode-128k-b8-gqa4-d128-paged", 8, 32, 8, 128, 131072, 64, 32, 2,
                                               "bf16", 0, "none", "decode", 0, paged=True),
    # the same steps with the 512-token local window beside the selected chunks
    "prefill-32k-h16-d64-w512": Workload("prefill-32k-h16-d64-w512", 1, 16, 16, 64, 32768, 64, 16, 1,
                                         "bf16", 32, "random", "prefill", 4096, window=512),
    "decode-128k-b8-gqa4-d128-w512": Workload("decode-128k-b8-gqa4-d128-w512", 8, 32, 8, 128, 131072, 64, 32, 2,
                                              "bf16", 0, "none", "decode", 0, window=512),
    "prefill-128k-gqa4-d128": Workload("prefill-128k-gqa4-d128", 1, 32, 8, 128, 131072, 64, 32, 3,
                                       "bf16", 64, "random", "prefill", 4096),
    # the 128K GQA workload's shape at 32K tokens: a profiling case for the d = 128 kernels that keeps the
    # device footprint near 1.5 GB while Q (268 MB) still exceeds L2
    "prefill-32k-gqa4-d128": Workload("prefill-32k-gqa4-d128", 1, 32, 8, 128, 32768, 64, 32, 3,
                                      "bf16", 16, "random", "prefill", 4096),
    "prefill-512k-h16-d64": Workload("prefill-512k-h16-d64", 1, 16, 16, 64, 524288, 64, 16, 4,
                                     "bf16", 128, "random", "prefill+decode", 4096),
    # the 512K workload with rank-16 Q-Cal: chunk scores from q^ = q + W_up W_down q
    "prefill-512k-h16-d64-qcal16": Workload("prefill-512k-h16-d64-qcal16", 1, 16, 16, 64, 524288, 64, 16, 4,
                                            "bf16", 128, "random", "prefill+decode", 4096, qcal=16),
    # the 512K workload's row lengths and kernels with two heads (about 0.3 GB
    # on the device): the case that profiler captures of the long-context
    # kernels run on
    "prefill-256k-h2-d64": Workload("prefill-256k-h2-d64", 1, 2, 2, 64, 262144, 64, 16, 5,
                                    "bf16", 16, "random", "prefill+decode", 4096),
}
WORKLOAD_ORDER = list(WORKLOADS)


def custom(name="custom", *, B=1, Hq=1, Hkv=1, d=64, N=1024, C=64, K=3, seed=0,
           dtype="bf16", needles=0, needle_mode="none", kind="prefill", sample_rows=0, window=0,
           qcal=0) -> Workload:
    """A workload with arbitrary sizes (used for small parity cases)."""
    if needles == 0:
        needle_mode = "none"
    return Workload(name, B, Hq, Hkv, d, N, C, K, seed, dtype, needles, needle_mode, kind, sample_rows,
                    window=window, qcal=qcal)


def round_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    lsb = u >> np.uint32(16)
    lsb &= np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u >>= np.uint32(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """Generated tensors.  ``*_f32`` hold the exact stored values as float32
    (for bf16 workloads these are the bf16 values widened, exactly);
    ``*_bits`` hold bf16 bit patterns (bf16 workloads only)."""
    w: Workload
    q_f32: np.ndarray
    k_f32: np.ndarray
    v_f32: np.ndarray
    lq_f32: np.ndarray
    needle_chunks: np.ndarray   # [n] chunk ids
    needle_blocks: np.ndarray   # [n] 256-query block ids
    q_bits: np.ndarray | None = None
    k_bits: np.ndarray | None = None
    v_bits: np.ndarray | None = None
    lq_bits: np.ndarray | None = None

    @property
    def seqlens(self) -> np.ndarray:
        return np.full((self.w.B,), self.w.N, dtype=np.int32)

    def decode_query(self) -> np.ndarray:
        """[B,Hq,d] decode query (exact values as fp32).  For a prefill+decode
        workload it is the last prefill row, so decode output == prefill row N-1."""
        if self.w.kind == "decode":
            return self.q_f32
        return np.ascontiguousarray(self.q_f32[:, :, -1, :])

    def decode_query_bits(self) -> np.ndarray | None:
        if self.q_bits is None:
            return None
        if self.w.kind == "decode":
            return self.q_bits
        return np.ascontiguousarray(self.q_bits[:, :, -1, :])


def _pick_needles(w: Workload, rng: np.random.Generator):
    nb = w.N // QUERY_BLOCK
    if w.needle_mode == "none" or w.needles == 0:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    if w.needle_mode == "per_block":
        chunks, blocks, used = [], [], set()
        for blk in range(1, nb):
            limit = blk * QUERY_BLOCK // w.C           # chunks ending at or before the block start
            free = [c for c in range(limit) if c not in used]
            c = int(free[int(rng.integers(len(free)))])
            used.add(c)
            chunks.append(c)
            blocks.append(blk)
            if len(chunks) == w.needles:
                break
        return np.array(chunks, np.int64), np.array(blocks, np.int64)
    # "random": chunks with a later block: (c+1)*C <= (nb-1)*QUERY_BLOCK
    n_elig = (nb - 1) * QUERY_BLOCK // w.C
    if w.needles > n_elig:
        raise ValueError("too many needles for the sequence length")
    chunks = np.sort(rng.choice(n_elig, size=w.needles, replace=False)).astype(np.int64)
    blocks = np.empty_like(chunks)
    for t, c in enumerate(chunks):
        first = -(-((int(c) + 1) * w.C) // QUERY_BLOCK)   # first block starting at/after chunk end
        blocks[t] = int(rng.integers(first, nb))
    return chunks, blocks


def _normal(shape, seed: int, tensor: int) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), np.float32)

    def fill(j):
        rng = np.random.default_rng(np.random.SeedSequence([seed, tensor, j]))
        rng.standard_normal(out=out[j * DRAW_BLOCK:(j + 1) * DRAW_BLOCK], dtype=np.float32)

    nblk = (out.size + DRAW_BLOCK - 1) // DRAW_BLOCK
    with ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(nblk)))
    return out.reshape(shape)


def _to_bf16(x: np.ndarray):
    """(bf16 bits, exact fp32 values) with round-to-nearest-even."""
    import torch
    t = torch.from_numpy(x).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16), t.float().numpy()


def generate(w: Workload) -> Inputs:
    if w.kind == "decode":
        q = _normal((w.B, w.Hq, w.d), w.seed, 0)
    else:
        q = _normal((w.B, w.Hq, w.N, w.d), w.seed, 0)
    k = _normal((w.B, w.Hkv, w.N, w.d), w.seed, 1)
    v = _normal((w.B, w.Hkv, w.N, w.d), w.seed, 2)
    lq = _normal((w.B, w.Hkv, w.nc, w.d), w.seed, 3)
    chunks, blocks = _pick_needles(w, np.random.default_rng(np.random.SeedSequence([w.seed, 4])))
    for c, blk in zip(chunks, blocks):
        s, e = blk * QUERY_BLOCK, (blk + 1) * QUERY_BLOCK
        for b in range(w.B):
            for h in range(w.Hkv):
                qs = q[b, h * w.G:(h + 1) * w.G, s:e, :].astype(np.float64)
                m = qs.reshape(-1, w.d).mean(axis=0)
                u = (m / np.linalg.norm(m)).astype(np.float32)
                k[b, h, c * w.C:(c + 1) * w.C, :] += np.float32(NEEDLE_SHIFT) * u
    inp = Inputs(w, q, k, v, lq, chunks, blocks)
    if w.dtype == "bf16":
        for name in ("q", "k", "v", "lq"):
            bits, vals = _to_bf16(getattr(inp, name + "_f32"))
            setattr(inp, name + "_bits", bits)
            setattr(inp, name + "_f32", vals)
    elif w.dtype != "fp32":
        raise ValueError(w.dtype)
    return inp


def page_table(w: Workload, spare: int = 0) -> tuple[np.ndarray, int]:
    """A chunk page table [B, nc] int32 for a pool of B * nc + spare pages:
    every logical chunk of every sequence gets a distinct page, in an order
    drawn from the workload's seed.  Returns (table, n_pages)."""
    n_pages = w.B * w.nc + spare
    rng = np.random.default_rng(np.random.SeedSequence([w.seed, 5]))
    table = rng.permutation(n_pages)[: w.B * w.nc].astype(np.int32).reshape(w.B, w.nc)
    return table, n_pages


def sample_rows(w: Workload, n: int | None = None) -> np.ndarray:
    """Sorted distinct flat row ids over (b, hq, i) that the oracle checks."""
    total = w.B * w.Hq * w.N
    n = w.sample_rows if n is None else n
    if n == 0 or n >= total:
        return np.arange(total, dtype=np.int64)
    rng = np.random.default_rng(w.seed + 1000)
    return np.sort(rng.choice(total, size=n, replace=False)).astype(np.int64)


@dataclasses.dataclass
class QcalWeights:
    """Random-init Q-Cal projections (no trained adapter exists here):
    w_down [Hq, r, d] ~ N(0, 1/d), w_up [Hq, d, r] ~ N(0, 0.25/r), so that
    W_down q has unit scale and the correction W_up W_down q about half the
    scale of q.  ``*_f32`` hold the exact stored values; ``*_bits`` the bf16
    patterns (bf16 only)."""
    rank: int
    w_down_f32: np.ndarray
    w_up_f32: np.ndarray
    w_down_bits: np.ndarray | None = None
    w_up_bits: np.ndarray | None = None


def qcal_weights(Hq: int, d: int, rank: int, seed: int, dtype: str = "bf16") -> QcalWeights:
    rng = np.random.default_rng(np.random.SeedSequence([seed, 17, rank]))
    wd = (rng.standard_normal((Hq, rank, d), dtype=np.float32) / np.float32(np.sqrt(d))).astype(np.float32)
    wu = (rng.standard_normal((Hq, d, rank), dtype=np.float32) * np.float32(0.5 / np.sqrt(rank))).astype(np.float32)
    if dtype == "bf16":
        bd, bu = round_bf16_bits(wd), round_bf16_bits(wu)
        return QcalWeights(rank, bf16_bits_to_f32(bd), bf16_bits_to_f32(bu), bd, bu)
    return QcalWeights(rank, wd, wu)
