"""Local window (AI Trends article, section "기술 상세": a sliding window of
512 tokens beside the selected chunks) through the C ABI.  The window is read
chunk-aligned: the own chunk and the window/C - 1 chunks before it form one
fusion branch scored by its exact log-sum-exp, and the top-K candidates are
the chunks before the window.  Same acceptance as the other parity tests
(tests/helpers.py), against the oracle built with the same window.
"""
import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from chunk_wise_sparse_b200.inputs import custom, generate
from oracle.oracle import Oracle
from tests.helpers import to_dev
from tests.test_gpu_parity import check_summary, run_decode_check, run_prefill_case

pytestmark = pytest.mark.gpu

PREFILL = [
    # the pages' 512-token window, tensor-core selection, ragged last tile
    custom("win512-bf16-d64", B=1, Hq=4, Hkv=2, d=64, N=4160, K=16, seed=81, dtype="bf16", needles=4,
           needle_mode="random", window=512),
    custom("win128-bf16-d128-gqa4", B=1, Hq=8, Hkv=2, d=128, N=2112, K=8, seed=82, dtype="bf16", needles=2,
           needle_mode="random", window=128),
    # G = 1: 128-position tiles that span two chunks; ragged last tile
    custom("win192-bf16-g1-ragged", B=2, Hq=2, Hkv=2, d=64, N=1600, K=8, seed=91, dtype="bf16", needles=2,
           needle_mode="random", window=192),
    # G = 16 (8-position tiles), d = 128, the longest window (15 chunks before the own one)
    custom("win1024-bf16-gqa16-d128", B=1, Hq=16, Hkv=1, d=128, N=2048, K=4, seed=92, dtype="bf16",
           window=1024),
    # CUDA-core selection and prefill (G = 3) under a window
    custom("win256-bf16-gqa3", B=1, Hq=6, Hkv=2, d=64, N=1600, K=7, seed=83, dtype="bf16", window=256),
    custom("win320-fp32-d64", B=2, Hq=2, Hkv=1, d=64, N=1024, K=5, seed=84, dtype="fp32", needles=2,
           needle_mode="random", window=320),
    custom("win192-fp32-d128", B=1, Hq=4, Hkv=2, d=128, N=1024, K=3, seed=85, dtype="fp32", window=192),
    # the window covers the whole sequence: no candidates, dense causal attention
    custom("win1024-covers-all", B=1, Hq=2, Hkv=1, d=64, N=768, K=4, seed=86, dtype="bf16", window=1024),
    # a one-chunk window is the own chunk alone (tensor-core prefill)
    custom("win64-own-chunk", B=1, Hq=4, Hkv=2, d=64, N=2048, K=8, seed=87, dtype="bf16", window=64),
]


@pytest.mark.parametrize("w", PREFILL, ids=[w.name for w in PREFILL])
def test_prefill_window(w):
    run_prefill_case(w)


def test_window_no_candidates_is_dense_causal_attention():
    """Whole sequence inside the window: ids all -1 and O = causal softmax
    attention, computed here with torch on the GPU in fp32."""
    w = custom("win-dense", B=1, Hq=2, Hkv=1, d=64, N=512, K=2, seed=88, dtype="fp32", window=512)
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o, aux = hils.prefill(q, k, v, lq, w.K, return_all=True, window=w.window)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    assert torch.all(aux["ids"] == -1)
    qq, kk, vv = q.double(), k.double().expand(-1, 2, -1, -1), v.double().expand(-1, 2, -1, -1)
    s = (qq @ kk.transpose(-1, -2)) / 8.0
    s = s.masked_fill(torch.triu(torch.ones(w.N, w.N, dtype=torch.bool, device="cuda"), 1), float("-inf"))
    ref = torch.softmax(s, -1) @ vv
    assert torch.max(torch.abs(o.double() - ref)).item() <= 1e-5
    lse = torch.logsumexp(s, -1)
    assert torch.max(torch.abs(aux["lse_own"].double() - lse)).item() <= 1e-4


@pytest.mark.parametrize("dtype,d,window", [("bf16", 128, 512), ("bf16", 64, 128), ("fp32", 64, 256)])
def test_decode_window_ragged_seqlens(dtype, d, window):
    w = custom(f"decode-win{window}-{dtype}-{d}", B=4, Hq=8, Hkv=2, d=d, N=8192, K=8, seed=89, dtype=dtype,
               kind="decode", window=window)
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    check_summary(w, inp, summ, kp, bp)
    # full, ragged, inside the first window, and exactly one candidate
    seqlens = np.array([8192, 8192 - 37, 100, window + 1], np.int32)
    run_decode_check(w, inp, q, k, v, summ, seqlens, oracle, kp, bp, inp.q_f32)


def test_decode_window_agrees_with_prefill_last_row():
    """The decode step at full length equals prefill row N-1 (fp32: the two
    paths use the same arithmetic up to summation order)."""
    w = custom("win-dec-vs-prefill", B=1, Hq=4, Hkv=2, d=64, N=2048, K=6, seed=90, dtype="fp32", window=384)
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o, aux = hils.prefill(q, k, v, lq, w.K, return_all=True, window=w.window)
    seq = torch.full((1,), w.N, dtype=torch.int32, device="cuda")
    od, ids, _ = hils.decode_step(q[:, :, -1, :].contiguous(), k, v, aux["summary"], seq, w.K, window=w.window)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    assert torch.equal(ids, aux["ids"][:, :, -1, :])
    assert torch.max(torch.abs(od - o[:, :, -1, :])).item() <= 1e-5


def test_prefill_window_full_size():
    """The bench's window workload (32K, window 512) on 4096 sampled rows."""
    from chunk_wise_sparse_b200.inputs import WORKLOADS
    run_prefill_case(WORKLOADS["prefill-32k-h16-d64-w512"])


def test_decode_window_full_size():
    """The bench's window decode workload (128K x 8, GQA 4, window 512)."""
    from chunk_wise_sparse_b200.inputs import WORKLOADS
    w = WORKLOADS["decode-128k-b8-gqa4-d128-w512"]
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    check_summary(w, inp, summ, kp, bp)
    run_decode_check(w, inp, q, k, v, summ, inp.seqlens, oracle, kp, bp, inp.q_f32)
