"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Acceptance (tests/helpers.py): k', b' within 1e-5; selected chunk-id sets
identical wherever the oracle's K-th/(K+1)-th score gap is at least 1e-3
(fp32) or 2e-2 (bf16), and valid (no dropped chunk beats a kept one by more
than that gap) on every row; outputs within max-abs 1e-5 (fp32) or max-abs
2e-2 and mean-abs 2e-3 (bf16), compared with the oracle run on the GPU's
own ids so that a selection flip cannot hide an attention error.
"""
import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from chunk_wise_sparse_b200.inputs import WORKLOADS, custom, generate, sample_rows
from oracle.oracle import Oracle, Rows
from tests.helpers import OUT_MAX, OUT_MEAN, SEL_GAP, SUMMARY_TOL, check_selection, gather_rows, to_dev

pytestmark = pytest.mark.gpu

SCORE_TOL = {"fp32": 1e-5, "bf16": 1e-2}


def bf16_to_f32(t):
    return t.float().cpu().numpy()


def check_summary(w, inp, summ, kp, bp):
    kp_g, bp_g = summ.kprime.cpu().numpy(), summ.bprime.cpu().numpy()
    assert np.max(np.abs(kp_g - kp)) <= SUMMARY_TOL
    assert np.max(np.abs(bp_g - bp)) <= SUMMARY_TOL
    if w.dtype == "bf16":
        mma = summ.kprime_mma.view(w.B, w.Hkv, w.nc, w.d + 16)
        assert torch.equal(mma[..., :w.d], summ.kprime.to(torch.bfloat16))
        x = mma[..., w.d].float() + mma[..., w.d + 1].float()
        assert torch.max(torch.abs(x / w.d ** 0.5 - summ.bprime)).item() < 1e-4
        assert not mma[..., w.d + 2:].float().abs().max().item()


def check_rows(w, inp, oracle, kp, bp, flat, ids_t, scores_t, o_t, lse_t=None, rows=None):
    """Selection, score and output parity on the given rows."""
    rows = rows or Rows.from_prefill(inp.q_f32, flat)
    ids_o, _, gap = oracle.select(kp, bp, rows)
    S = oracle.scores(kp, bp, rows)
    ids_g = np.ascontiguousarray(ids_t).astype(np.int32)
    graded, n, valid = check_selection(ids_g, ids_o, gap, S, SEL_GAP[w.dtype], SEL_GAP[w.dtype])
    kept = ids_g >= 0
    rr = np.nonzero(kept)
    serr = np.abs(scores_t[kept] - S[rr[0], ids_g[kept]]) if kept.any() else np.zeros(1)
    assert serr.max() <= SCORE_TOL[w.dtype], serr.max()
    assert np.all(np.isneginf(scores_t[~kept]))
    O_o, lse_o = oracle.attend(inp.k_f32 if w.kind != "decode" else inp.k_f32, inp.v_f32, kp, bp, rows, ids_g)
    err = np.abs(o_t - O_o)
    assert err.max() <= OUT_MAX[w.dtype], err.max()
    assert err.mean() <= OUT_MEAN[w.dtype], err.mean()
    if lse_t is not None:
        assert np.max(np.abs(lse_t - lse_o)) <= 1e-4
    print(f"[{w.name}] rows {n}: graded {graded} ({graded / n:.1%}), valid {valid}; "
          f"score err max {serr.max():.2e}; O err max {err.max():.2e} mean {err.mean():.2e}")
    return graded


def run_prefill_case(w):
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o, aux = hils.prefill(q, k, v, lq, w.K, return_all=True, window=w.window)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    check_summary(w, inp, aux["summary"], kp, bp)
    flat = sample_rows(w)
    check_rows(w, inp, oracle, kp, bp, flat, gather_rows(aux["ids"], flat), gather_rows(aux["scores"], flat),
               gather_rows(o, flat), gather_rows(aux["lse_own"][..., None], flat)[:, 0])
    return inp, (q, k, v, lq), o, aux, (oracle, kp, bp)


SMALL = [
    WORKLOADS["tiny-fp32-1k"],
    custom("bf16-d64-ragged", B=2, Hq=2, Hkv=2, d=64, N=4288, K=16, seed=31, dtype="bf16", needles=4,
           needle_mode="random"),
    custom("bf16-d128-gqa4", B=1, Hq=8, Hkv=2, d=128, N=2112, K=32, seed=32, dtype="bf16", needles=2,
           needle_mode="random"),
    custom("fp32-d128-gqa2", B=1, Hq=4, Hkv=2, d=128, N=1024, K=5, seed=33, dtype="fp32", needles=2,
           needle_mode="random"),
    custom("bf16-one-chunk", B=2, Hq=4, Hkv=1, d=64, N=64, K=1, seed=34, dtype="bf16"),
    custom("bf16-k64-short", B=1, Hq=2, Hkv=1, d=64, N=2048, K=64, seed=35, dtype="bf16"),
    custom("bf16-k1", B=1, Hq=2, Hkv=2, d=128, N=1536, K=1, seed=36, dtype="bf16", needles=2,
           needle_mode="random"),
    custom("bf16-gqa3-cuda-core-select", B=1, Hq=6, Hkv=2, d=64, N=1600, K=7, seed=37, dtype="bf16", needles=2,
           needle_mode="random"),
    custom("bf16-gqa16-d128", B=1, Hq=16, Hkv=1, d=128, N=1024, K=12, seed=38, dtype="bf16"),
    # N a multiple of 4096: pairs are counted through the shared-memory histogram
    custom("bf16-gqa2-8k-hist-count", B=2, Hq=4, Hkv=2, d=64, N=8192, K=16, seed=39, dtype="bf16", needles=4,
           needle_mode="random"),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_prefill_small(w):
    run_prefill_case(w)


@pytest.mark.parametrize("name", ["prefill-32k-h16-d64", "prefill-128k-gqa4-d128"])
def test_prefill_full_size(name):
    run_prefill_case(WORKLOADS[name])


def run_decode_check(w, inp, q_dev, kc, vc, summ, seqlens, oracle, kp, bp, q_f32):
    seq_dev = torch.from_numpy(seqlens.astype(np.int32)).cuda()
    o, ids, scores = hils.decode_step(q_dev, kc, vc, summ, seq_dev, w.K, window=w.window)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    rows = Rows.from_decode(q_f32, seqlens)
    check_rows(w, inp, oracle, kp, bp, None, ids.reshape(-1, w.K).cpu().numpy(),
               scores.reshape(-1, w.K).cpu().numpy(), o.float().reshape(-1, w.d).cpu().numpy(), rows=rows)
    return o, ids


def test_decode_full_size():
    w = WORKLOADS["decode-128k-b8-gqa4-d128"]
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    check_summary(w, inp, summ, kp, bp)
    run_decode_check(w, inp, q, k, v, summ, inp.seqlens, oracle, kp, bp, inp.q_f32)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_decode_ragged_seqlens(dtype):
    # lengths 1 (no candidate chunk, one key) and 65 (one candidate) besides ragged long ones
    w = custom(f"decode-ragged-{dtype}", B=5, Hq=8, Hkv=2, d=64, N=8192, K=8, seed=41, dtype=dtype, kind="decode")
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    seqlens = np.array([8192, 8192 - 37, 100, 1, 65], np.int32)
    run_decode_check(w, inp, q, k, v, summ, seqlens, oracle, kp, bp, inp.q_f32)


DECODE_GROUPS = [
    # query heads per kv head beyond one group of eight (the bf16 partial
    # kernel takes eight heads per tensor-core tile), an odd group, d 128
    custom("decode-g12-d128", B=2, Hq=12, Hkv=1, d=128, N=4096, K=8, seed=42, dtype="bf16", kind="decode"),
    custom("decode-g3-d64", B=3, Hq=6, Hkv=2, d=64, N=4096, K=16, seed=43, dtype="bf16", kind="decode"),
    custom("decode-g32-d64", B=1, Hq=32, Hkv=1, d=64, N=2048, K=4, seed=44, dtype="bf16", kind="decode"),
]


@pytest.mark.parametrize("w", DECODE_GROUPS, ids=[w.name for w in DECODE_GROUPS])
def test_decode_head_groups(w):
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    # a full cache, a ragged one and one whose own chunk holds a single key
    seqlens = np.array([w.N, w.N - 29, 64 * 7 + 1][:w.B], np.int32)
    run_decode_check(w, inp, q, k, v, summ, seqlens, oracle, kp, bp, inp.q_f32)


def test_prefill_and_decode_512k():
    """512K workload: sampled-row prefill parity, then the decode step at full
    length, which must agree with prefill row N-1."""
    w = WORKLOADS["prefill-512k-h16-d64"]
    inp, (q, k, v, lq), o, aux, (oracle, kp, bp) = run_prefill_case(w)
    qd = q[:, :, -1, :].contiguous()
    seqlens = inp.seqlens
    od, ids = run_decode_check(w, inp, qd, k, v, aux["summary"], seqlens, oracle, kp, bp, inp.decode_query())
    assert torch.equal(ids, aux["ids"][:, :, -1, :])
    assert torch.max(torch.abs(od.float() - o[:, :, -1, :].float())).item() <= 2e-2


def test_out_of_range_id_is_recorded_and_skipped():
    w = custom("bounds", B=1, Hq=1, Hkv=1, d=64, N=512, K=3, seed=51, dtype="bf16")
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o, aux = hils.prefill(q, k, v, lq, w.K, return_all=True)
    assert hils.hils_get_status() == 0
    ids = aux["ids"].clone()
    ids[0, 0, 300, 0] = 7       # row 300 is in chunk 4: chunk 7 is not a candidate
    o2 = torch.empty_like(o)
    dims = hils.dims_for(q, k, w.K)
    summ = aux["summary"]
    hils.hils_attn_prefill(dims, q, k, v, summ.kprime, summ.bprime, summ.kprime_mma, ids, aux["scores"], o2, None,
                           hils.prefill_workspace(dims, q.device))
    assert hils.hils_get_status() == 6
    assert hils.hils_get_status() == 0
    others = torch.ones(w.N, dtype=torch.bool)
    others[300] = False
    # the bf16 path accumulates partial outputs with atomics in no fixed order,
    # so untouched rows agree to rounding, not bit for bit
    assert torch.max(torch.abs(o2[0, 0, others].float() - o[0, 0, others].float())).item() <= 1e-2
    assert torch.all(torch.isfinite(o2.float()))


def test_status_word_reports_bad_seqlen_and_clears():
    w = custom("bad-seqlen", B=2, Hq=2, Hkv=1, d=64, N=1024, K=3, seed=52, dtype="bf16", kind="decode")
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    seq = torch.tensor([1024, 0], dtype=torch.int32, device="cuda")
    o, ids, _ = hils.decode_step(q, k, v, summ, seq, w.K)
    assert hils.hils_get_status() == 6
    assert hils.hils_get_status() == 0
    assert torch.all(o[1] == 0) and torch.all(ids[1] == -1)
    assert torch.all(torch.isfinite(o[0].float()))


def test_bounded_wait_times_out_cleanly_and_context_survives():
    """A device wait on a phase that never completes gives up after its limit,
    records HILS_ERR_DEVICE_TIMEOUT and returns; later work still runs."""
    import time
    t0 = time.time()
    hils.hils_selftest_bounded_wait(50)
    assert hils.hils_get_status() == 5
    assert time.time() - t0 < 10
    assert hils.hils_get_status() == 0
    w = custom("after-timeout", B=1, Hq=2, Hkv=1, d=64, N=512, K=3, seed=71, dtype="bf16")
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o = hils.prefill(q, k, v, lq, w.K)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    assert torch.all(torch.isfinite(o.float()))
