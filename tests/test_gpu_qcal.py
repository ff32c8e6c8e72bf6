"""Q-Cal (aitrends.kr article, section "방법론" and glossary entry "저계수
쿼리 보정") through the C ABI: the calibrated query q^ = q + W_up (W_down q)
against the oracle, then the prefill and the decode step whose chunk scores
use q^ while the attention keeps q.

Where a rounding decides the selection, both sides decide in the kernel's
precision: for bf16 the oracle's q^ is rounded to bf16 (round to nearest
even) before it scores the chunks, as the kernels score a bf16 q^.
"""
import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from chunk_wise_sparse_b200.inputs import bf16_bits_to_f32, custom, generate, qcal_weights, round_bf16_bits, sample_rows
from oracle.oracle import Oracle, Rows, qcal
from tests.helpers import OUT_MAX, OUT_MEAN, SEL_GAP, check_selection, gather_rows, to_dev

pytestmark = pytest.mark.gpu

SCORE_TOL = {"fp32": 1e-5, "bf16": 1e-2}


def dev_weights(wt, dtype):
    if dtype == "bf16":
        f = lambda b: torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16)
        return f(wt.w_down_bits), f(wt.w_up_bits)
    return torch.from_numpy(wt.w_down_f32).cuda(), torch.from_numpy(wt.w_up_f32).cuda()


def scoring_query(q_hat64, dtype):
    """The oracle's q^ in the precision the kernels score with."""
    if dtype == "bf16":
        return bf16_bits_to_f32(round_bf16_bits(q_hat64.astype(np.float32)))
    return q_hat64.astype(np.float32)


def calib_bound(q, hq, wt, q_hat64, dtype):
    """Per-element error bound of the kernel's q^: for bf16 (8-bit precision,
    unit roundoff u = 2^-8), the final rounding u |q^| plus the rounding of
    W_down q before the up projection, u sum_a |W_up[t,a] z_a|, and the
    propagation of the latter through the final rounding; fp32 accumulation
    slop."""
    if dtype != "bf16":
        return 1e-5 + 1e-6 * np.abs(q_hat64)
    u = 2.0 ** -8
    z = np.einsum("nrd,nd->nr", wt.w_down_f32[hq].astype(np.float64), q.astype(np.float64))
    up = np.einsum("ndr,nr->nd", np.abs(wt.w_up_f32[hq]).astype(np.float64), np.abs(z))
    return u * np.abs(q_hat64) + u * (1 + u) * up + 1e-5


CALIB = [
    # (dtype, B, Hq, d, n_pos, rank): tensor-core tiles with a ragged last tile, both head dims, the rank range
    ("bf16", 2, 3, 64, 4160, 16),
    ("bf16", 1, 4, 128, 1024, 64),
    ("bf16", 1, 2, 64, 64, 8),
    ("bf16", 3, 8, 128, 1, 32),     # a decode step: CUDA-core kernel
    ("fp32", 1, 4, 64, 512, 32),
    ("fp32", 2, 2, 128, 192, 8),
]


@pytest.mark.parametrize("dtype,B,Hq,d,n_pos,rank", CALIB, ids=[f"{c[0]}-d{c[3]}-n{c[4]}-r{c[5]}" for c in CALIB])
def test_calibrate_matches_oracle(dtype, B, Hq, d, n_pos, rank):
    # the smallest whole number of chunks that holds n_pos positions
    w = custom("qcal", B=B, Hq=Hq, Hkv=Hq, d=d, N=64 * ((n_pos + 63) // 64), K=1, seed=101, dtype=dtype)
    inp = generate(w)
    q_np = inp.q_f32[:, :, :n_pos, :]
    wt = qcal_weights(Hq, d, rank, seed=7, dtype=dtype)
    q = to_dev(inp, "q")[:, :, :n_pos, :].contiguous()
    wd, wu = dev_weights(wt, dtype)
    q_hat = hils.query_calibrate(q, wd, wu)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    flat = q_np.reshape(-1, d)
    hq = np.repeat(np.tile(np.arange(Hq), B), n_pos).astype(np.int32)
    ref = qcal(flat, hq, wt.w_down_f32, wt.w_up_f32)
    got = q_hat.float().reshape(-1, d).cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    bound = calib_bound(flat, hq, wt, ref, dtype)
    assert np.all(err <= bound), (err.max(), np.unravel_index(np.argmax(err - bound), err.shape))
    # in place gives the same bits
    q2 = q.clone()
    hils.query_calibrate(q2, wd, wu, out=q2)
    torch.cuda.synchronize()
    assert torch.equal(q2, q_hat)


PREFILL = [
    custom("qcal-bf16-d64-g2", B=1, Hq=4, Hkv=2, d=64, N=4160, K=16, seed=102, dtype="bf16", needles=4,
           needle_mode="random"),
    custom("qcal-bf16-d128-g4-w256", B=1, Hq=8, Hkv=2, d=128, N=2112, K=8, seed=103, dtype="bf16", window=256),
    custom("qcal-fp32-d64", B=2, Hq=2, Hkv=1, d=64, N=1024, K=5, seed=104, dtype="fp32", needles=2,
           needle_mode="random"),
]


@pytest.mark.parametrize("w", PREFILL, ids=[w.name for w in PREFILL])
def test_prefill_with_qcal(w):
    rank = 16
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    wt = qcal_weights(w.Hq, w.d, rank, seed=w.seed, dtype=w.dtype)
    wd, wu = dev_weights(wt, w.dtype)
    o, aux = hils.prefill_qcal(q, k, v, lq, w.K, wd, wu, return_all=True, window=w.window)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    flat = sample_rows(w)
    rows = Rows.from_prefill(inp.q_f32, flat)
    qs = scoring_query(qcal(rows.q, rows.hq, wt.w_down_f32, wt.w_up_f32), w.dtype)
    srows = Rows(rows.b, rows.hq, rows.pos, qs)
    ids_o, _, gap = oracle.select(kp, bp, srows)
    S = oracle.scores(kp, bp, srows)
    ids_g = gather_rows(aux["ids"], flat).astype(np.int32)
    graded, n, valid = check_selection(ids_g, ids_o, gap, S, SEL_GAP[w.dtype], SEL_GAP[w.dtype])
    kept = ids_g >= 0
    sc_g = gather_rows(aux["scores"], flat)
    rr = np.nonzero(kept)
    if kept.any():
        assert np.abs(sc_g[kept] - S[rr[0], ids_g[kept]]).max() <= SCORE_TOL[w.dtype]
    O_o, lse_o = oracle.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids_g, qscore=qs)
    err = np.abs(gather_rows(o, flat) - O_o)
    assert err.max() <= OUT_MAX[w.dtype], err.max()
    assert err.mean() <= OUT_MEAN[w.dtype], err.mean()
    assert np.max(np.abs(gather_rows(aux["lse_own"][..., None], flat)[:, 0] - lse_o)) <= 1e-4
    # the calibration changed the selection somewhere (the adapter is not a no-op)
    ids_plain, _, _ = oracle.select(kp, bp, rows)
    assert np.any(np.sort(ids_plain, 1) != np.sort(ids_o, 1))
    print(f"[{w.name}] rows {n}: graded {graded}, valid {valid}; O err max {err.max():.2e}")


@pytest.mark.parametrize("dtype,d,paged", [("bf16", 128, False), ("fp32", 64, False), ("bf16", 64, True)])
def test_decode_with_qcal(dtype, d, paged):
    from chunk_wise_sparse_b200.inputs import page_table
    w = custom(f"qcal-decode-{dtype}-{d}", B=3, Hq=8, Hkv=2, d=d, N=8192, K=8, seed=105, dtype=dtype,
               kind="decode")
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    wt = qcal_weights(w.Hq, w.d, 32, seed=5, dtype=dtype)
    wd, wu = dev_weights(wt, dtype)
    summ = hils.landmark_summary(k, lq, w.K)
    seqlens = np.array([8192, 8192 - 37, 300], np.int32)
    seq = torch.from_numpy(seqlens).cuda()
    q_hat = hils.query_calibrate(q, wd, wu)
    o, ids, scores = hils.decode_step_qcal(q, q_hat, k, v, summ, seq, w.K)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    if paged:
        from tests.test_gpu_paged import _pool
        table, n_pages = page_table(w, 5)
        kpool, vpool = _pool(k, table, n_pages), _pool(v, table, n_pages)
        dims = hils.make_dims(w.B, w.Hq, w.Hkv, w.d, w.N, w.K, q.dtype)
        ws = torch.empty((hils.hils_decode_workspace_bytes(dims),), dtype=torch.uint8, device="cuda")
        o_p, ids_p = torch.empty_like(o), torch.empty_like(ids)
        hils.hils_attn_decode_qcal(dims, q, q_hat, kpool, vpool, torch.from_numpy(table).cuda(), n_pages,
                                   summ.kprime, summ.bprime, summ.kprime_mma, seq, o_p, ids_p, None, ws)
        torch.cuda.synchronize()
        assert hils.hils_get_status() == 0
        assert torch.equal(ids_p, ids) and torch.equal(o_p, o)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    rows = Rows.from_decode(inp.q_f32, seqlens)
    qs = scoring_query(qcal(rows.q, rows.hq, wt.w_down_f32, wt.w_up_f32), dtype)
    srows = Rows(rows.b, rows.hq, rows.pos, qs)
    ids_o, _, gap = oracle.select(kp, bp, srows)
    ids_g = ids.reshape(-1, w.K).cpu().numpy()
    check_selection(ids_g, ids_o, gap, oracle.scores(kp, bp, srows), SEL_GAP[dtype], SEL_GAP[dtype])
    O_o, _ = oracle.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids_g, qscore=qs)
    err = np.abs(o.float().reshape(-1, w.d).cpu().numpy() - O_o)
    assert err.max() <= OUT_MAX[dtype], err.max()
    assert err.mean() <= OUT_MEAN[dtype], err.mean()


def test_prefill_with_qcal_full_size():
    """The bench's Q-Cal workload (512K, 16 heads, rank 16) on 4096 sampled rows."""
    from chunk_wise_sparse_b200.inputs import WORKLOADS
    w = WORKLOADS["prefill-512k-h16-d64-qcal16"]
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    wt = qcal_weights(w.Hq, w.d, w.qcal, seed=w.seed, dtype=w.dtype)
    wd, wu = dev_weights(wt, w.dtype)
    o, aux = hils.prefill_qcal(q, k, v, lq, w.K, wd, wu, return_all=True)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    flat = sample_rows(w)
    rows = Rows.from_prefill(inp.q_f32, flat)
    qs = scoring_query(qcal(rows.q, rows.hq, wt.w_down_f32, wt.w_up_f32), w.dtype)
    srows = Rows(rows.b, rows.hq, rows.pos, qs)
    ids_o, _, gap = oracle.select(kp, bp, srows)
    ids_g = gather_rows(aux["ids"], flat).astype(np.int32)
    check_selection(ids_g, ids_o, gap, oracle.scores(kp, bp, srows), SEL_GAP[w.dtype], SEL_GAP[w.dtype])
    O_o, _ = oracle.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids_g, qscore=qs)
    err = np.abs(gather_rows(o, flat) - O_o)
    assert err.max() <= OUT_MAX[w.dtype], err.max()
    assert err.mean() <= OUT_MEAN[w.dtype], err.mean()
