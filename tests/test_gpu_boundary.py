"""The optional arguments of the C ABI against the fp64 oracle.

- hils_select on a listed subset of query positions (row_pos, n_rows).
- hils_attn_prefill without the selection's scores: the chunk scores of the
  kept ids are recomputed from q and the landmark summaries (aitrends.kr
  article, section "방법론": s^ = tau <q, k'> + b').
- Run-to-run reproducibility of the bf16 prefill, whose partial outputs are
  summed in fp32 in no fixed order: at most one bf16 ulp apart (about 1e-6
  for outputs that are almost zero).

Acceptance as in test_gpu_parity.py (tests/helpers.py): exact id sets where
the oracle's K-th/(K+1)-th gap is at least 1e-3 (fp32) or 2e-2 (bf16), valid
selections on every row, outputs within max-abs 1e-5 (fp32) or max-abs 2e-2
and mean-abs 2e-3 (bf16) of the oracle run on the GPU's ids.
"""
import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from chunk_wise_sparse_b200.inputs import WORKLOADS, custom, generate, sample_rows
from oracle.oracle import Oracle, Rows
from tests.helpers import OUT_MAX, OUT_MEAN, SEL_GAP, check_selection, gather_rows, to_dev

pytestmark = pytest.mark.gpu

SCORE_TOL = {"fp32": 1e-5, "bf16": 1e-2}

CASES = [
    custom("bf16-d64-ragged-noscores", B=2, Hq=2, Hkv=2, d=64, N=4288, K=16, seed=71, dtype="bf16", needles=4,
           needle_mode="random"),
    custom("bf16-d128-gqa4-noscores", B=1, Hq=8, Hkv=2, d=128, N=2112, K=32, seed=72, dtype="bf16", needles=2,
           needle_mode="random"),
    custom("fp32-d64-noscores", B=1, Hq=2, Hkv=1, d=64, N=1024, K=5, seed=73, dtype="fp32", needles=2,
           needle_mode="random"),
    custom("bf16-gqa3-cuda-core-noscores", B=1, Hq=6, Hkv=2, d=64, N=1600, K=7, seed=74, dtype="bf16"),
    custom("bf16-window512-noscores", B=1, Hq=4, Hkv=2, d=64, N=3072, K=8, seed=75, dtype="bf16", window=512),
]


def oracle_check(w, inp, oracle, kp, bp, flat, ids, o):
    rows = Rows.from_prefill(inp.q_f32, flat)
    ids_o, _, gap = oracle.select(kp, bp, rows)
    S = oracle.scores(kp, bp, rows)
    check_selection(ids, ids_o, gap, S, SEL_GAP[w.dtype], SEL_GAP[w.dtype])
    O_o, _ = oracle.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids)
    err = np.abs(o - O_o)
    assert err.max() <= OUT_MAX[w.dtype] and err.mean() <= OUT_MEAN[w.dtype], (err.max(), err.mean())
    return err


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_prefill_without_scores(w):
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o_ref, aux = hils.prefill(q, k, v, lq, w.K, return_all=True, window=w.window)
    o, aux0 = hils.prefill(q, k, v, lq, w.K, return_all=True, window=w.window, scores_buffer=False)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    assert aux0["scores"] is None
    # the selection does not depend on whether it writes scores
    assert torch.equal(aux0["ids"], aux["ids"])
    # the recomputed scores differ from the selection's only in the order of fp32 sums
    diff = (o.float() - o_ref.float()).abs().max().item()
    assert diff <= (1e-6 if w.dtype == "fp32" else 2 ** -7), diff
    assert torch.allclose(aux0["lse_own"], aux["lse_own"], rtol=0, atol=1e-6)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    flat = sample_rows(w, 4096)
    oracle_check(w, inp, oracle, kp, bp, flat, gather_rows(aux0["ids"], flat).astype(np.int32),
                 gather_rows(o, flat))


def test_prefill_without_scores_32k():
    """The 345M-shaped workload (32K, 16 heads) without a scores buffer:
    sampled rows against the oracle, every row against the scores path."""
    w = WORKLOADS["prefill-32k-h16-d64"]
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o_ref = hils.prefill(q, k, v, lq, w.K)
    o, aux = hils.prefill(q, k, v, lq, w.K, return_all=True, scores_buffer=False)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    assert (o.float() - o_ref.float()).abs().max().item() <= 2 ** -7
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    flat = sample_rows(w, 4096)
    oracle_check(w, inp, oracle, kp, bp, flat, gather_rows(aux["ids"], flat).astype(np.int32), gather_rows(o, flat))


SUBSET = [
    custom("bf16-d64-rows", B=2, Hq=2, Hkv=2, d=64, N=4096, K=16, seed=76, dtype="bf16", needles=4,
           needle_mode="random"),
    custom("bf16-d128-gqa4-rows", B=1, Hq=8, Hkv=2, d=128, N=2048, K=32, seed=77, dtype="bf16"),
    custom("fp32-d64-rows", B=1, Hq=2, Hkv=1, d=64, N=1024, K=3, seed=78, dtype="fp32", needles=2,
           needle_mode="random"),
    custom("bf16-window-rows", B=1, Hq=2, Hkv=1, d=64, N=2048, K=4, seed=79, dtype="bf16", window=256),
]


@pytest.mark.parametrize("w", SUBSET, ids=[w.name for w in SUBSET])
def test_select_row_subset(w):
    """Listed positions (unsorted, with repeats, the first and last position,
    a ragged count) select exactly what the oracle selects for them."""
    inp = generate(w)
    q, k, lq = (to_dev(inp, n) for n in ("q", "k", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    rng = np.random.default_rng(w.seed)
    pos = np.concatenate([[w.N - 1, 0, 63, 64, 65], rng.integers(0, w.N, size=300), [w.N - 1]]).astype(np.int64)
    pos_dev = torch.from_numpy(pos).cuda()
    ids, sc = hils.select(q, summ, w.Hkv, w.K, window=w.window, row_pos=pos_dev)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    assert ids.shape == (w.B, w.Hq, len(pos), w.K)
    # the repeated position gives the same row twice
    assert torch.equal(ids[:, :, 0], ids[:, :, -1]) and torch.equal(sc[:, :, 0], sc[:, :, -1])
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    b = np.repeat(np.arange(w.B), w.Hq * len(pos))
    hq = np.tile(np.repeat(np.arange(w.Hq), len(pos)), w.B)
    p = np.tile(pos, w.B * w.Hq)
    rows = Rows(b, hq, p, inp.q_f32[b, hq, p, :])
    ids_o, _, gap = oracle.select(kp, bp, rows)
    S = oracle.scores(kp, bp, rows)
    ids_g = ids.reshape(-1, w.K).cpu().numpy().astype(np.int32)
    sc_g = sc.reshape(-1, w.K).cpu().numpy()
    graded, n, valid = check_selection(ids_g, ids_o, gap, S, SEL_GAP[w.dtype], SEL_GAP[w.dtype])
    kept = ids_g >= 0
    rr = np.nonzero(kept)
    if kept.any():
        assert np.abs(sc_g[kept] - S[rr[0], ids_g[kept]]).max() <= SCORE_TOL[w.dtype]
    assert np.all(np.isneginf(sc_g[~kept]))
    # the same positions out of the full selection agree where the choice is clear
    ids_all, _ = hils.select(q, summ, w.Hkv, w.K, window=w.window)
    full = ids_all[:, :, pos_dev].reshape(-1, w.K).cpu().numpy()
    clear = gap >= SEL_GAP[w.dtype]
    assert np.array_equal(np.sort(full[clear], axis=1), np.sort(ids_g[clear], axis=1))
    print(f"[{w.name}] rows {n}: graded {graded}, valid {valid}")


def test_select_row_subset_out_of_range_position_is_recorded():
    w = custom("rows-bounds", B=1, Hq=2, Hkv=2, d=64, N=1024, K=3, seed=80, dtype="bf16")
    inp = generate(w)
    q, k, lq = (to_dev(inp, n) for n in ("q", "k", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    pos = torch.tensor([700, 1024, 900, -3], dtype=torch.int64, device="cuda")
    ids, sc = hils.select(q, summ, w.Hkv, w.K, row_pos=pos)
    assert hils.hils_get_status() == 6
    assert hils.hils_get_status() == 0
    assert torch.all(ids[:, :, 1] == -1) and torch.all(ids[:, :, 3] == -1)
    assert torch.all(torch.isneginf(sc[:, :, 1]))
    ids_ok, _ = hils.select(q, summ, w.Hkv, w.K, row_pos=pos[[0, 2]].contiguous())
    assert torch.equal(ids[:, :, [0, 2]], ids_ok)


def test_prefill_bf16_run_to_run_within_one_ulp():
    """Two prefills of the 32K workload on the same inputs: identical ids and
    log-sum-exps; outputs at most one bf16 ulp apart, plus 2^-20 for outputs
    near zero (the fp32 sums of the partial outputs run in no fixed order; two
    such sums differ by far less than a bf16 ulp unless they cancel to almost
    nothing)."""
    w = WORKLOADS["prefill-32k-h16-d64"]
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o1, a1 = hils.prefill(q, k, v, lq, w.K, return_all=True)
    o2, a2 = hils.prefill(q, k, v, lq, w.K, return_all=True)
    torch.cuda.synchronize()
    assert torch.equal(a1["ids"], a2["ids"]) and torch.equal(a1["lse_own"], a2["lse_own"])
    x1, x2 = o1.float(), o2.float()
    mag = torch.maximum(x1.abs(), x2.abs())
    # one bf16 ulp of the larger magnitude (8 significant bits), a subnormal floor
    ulp = torch.where(mag > 0, torch.exp2(torch.floor(torch.log2(mag)) - 7), torch.zeros_like(mag))
    ulp = torch.clamp(ulp, min=2.0 ** -133)
    d = (x1 - x2).abs()
    n_diff = int((d > 0).sum().item())
    n_over = int((d > ulp).sum().item())
    assert torch.all(d <= ulp + 2.0 ** -20), (d - ulp).max().item()
    print(f"run-to-run: {n_diff} of {d.numel()} outputs differ, {n_over} by more than one bf16 ulp "
          f"(all near zero), max diff {d.max().item():.3e}")
