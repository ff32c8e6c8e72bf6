"""Chunk-paged KV cache (aitrends.kr article, section "기술 상세": chunk-unit
KV paging) through the C ABI: the paged summary and decode step must equal the
contiguous calls bit for bit on the cache the page table describes (same
kernels, same arithmetic), match the oracle on that cache, and record a page
outside the pool as HILS_ERR_DEVICE_BOUNDS without touching other sequences.
"""
import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from chunk_wise_sparse_b200.inputs import custom, generate, page_table
from oracle.oracle import Oracle, Rows, gather_pages
from tests.helpers import OUT_MAX, OUT_MEAN, SEL_GAP, check_selection, to_dev

pytestmark = pytest.mark.gpu

C = 64


def _pool(cache, table, n_pages):
    """[n_pages, Hkv, C, d] pool holding chunk (b, c) of `cache` at page table[b, c];
    the spare pages hold noise."""
    B, H, N, d = cache.shape
    nc = N // C
    pool = torch.randn((n_pages, H, C, d), device=cache.device).to(cache.dtype)
    chunks = cache.view(B, H, nc, C, d).permute(0, 2, 1, 3, 4).reshape(B * nc, H, C, d)
    pool[torch.from_numpy(table.reshape(-1).astype(np.int64)).to(cache.device)] = chunks
    return pool


def _run(w, seqlens, spare=9, corrupt=None):
    win = w.window
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    table, n_pages = page_table(w, spare)
    kpool, vpool = _pool(k, table, n_pages), _pool(v, table, n_pages)
    if corrupt is not None:
        # only the table the kernels read gets the entry outside the pool
        table = table.copy()
        table[corrupt] = n_pages + 3
    tab = torch.from_numpy(table).cuda()
    dims = hils.make_dims(w.B, w.Hq, w.Hkv, w.d, w.N, w.K, q.dtype, window=win)
    seq = torch.from_numpy(seqlens.astype(np.int32)).cuda()
    # contiguous reference calls
    summ = hils.landmark_summary(k, lq, w.K)
    o_c, ids_c, sc_c = hils.decode_step(q, k, v, summ, seq, w.K, window=win)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    # paged calls
    summ_p = hils.Summary(dims, q.device)
    for t in (summ_p.kprime, summ_p.bprime, summ_p.kprime_mma):
        if t is not None:
            t.zero_()   # a chunk whose page is bad stays unwritten: keep it finite
    hils.hils_landmark_summary_paged(dims, kpool, tab, n_pages, lq, 0, w.nc, summ_p.kprime, summ_p.bprime,
                                     summ_p.kprime_mma)
    ws = torch.empty((hils.hils_decode_workspace_bytes(dims),), dtype=torch.uint8, device="cuda")
    o_p = torch.empty_like(q)
    ids_p = torch.empty((w.B, w.Hq, w.K), dtype=torch.int32, device="cuda")
    sc_p = torch.empty((w.B, w.Hq, w.K), dtype=torch.float32, device="cuda")
    hils.hils_attn_decode_paged(dims, q, kpool, vpool, tab, n_pages, summ_p.kprime, summ_p.bprime,
                                summ_p.kprime_mma, seq, o_p, ids_p, sc_p, ws)
    torch.cuda.synchronize()
    status = hils.hils_get_status()
    return dict(inp=inp, table=table, n_pages=n_pages, kpool=kpool, vpool=vpool, summ=summ, summ_p=summ_p,
                o_c=o_c, ids_c=ids_c, sc_c=sc_c, o_p=o_p, ids_p=ids_p, sc_p=sc_p, status=status)


@pytest.mark.parametrize("dtype,d,window", [("bf16", 128, 0), ("bf16", 64, 0), ("fp32", 64, 0), ("bf16", 128, 512)])
def test_paged_equals_contiguous_and_matches_the_oracle(dtype, d, window):
    w = custom(f"paged-{dtype}-{d}-w{window}", B=3, Hq=8, Hkv=2, d=d, N=16384, K=16, seed=71, dtype=dtype,
               kind="decode", window=window)
    seqlens = np.array([16384, 16384 - 45, 700], np.int32)
    r = _run(w, seqlens)
    assert r["status"] == 0
    assert torch.equal(r["summ"].kprime, r["summ_p"].kprime)
    assert torch.equal(r["summ"].bprime, r["summ_p"].bprime)
    if dtype == "bf16":
        assert torch.equal(r["summ"].kprime_mma, r["summ_p"].kprime_mma)
    assert torch.equal(r["ids_c"], r["ids_p"])
    assert torch.equal(r["sc_c"], r["sc_p"])
    assert torch.equal(r["o_c"], r["o_p"])
    # oracle on the cache the pool and table describe
    inp = r["inp"]
    pool_k = r["kpool"].float().cpu().numpy().astype(np.float64)
    pool_v = r["vpool"].float().cpu().numpy().astype(np.float64)
    kg, vg = gather_pages(pool_k, r["table"]), gather_pages(pool_v, r["table"])
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(kg, inp.lq_f32)
    ref = oracle.decode(inp.q_f32, kg, vg, kp, bp, seqlens)
    rows = ref["rows"]
    ids_g = r["ids_p"].reshape(-1, w.K).cpu().numpy()
    check_selection(ids_g, ref["ids"].reshape(-1, w.K), ref["gap"].reshape(-1), oracle.scores(kp, bp, rows),
                    SEL_GAP[dtype], SEL_GAP[dtype])
    O_o, _ = oracle.attend(kg, vg, kp, bp, rows, ids_g)
    err = np.abs(r["o_p"].float().reshape(-1, w.d).cpu().numpy() - O_o)
    assert err.max() <= OUT_MAX[dtype], err.max()
    assert err.mean() <= OUT_MEAN[dtype], err.mean()


def test_page_outside_the_pool_is_recorded_and_other_sequences_are_untouched():
    w = custom("paged-bad", B=2, Hq=4, Hkv=1, d=64, N=8192, K=8, seed=72, dtype="bf16", kind="decode")
    seqlens = np.array([8192, 8192], np.int32)
    r = _run(w, seqlens, corrupt=(0, 5))   # sequence 0, chunk 5
    assert r["status"] == 6   # HILS_ERR_DEVICE_BOUNDS
    assert torch.isfinite(r["o_p"].float()).all()
    # sequence 1 does not read the bad entry: identical to the contiguous call
    assert torch.equal(r["o_c"][1], r["o_p"][1])
    assert torch.equal(r["ids_c"][1], r["ids_p"][1])
