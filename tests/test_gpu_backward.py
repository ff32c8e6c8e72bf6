"""Backward pass through the C ABI against the oracle's backward.

The GPU backward is driven by the oracle's forward state for the same inputs
(its selection, chunk scores, window log-sum-exp, compressed keys and output,
rounded to the types the ABI takes), so both sides differentiate the same
forward; no oracle input comes from the GPU.  Tolerances: fp32, max error
1e-4 of the gradient's largest magnitude; bf16 inputs (gradients still in
fp32), 1e-2 of it and 1e-3 on average -- the bf16 output O enters
<dO, O> rounded to 8 bits of precision.
"""
import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from chunk_wise_sparse_b200.inputs import bf16_bits_to_f32, custom, generate, qcal_weights, round_bf16_bits
from oracle.oracle import Oracle, Rows, qcal
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu

TOL = {"fp32": (1e-4, 1e-5), "bf16": (1e-2, 1e-3)}


def dev_dtype(x, dtype):
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return torch.from_numpy(round_bf16_bits(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(x).cuda()


def as_stored(x, dtype):
    x = np.ascontiguousarray(x, dtype=np.float32)
    return bf16_bits_to_f32(round_bf16_bits(x)) if dtype == "bf16" else x


def run_case(w, use_qcal=False, corrupt=None):
    inp = generate(w)
    B, Hq, Hkv, N, d, K = w.B, w.Hq, w.Hkv, w.N, w.d, w.K
    rng = np.random.default_rng(w.seed + 500)
    dO = as_stored(rng.standard_normal((B, Hq, N, d)).astype(np.float32), w.dtype)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    rows = Rows.from_prefill(inp.q_f32, np.arange(B * Hq * N))
    Qs = None
    if use_qcal:
        wt = qcal_weights(Hq, d, 16, seed=w.seed, dtype=w.dtype)
        Qs = as_stored(qcal(rows.q, rows.hq, wt.w_down_f32, wt.w_up_f32), w.dtype).reshape(B, Hq, N, d)
        srows = Rows(rows.b, rows.hq, rows.pos, Qs.reshape(len(rows), d))
    else:
        srows = rows
    ids, sel, _ = oracle.select(kp, bp, srows)
    O, lse = oracle.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids,
                           qscore=None if Qs is None else Qs.reshape(len(rows), d))
    ref = oracle.backward(inp.q_f32, inp.k_f32, inp.v_f32, inp.lq_f32, ids.reshape(B, Hq, N, K), dO, Qs=Qs)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    ids_d = torch.from_numpy(ids.reshape(B, Hq, N, K)).cuda()
    if corrupt is not None:
        ids_d[corrupt] = N // 64 + 3
    dims = hils.make_dims(B, Hq, Hkv, d, N, K, q.dtype, window=w.window)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    g = dict(dq=torch.empty((B, Hq, N, d), device="cuda"), dk=torch.empty((B, Hkv, N, d), device="cuda"),
             dv=torch.empty((B, Hkv, N, d), device="cuda"), dlq=torch.empty((B, Hkv, N // 64, d), device="cuda"),
             dq_score=torch.empty((B, Hq, N, d), device="cuda") if use_qcal else None)
    ws = torch.empty((hils.hils_attn_backward_workspace_bytes(dims),), dtype=torch.uint8, device="cuda")
    hils.hils_attn_backward(dims, q, dev_dtype(Qs, w.dtype) if use_qcal else None, k, v, lq, f32(kp),
                            ids_d, f32(sel.reshape(B, Hq, N, K)), f32(lse.reshape(B, Hq, N)),
                            dev_dtype(O.reshape(B, Hq, N, d), w.dtype), dev_dtype(dO, w.dtype),
                            g["dq"], g["dq_score"], g["dk"], g["dv"], g["dlq"], ws)
    torch.cuda.synchronize()
    return g, ref, hils.hils_get_status()


def check(g, ref, dtype, names):
    rmax, rmean = TOL[dtype]
    for n in names:
        got = g[n].cpu().numpy().astype(np.float64)
        want = ref["dQs" if n == "dq_score" else {"dq": "dQ", "dk": "dK", "dv": "dV", "dlq": "dLQ"}[n]]
        scale = max(1e-6, np.max(np.abs(want)))
        err = np.abs(got - want)
        assert err.max() <= rmax * scale, (n, err.max(), scale)
        assert err.mean() <= rmean * scale, (n, err.mean(), scale)
        print(f"{n}: max err {err.max() / scale:.2e}, mean {err.mean() / scale:.2e} of {scale:.3g}")


CASES = [
    custom("bwd-fp32-d64-g2", B=1, Hq=4, Hkv=2, d=64, N=512, K=3, seed=201, dtype="fp32"),
    custom("bwd-fp32-d128-w192", B=2, Hq=2, Hkv=2, d=128, N=448, K=4, seed=202, dtype="fp32", window=192),
    custom("bwd-bf16-d64-g4", B=1, Hq=8, Hkv=2, d=64, N=1024, K=8, seed=203, dtype="bf16"),
    custom("bwd-bf16-d128-w256", B=1, Hq=2, Hkv=1, d=128, N=640, K=5, seed=204, dtype="bf16", window=256),
    custom("bwd-fp32-d64-g3", B=1, Hq=6, Hkv=2, d=64, N=384, K=2, seed=205, dtype="fp32"),
    # bf16 without a window, d 128, two batch elements: full and ragged tiles of the tensor-core kernel
    custom("bwd-bf16-d128-g2", B=2, Hq=4, Hkv=2, d=128, N=1024, K=6, seed=209, dtype="bf16"),
    # one query head per kv head with a window (tiles of every pair count), and eight heads per kv head
    custom("bwd-bf16-d64-g1-w128", B=2, Hq=2, Hkv=2, d=64, N=768, K=3, seed=210, dtype="bf16", window=128),
    custom("bwd-bf16-d128-g8", B=1, Hq=8, Hkv=1, d=128, N=512, K=4, seed=211, dtype="bf16"),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_backward_matches_oracle(w):
    g, ref, status = run_case(w)
    assert status == 0
    check(g, ref, w.dtype, ["dq", "dk", "dv", "dlq"])


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_backward_with_a_scoring_query(dtype):
    w = custom(f"bwd-qcal-{dtype}", B=1, Hq=4, Hkv=2, d=64, N=512, K=4, seed=206, dtype=dtype)
    g, ref, status = run_case(w, use_qcal=True)
    assert status == 0
    check(g, ref, dtype, ["dq", "dq_score", "dk", "dv", "dlq"])


def test_backward_records_an_id_outside_the_candidates():
    w = custom("bwd-bad-id", B=1, Hq=2, Hkv=1, d=64, N=256, K=2, seed=207, dtype="fp32")
    g, ref, status = run_case(w, corrupt=(0, 0, 200, 0))
    assert status == 6
    assert all(torch.isfinite(g[n]).all() for n in ("dq", "dk", "dv", "dlq"))


def test_backward_after_the_gpu_forward():
    """fp32: the GPU forward selects what the oracle selects here, so the
    gradients of the whole GPU chain match the oracle's."""
    w = custom("bwd-chain-fp32", B=1, Hq=2, Hkv=1, d=64, N=512, K=3, seed=208, dtype="fp32")
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o, aux = hils.prefill(q, k, v, lq, w.K, return_all=True)
    oracle = Oracle.for_workload(w)
    kp, bp = oracle.summary(inp.k_f32, inp.lq_f32)
    ids_o, _, _ = oracle.select(kp, bp, Rows.from_prefill(inp.q_f32, np.arange(w.Hq * w.N)))
    assert np.array_equal(aux["ids"].reshape(-1, w.K).cpu().numpy(), ids_o)
    dO = np.random.default_rng(3).standard_normal((1, 2, w.N, w.d)).astype(np.float32)
    g = hils.backward(q, k, v, lq, aux, o, torch.from_numpy(dO).cuda(), w.K)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    ref = oracle.backward(inp.q_f32, inp.k_f32, inp.v_f32, inp.lq_f32, ids_o.reshape(1, 2, w.N, w.K), dO)
    check(g, ref, "fp32", ["dq", "dk", "dv", "dlq"])


def test_backward_full_size_identities():
    """The bench's 32K workload after the GPU forward: at any size each row's
    fusion weights sum to 1, so sum_j dV_j = sum over the kv head's query heads
    of sum_i dO_i; and a common shift of all keys of a kv head leaves the output
    unchanged, so sum_j dK_j = 0 (up to the bf16 rounding of O in <dO, O>)."""
    from chunk_wise_sparse_b200.inputs import WORKLOADS
    w = WORKLOADS["prefill-32k-h16-d64"]
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    o, aux = hils.prefill(q, k, v, lq, w.K, return_all=True)
    d_o = torch.randn(q.shape, device="cuda", generator=torch.Generator(device="cuda").manual_seed(5)).to(q.dtype)
    g = hils.backward(q, k, v, lq, aux, o, d_o, w.K)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0
    G = w.Hq // w.Hkv
    dO = d_o.float().view(w.B, w.Hkv, G, w.N, w.d).sum(dim=(2, 3))
    sv = g["dv"].sum(dim=2)
    assert torch.max(torch.abs(sv - dO)).item() <= 1e-3 * max(1.0, torch.max(torch.abs(dO)).item())
    sk = g["dk"].sum(dim=2)
    scale = g["dk"].abs().sum(dim=2)
    assert torch.all(torch.abs(sk) <= 1e-2 * scale + 1e-3), (torch.abs(sk) / scale).max().item()
    assert all(torch.isfinite(g[n]).all() for n in ("dq", "dk", "dv", "dlq"))
