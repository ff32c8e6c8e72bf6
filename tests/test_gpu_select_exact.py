"""Chunk selection on scores that are exact in every precision.

The scoring operand is built directly from small integers (k' entries and
query entries in {-1, 0, 1}, or an ascending ramp), so every score
tau * <q, k'> is a multiple of 1/8 that the tensor-core path, the fp32
epilogue and the fp64 oracle all compute exactly.  Ties are then real ties and
the selection must equal the oracle's element for element: the K largest
scores, equal scores ordered by lower chunk id (HiLS paper, aitrends.kr
article, section "방법론"; tie rule as read in the design notes), ids in
ascending order, -1 padding.  Rows are sampled across every row length at
which a kernel changes how it bounds the K-th score (no bound, groups of 8,
16, 32, 64 and 128 chunks) and both rows of each boundary.  At d = 64 and
K <= 16 the selection runs with two threads per row, whose halves exchange
their bounds and merge their lists: the ties cases check that merge against
the lower-id rule.
"""
import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from oracle.oracle import Oracle, Rows

pytestmark = pytest.mark.gpu

C = 64


def _operand(kp):
    """Scoring operand [B, Hkv, nc, d+16] bf16: k' then x_hi = x_lo = 0 (b' = 0)."""
    B, H, nc, d = kp.shape
    op = torch.zeros((B, H, nc, d + 16), dtype=torch.bfloat16)
    op[..., :d] = torch.from_numpy(kp.astype(np.float32)).to(torch.bfloat16)
    assert torch.equal(op[..., :d].float(), torch.from_numpy(kp.astype(np.float32)))
    return op.cuda()


def _rows(N, K, Hq, rng):
    """Sampled positions: random ones plus both sides of every length at
    which a bound changes (n = 8K, 16K, 32K, 64K, 128K candidates)."""
    pos = set(rng.integers(0, N, 192).tolist()) | {0, 1, C - 1, C, 2 * C, N - 1}
    for mult in (8, 16, 32, 64, 128):
        for n in (mult * K - 1, mult * K, mult * K + 1):
            for off in (0, C - 1):
                p = n * C + off
                if 0 <= p < N:
                    pos.add(p)
    pos = np.array(sorted(pos), np.int64)
    hq = np.arange(len(pos)) % Hq
    return pos, hq


@pytest.mark.parametrize("kind,K", [("ties", 16), ("ascending", 16), ("ties", 32), ("ascending", 32),
                                    ("ties", 3), ("ties", 64), ("ascending", 64)])
def test_select_exact_on_representable_scores(kind, K):
    B, Hq, Hkv, d, N = 1, 2, 1, 64, 262144
    nc = N // C
    rng = np.random.default_rng(11 + K)
    if kind == "ties":
        q = rng.integers(-1, 2, (B, Hq, N, d)).astype(np.float32)
        kp = rng.integers(-1, 2, (B, Hkv, nc, d)).astype(np.float64)
    else:
        # score of chunk c = c / 8: every new chunk beats all earlier ones
        q = np.zeros((B, Hq, N, d), np.float32)
        q[..., 0] = 1.0
        q[..., 1] = 1.0
        c = np.arange(nc)
        kp = np.zeros((B, Hkv, nc, d), np.float64)
        kp[..., 0] = (c // 16) * 16
        kp[..., 1] = c % 16
    bp = np.zeros((B, Hkv, nc), np.float64)
    q_dev = torch.from_numpy(q).to(torch.bfloat16).cuda()
    assert torch.equal(q_dev.float().cpu(), torch.from_numpy(q))
    op = _operand(kp)
    dims = hils.make_dims(B, Hq, Hkv, d, N, K, torch.bfloat16)
    ids = torch.empty((B, Hq, N, K), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, Hq, N, K), dtype=torch.float32, device="cuda")
    dummy = torch.zeros((1,), dtype=torch.float32, device="cuda")
    hils.hils_select(dims, q_dev, dummy, dummy, op, None, 0, ids, sc)
    torch.cuda.synchronize()
    assert hils.hils_get_status() == 0

    pos, hq = _rows(N, K, Hq, rng)
    b = np.zeros_like(pos)
    rows = Rows(b, hq, pos, q[0, hq, pos, :])
    o = Oracle(B, Hq, Hkv, N, d, C, K)
    ids_o, sc_o, _ = o.select(kp, bp, rows)
    ids_g = ids[0, hq, pos].cpu().numpy()
    sc_g = sc[0, hq, pos].cpu().numpy()
    for r in range(len(pos)):
        assert np.array_equal(ids_g[r], ids_o[r]), f"pos {pos[r]} head {hq[r]}: {ids_g[r]} vs {ids_o[r]}"
        kept = ids_o[r] >= 0
        assert np.array_equal(sc_g[r][kept], sc_o[r][kept].astype(np.float32)), f"pos {pos[r]}: scores differ"
        assert np.all(np.isneginf(sc_g[r][~kept]))
