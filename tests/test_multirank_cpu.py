"""The multi-rank path on CPU ranks (gloo, world size 2).

- bench.py's timing arithmetic: every rank reports the max over ranks of its
  step time; job throughput counts every rank's tokens.
- The split of one problem across ranks (chunk_wise_sparse_b200/partition.py):
  every (batch, kv head) group, or decode sequence, goes to exactly one rank,
  and the per-rank results, gathered, equal the one-rank result.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, world)
        out[rank] = (m, bench.job_throughput(world, 1000, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]
    ms, tput = res[0]
    assert ms == pytest.approx(15.0)
    assert tput == pytest.approx(2 * 1000 / 0.015)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1, 524288, 100.0) == pytest.approx(5242880.0)


# ------------------------------------------------------------------ head / batch split of one problem

def test_partition_covers_every_unit_once():
    """For any world size, the ranks' (b, kv head) slices cover every group
    exactly once, each rank's share is contiguous, and shares differ by at most
    one group; the same for the sequences of a decode batch."""
    sys.path.insert(0, ROOT)
    from chunk_wise_sparse_b200.partition import decode_slice, prefill_slices, unit_range
    for B in (1, 2, 3, 8):
        for Hkv in (1, 2, 3, 8, 16):
            for world in (1, 2, 3, 4, 8):
                seen = []
                sizes = []
                for r in range(world):
                    lo, hi = unit_range(B * Hkv, world, r)
                    units = [s.b * Hkv + h for s in prefill_slices(B, Hkv, world, r) for h in range(s.h_lo, s.h_hi)]
                    assert units == list(range(lo, hi))
                    for s in prefill_slices(B, Hkv, world, r):
                        assert 0 <= s.b < B and 0 <= s.h_lo < s.h_hi <= Hkv
                    seen += units
                    sizes.append(hi - lo)
                assert seen == list(range(B * Hkv))
                assert max(sizes) - min(sizes) <= 1
                seqs = [b for r in range(world) for b in range(*decode_slice(B, world, r))]
                assert seqs == list(range(B))


def _split_worker(rank, world, port, out):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from chunk_wise_sparse_b200.inputs import custom, generate
    from chunk_wise_sparse_b200.partition import gather_rows, prefill_slices, slice_heads, unit_range
    from oracle.oracle import Oracle, Rows
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        # 3 batch elements x 2 kv heads = 6 groups: rank 0 takes (b0: h0-1, b1: h0), a range across batch elements
        w = custom("split", B=3, Hq=4, Hkv=2, d=64, N=512, K=3, seed=91, dtype="fp32", needles=2,
                   needle_mode="random")
        inp = generate(w)
        G = w.G
        parts = []
        for s in prefill_slices(w.B, w.Hkv, world, rank):
            Q = np.ascontiguousarray(slice_heads(inp.q_f32, s, G))
            Kt, Vt, LQ = (np.ascontiguousarray(slice_heads(a, s)) for a in (inp.k_f32, inp.v_f32, inp.lq_f32))
            o = Oracle(1, s.heads_kv * G, s.heads_kv, w.N, w.d, w.C, w.K)
            kp, bp = o.summary(Kt, LQ)
            rows = Rows.from_prefill(Q, np.arange(s.heads_kv * G * w.N))
            ids, _, _ = o.select(kp, bp, rows)
            O, _ = o.attend(Kt, Vt, kp, bp, rows, ids)
            parts.append(O.reshape(s.heads_kv, G, w.N, w.d))
        local = torch.from_numpy(np.concatenate(parts, axis=0))
        full = gather_rows(local, world, w.B * w.Hkv, lambda r: unit_range(w.B * w.Hkv, world, r))
        out[rank] = full.numpy()
    finally:
        dist.destroy_process_group()


def test_head_split_gloo_world2_equals_one_rank():
    """Each of two CPU ranks runs the oracle on its (b, kv head) groups only;
    the gathered outputs equal the one-rank result on the whole problem bit
    for bit (the groups are independent problems)."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from chunk_wise_sparse_b200.inputs import custom, generate
    from oracle.oracle import Oracle, Rows
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_split_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(out)
    w = custom("split", B=3, Hq=4, Hkv=2, d=64, N=512, K=3, seed=91, dtype="fp32", needles=2, needle_mode="random")
    inp = generate(w)
    o = Oracle.for_workload(w)
    kp, bp = o.summary(inp.k_f32, inp.lq_f32)
    rows = Rows.from_prefill(inp.q_f32, np.arange(w.B * w.Hq * w.N))
    ids, _, _ = o.select(kp, bp, rows)
    O, _ = o.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids)
    want = O.reshape(w.B * w.Hkv, w.G, w.N, w.d)
    assert np.array_equal(res[0], res[1])
    assert np.array_equal(res[0], want)
