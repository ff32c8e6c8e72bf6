"""The decode entry point that allocates nothing (hils_attn_decode_fixed_scratch).

Some callers cannot call cudaMalloc: a plugin inside a host inference engine
that owns all device memory and hands out no workspace, or a decode loop that
must not pay the device-wide synchronisation cudaMalloc implies.  For them the
library keeps the decode scratch in a fixed device array of its own.  These
tests check, through the C ABI, that two calls in a row give the results of
hils_attn_decode with a caller-provided workspace, that those calls take no
device memory, and that sizes beyond the array are refused before anything
is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

from chunk_wise_sparse_b200 import hils
from chunk_wise_sparse_b200.inputs import custom, generate
from tests.helpers import OUT_MAX, OUT_MEAN, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fixed_scratch_decode_matches_workspace_decode(dtype):
    w = custom(f"fixed-scratch-{dtype}", B=3, Hq=8, Hkv=2, d=128, N=16384, K=16, seed=61, dtype=dtype,
               kind="decode")
    inp = generate(w)
    q, k, v, lq = (to_dev(inp, n) for n in ("q", "k", "v", "lq"))
    summ = hils.landmark_summary(k, lq, w.K)
    dims = hils.make_dims(w.B, w.Hq, w.Hkv, w.d, w.N, w.K, q.dtype)
    assert hils.hils_decode_workspace_bytes(dims) <= hils.DECODE_FIXED_SCRATCH_BYTES
    cases = []
    for seqlens in ([16384, 16384 - 100, 777], [9000, 64, 16384]):
        seq = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
        ref = hils.decode_step(q, k, v, summ, seq, w.K)
        out = (torch.full_like(q, float("nan")),
               torch.full((w.B, w.Hq, w.K), -7, dtype=torch.int32, device="cuda"),
               torch.full((w.B, w.Hq, w.K), float("nan"), dtype=torch.float32, device="cuda"))
        cases.append((seq, ref, out))
    # a first call loads the library's device code (and with it the array) on this GPU
    warm = torch.empty_like(q)
    hils.hils_attn_decode_fixed_scratch(dims, q, k, v, summ.kprime, summ.bprime, summ.kprime_mma, cases[0][0], warm,
                                        None, None)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    # two calls in a row with different lengths: stale scratch from the first call must not leak
    for seq, _, (o, ids, sc) in cases:
        hils.hils_attn_decode_fixed_scratch(dims, q, k, v, summ.kprime, summ.bprime, summ.kprime_mma, seq, o,
                                            ids, sc)
    torch.cuda.synchronize()
    # nothing was allocated on the device by the two calls
    assert torch.cuda.mem_get_info()[0] == free_before
    assert hils.hils_get_status() == 0
    for seq, (ref_o, ref_ids, ref_sc), (o, ids, sc) in cases:
        assert torch.equal(ids, ref_ids)
        err = (o.float() - ref_o.float()).abs()
        assert err.max().item() <= OUT_MAX[dtype] and err.mean().item() <= OUT_MEAN[dtype]
        fin = torch.isfinite(ref_sc)
        assert torch.equal(fin, torch.isfinite(sc))
        assert torch.max(torch.abs(sc[fin] - ref_sc[fin])).item() <= 1e-5


def test_fixed_scratch_rejects_sizes_beyond_its_maximum():
    dims = hils.make_dims(16, 64, 8, 128, 1 << 20, 64, hils.BF16)
    assert hils.hils_decode_workspace_bytes(dims) > hils.DECODE_FIXED_SCRATCH_BYTES
    p = ctypes.c_void_p(256)   # never dereferenced: the size check comes first
    rc = hils.lib().hils_attn_decode_fixed_scratch(ctypes.byref(dims), p, p, p, None, None, p, p, p, None, None,
                                                   None)
    assert rc == 4
    assert "workspace" in hils.strerror(rc)
