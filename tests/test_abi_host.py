"""C ABI checks that need no GPU: the library loads, exports every entry point
declared in include/hils.h, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from chunk_wise_sparse_b200 import hils

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hils.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hils_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from chunk_wise_sparse_b200 import build
    build.build()
    return hils.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(hils.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n


def dims(**kw):
    base = dict(batch=1, heads_q=2, heads_kv=1, head_dim=64, seqlen=1024, topk=4, dtype=hils.BF16)
    base.update(kw)
    return hils.make_dims(base["batch"], base["heads_q"], base["heads_kv"], base["head_dim"], base["seqlen"],
                          base["topk"], base["dtype"], base.get("chunk", 64), base.get("window", 0))


def test_sizes(lib):
    d = dims(batch=2, heads_q=8, heads_kv=2, head_dim=128, seqlen=4096, topk=8)
    assert hils.hils_kprime_mma_bytes(d) == 2 * 2 * 64 * (128 + 16) * 2
    assert hils.hils_decode_workspace_bytes(d) > 2 * 8 * 64 * 4
    assert hils.hils_kprime_mma_bytes(dims(chunk=32)) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(chunk=32), 2), (dict(head_dim=96), 2), (dict(topk=0), 2), (dict(topk=65), 2),
    (dict(seqlen=1000), 1), (dict(heads_q=3, heads_kv=2), 1), (dict(dtype=7), 1), (dict(batch=0), 1),
    (dict(window=100), 1), (dict(window=-64), 1), (dict(window=17 * 64), 2),
])
def test_bad_dims_rejected_before_launch(lib, kw, code):
    d = dims(**kw)
    p = ctypes.c_void_p(256)     # never dereferenced: validation fails first
    rc = lib.hils_select(ctypes.byref(d), p, p, p, p, None, 0, p, None, None)
    assert rc == code
    rc = lib.hils_attn_prefill(ctypes.byref(d), p, p, p, p, p, p, p, p, p, None, None, 0, None)
    assert rc == code


def test_null_and_misaligned_pointers_rejected(lib):
    d = dims()
    p, bad = ctypes.c_void_p(256), ctypes.c_void_p(258)
    assert lib.hils_select(ctypes.byref(d), None, p, p, p, None, 0, p, None, None) == 1
    assert lib.hils_select(ctypes.byref(d), bad, p, p, p, None, 0, p, None, None) == 1
    assert lib.hils_select(ctypes.byref(d), p, p, p, None, None, 0, p, None, None) == 1   # bf16 needs the MMA operand
    assert lib.hils_landmark_summary(ctypes.byref(d), p, p, 0, 17, p, p, None, None) == 1   # range past nc
    assert lib.hils_landmark_summary(ctypes.byref(d), p, p, 3, 3, p, p, None, None) == 0    # empty range
    small = hils.hils_decode_workspace_bytes(d) - 1
    assert lib.hils_attn_decode(ctypes.byref(d), p, p, p, None, None, p, p, p, None, None, p, small, None) == 4
    assert lib.hils_get_status(None, None) == 1
    assert lib.hils_selftest_bounded_wait(0, None) == 1
    assert lib.hils_selftest_bounded_wait(5000, None) == 1
    # bf16 prefill needs its workspace
    need = hils.hils_prefill_workspace_bytes(d)
    assert need > 0
    assert lib.hils_attn_prefill(ctypes.byref(d), p, p, p, None, None, None, p, p, p, None, p, need - 1, None) == 4
    assert hils.hils_prefill_workspace_bytes(dims(dtype=hils.FP32)) == 0


def test_select_row_subset_arguments(lib):
    """A listed row subset (row_pos) needs a 16-byte aligned list; without a
    list n_rows must be 0 or seqlen; an empty list launches nothing."""
    d = dims()
    p, bad = ctypes.c_void_p(256), ctypes.c_void_p(264)
    assert lib.hils_select(ctypes.byref(d), p, p, p, p, None, 7, p, None, None) == 1          # n_rows without a list
    assert lib.hils_select(ctypes.byref(d), p, p, p, p, None, d.seqlen + 64, p, None, None) == 1
    assert lib.hils_select(ctypes.byref(d), p, p, p, p, p, -1, p, None, None) == 1            # negative count
    assert lib.hils_select(ctypes.byref(d), p, p, p, p, bad, 4, p, None, None) == 1           # misaligned list
    before = hils.hils_kernel_launches()
    assert lib.hils_select(ctypes.byref(d), p, p, p, p, p, 0, p, None, None) == 0             # empty list: no work
    assert hils.hils_kernel_launches() == before


def test_prefill_without_scores_needs_the_summaries(lib):
    """scores NULL makes the prefill recompute the chunk scores: bf16 then needs
    the scoring operand, fp32 needs k' and b' (refused before any launch)."""
    p = ctypes.c_void_p(256)
    d = dims()
    need = hils.hils_prefill_workspace_bytes(d)
    assert lib.hils_attn_prefill(ctypes.byref(d), p, p, p, p, p, None, p, None, p, None, p, need, None) == 1
    d32 = dims(dtype=hils.FP32)
    assert lib.hils_attn_prefill(ctypes.byref(d32), p, p, p, None, p, p, p, None, p, None, None, 0, None) == 1
    assert lib.hils_attn_prefill(ctypes.byref(d32), p, p, p, p, None, p, p, None, p, None, None, 0, None) == 1
    # misaligned scores are refused too
    assert lib.hils_attn_prefill(ctypes.byref(d), p, p, p, p, p, p, p, ctypes.c_void_p(260), p, None, p, need,
                                 None) == 1


def test_decode_rejects_more_than_32_query_heads_per_kv_head(lib):
    d = dims(heads_q=64, heads_kv=1)
    p = ctypes.c_void_p(256)     # never dereferenced: validation fails first
    big = hils.hils_decode_workspace_bytes(d)
    assert lib.hils_attn_decode(ctypes.byref(d), p, p, p, None, None, p, p, p, None, None, p, big, None) == 2
    assert lib.hils_attn_decode_fixed_scratch(ctypes.byref(d), p, p, p, None, None, p, p, p, None, None, None) == 2


def test_window_sizes(lib):
    """The window leaves the prefill workspace unchanged and gives the decode
    one partial slot per window chunk."""
    assert hils.hils_prefill_workspace_bytes(dims(window=64)) == hils.hils_prefill_workspace_bytes(dims())
    assert hils.hils_prefill_workspace_bytes(dims(window=512)) == hils.hils_prefill_workspace_bytes(dims())
    d0, d8 = dims(window=0), dims(window=512)
    assert hils.hils_decode_workspace_bytes(d8) > hils.hils_decode_workspace_bytes(d0)
    d16 = dims(window=1024)
    assert lib.hils_select(ctypes.byref(d16), None, None, None, None, None, 0, None, None, None) == 1   # dims pass, q NULL


def test_qcal_arguments_rejected_before_launch(lib):
    d = dims()
    p, q2 = ctypes.c_void_p(256), ctypes.c_void_p(512)
    for rank in (0, 7, 12, 72):
        assert lib.hils_query_calibrate(ctypes.byref(d), p, 64, p, p, rank, q2, None) == 1
    assert lib.hils_query_calibrate(ctypes.byref(d), p, 0, p, p, 16, q2, None) == 1        # no positions
    assert lib.hils_query_calibrate(ctypes.byref(d), p, 64, p, p, 16, ctypes.c_void_p(272), None) == 1  # overlap
    assert lib.hils_query_calibrate(ctypes.byref(d), p, 64, None, p, 16, q2, None) == 1
    big = hils.hils_decode_workspace_bytes(d)
    assert lib.hils_attn_decode_qcal(ctypes.byref(d), p, None, p, p, None, 0, None, None, p, p, p, None, None, p,
                                     big, None) == 1      # no scoring query
    assert lib.hils_attn_decode_qcal(ctypes.byref(d), p, p, p, p, p, 0, None, None, p, p, p, None, None, p,
                                     big, None) == 1      # a page table needs pages


def test_backward_arguments_rejected_before_launch(lib):
    d = dims()
    p = ctypes.c_void_p(256)
    need = hils.hils_attn_backward_workspace_bytes(d)
    assert need > 0
    args = [p] * 11
    # q_score and dq_score may be NULL; every other pointer is required
    assert lib.hils_attn_backward(ctypes.byref(d), p, None, p, p, p, p, p, p, None, p, p, p, None, p, p, p, p,
                                  need, None) == 1
    assert lib.hils_attn_backward(ctypes.byref(d), p, None, p, p, p, p, p, p, p, p, p, p, None, p, p, p, p,
                                  need - 1, None) == 4


def test_strerror(lib):
    for code in range(7):
        assert len(hils.strerror(code)) >= 2
    assert hils.strerror(99) == "unknown status"


def test_host_tensors_are_refused_by_the_binding(lib):
    """Every buffer of the ABI is device memory: the binding refuses a host
    tensor before the library is called (no launch, no host fallback)."""
    import torch
    d = dims()
    q = torch.zeros((1, 2, 1024, 64), dtype=torch.bfloat16)
    ids = torch.zeros((1, 2, 1024, 4), dtype=torch.int32)
    before = hils.hils_kernel_launches()
    with pytest.raises(ValueError, match="CUDA tensor"):
        hils.hils_select(d, q, None, None, q, None, 0, ids)
    with pytest.raises(ValueError, match="CUDA tensor"):
        hils.hils_landmark_summary(d, q, q, 0, 16, ids, ids)
    assert hils.hils_kernel_launches() == before


def test_empty_summary_range_launches_nothing(lib):
    """[c, c) is a valid range with no chunk: the call succeeds and launches
    no kernel (the pointers, 16-byte aligned, are never touched)."""
    d = dims()
    fake = 1 << 20
    before = hils.hils_kernel_launches()
    hils.hils_landmark_summary(d, fake, fake, 5, 5, fake, fake, fake, stream=0)
    assert hils.hils_kernel_launches() == before
    with pytest.raises(hils.HilsError):
        hils.hils_landmark_summary(d, fake, fake, 6, 5, fake, fake, fake, stream=0)
