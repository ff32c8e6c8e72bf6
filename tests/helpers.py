"""Shared helpers of the GPU tests: device copies of generated inputs and the
acceptance rules (tolerances written here, used by every parity test)."""
import numpy as np
import torch

# Acceptance: selection exact where the oracle's K-th/(K+1)-th gap is at least
# SEL_GAP; outputs within max-abs / mean-abs; summaries within SUMMARY_TOL.
SEL_GAP = {"fp32": 1e-3, "bf16": 2e-2}
OUT_MAX = {"fp32": 1e-5, "bf16": 2e-2}
OUT_MEAN = {"fp32": 1e-5, "bf16": 2e-3}
SUMMARY_TOL = 1e-5


def to_dev(inp, name, device="cuda"):
    """Device tensor of a generated input (bf16 bit patterns or fp32 values)."""
    bits = getattr(inp, name + "_bits")
    if bits is not None:
        return torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(getattr(inp, name + "_f32")).to(device)


def gather_rows(t, flat):
    """Rows (b, hq, i) of a [B,Hq,N,X] tensor as a [n, X] numpy array."""
    B, Hq, N = t.shape[:3]
    idx = torch.from_numpy(np.asarray(flat, np.int64)).to(t.device)
    return t.reshape(B * Hq * N, -1)[idx].float().cpu().numpy()


def check_selection(ids_gpu, oracle_ids, gap, scores_oracle_all, thr, eps):
    """Exact id sets on rows with gap >= thr; validity on every row:
    min over kept oracle scores >= max over dropped oracle scores - eps.
    Returns (graded rows, total rows, valid rows)."""
    n = len(ids_gpu)
    graded = gap >= thr
    for r in np.nonzero(graded)[0]:
        assert np.array_equal(np.sort(ids_gpu[r]), np.sort(oracle_ids[r])), \
            f"row {r}: ids {ids_gpu[r]} vs oracle {oracle_ids[r]} (gap {gap[r]})"
    n_valid = 0
    for r in range(n):
        kept = ids_gpu[r][ids_gpu[r] >= 0]
        s = scores_oracle_all[r]
        cand = np.isfinite(s)
        assert len(kept) == min(cand.sum(), ids_gpu.shape[1]), f"row {r}: {len(kept)} ids kept"
        assert len(np.unique(kept)) == len(kept) and np.all(cand[kept]), f"row {r}: invalid ids {kept}"
        if len(kept) == cand.sum():
            n_valid += 1
            continue
        dropped = np.ones_like(cand)
        dropped[kept] = False
        dropped &= cand
        ok = s[kept].min() >= s[dropped].max() - eps
        assert ok, f"row {r}: kept min {s[kept].min()} < dropped max {s[dropped].max()} - {eps}"
        n_valid += 1
    return int(graded.sum()), n, n_valid
