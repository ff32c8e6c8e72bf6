"""Splitting one HiLS problem across GPUs (one process per GPU).

The (batch, kv head) groups of a prefill are independent: a group's landmark
summaries, its chunk selection and its sparse attention read only that
group's keys, values, landmark queries and the queries of the G query heads
that share its kv head.  The sequences of a decode batch are independent the
same way.  So rank r of N takes a contiguous range of groups (prefill) or of
sequences (decode) and runs the same C ABI calls on its slice; nothing crosses
GPUs on the hot path.  Gathering the output onto every rank is a separate,
optional step (``gather_rows``), for a caller that wants the whole O on one
device.

Host logic only: which units a rank owns and how a slice maps onto the
row-major [B, H, ...] tensors.  No arithmetic of the method lives here.
"""
from __future__ import annotations

import dataclasses


def unit_range(n_units: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi): rank's contiguous share of n_units, balanced (sizes differ by
    at most one; the first n_units % world ranks take the larger share)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


@dataclasses.dataclass(frozen=True)
class HeadSlice:
    """kv heads [h_lo, h_hi) of batch element b, i.e. query heads
    [h_lo * G, h_hi * G): contiguous in every [B, H, ...] tensor."""
    b: int
    h_lo: int
    h_hi: int

    @property
    def heads_kv(self) -> int:
        return self.h_hi - self.h_lo


def prefill_slices(B: int, Hkv: int, world: int, rank: int) -> list[HeadSlice]:
    """The (b, kv head) groups of rank as runs of consecutive kv heads within
    one batch element (a range of the flattened b * Hkv + h index can span
    several batch elements)."""
    lo, hi = unit_range(B * Hkv, world, rank)
    out = []
    u = lo
    while u < hi:
        b, h = divmod(u, Hkv)
        h_hi = min(Hkv, h + (hi - u))
        out.append(HeadSlice(b, h, h_hi))
        u += h_hi - h
    return out


def decode_slice(B: int, world: int, rank: int) -> tuple[int, int]:
    """[b_lo, b_hi): the sequences of a decode batch that rank owns."""
    return unit_range(B, world, rank)


def slice_heads(t, s: HeadSlice, G: int = 1):
    """The part of a [B, H, ...] tensor that slice s covers: kv-head tensors
    with G = 1, query-head tensors with the group size G (a view)."""
    return t[s.b:s.b + 1, s.h_lo * G:s.h_hi * G]


def gather_rows(local, world: int, n_units_total: int, unit_of_rank, device=None):
    """Optional all-gather of per-rank outputs onto every rank.

    local is this rank's output as a [n_units, ...] tensor (its units in
    order); unit_of_rank(r) -> (lo, hi) gives every rank's unit range.  The
    result is the [n_units_total, ...] tensor of all ranks' units in order.
    Uses torch.distributed (NCCL between GPUs, gloo on CPU); shares are padded
    to the largest one so every rank sends the same number of elements."""
    import torch
    import torch.distributed as dist
    sizes = [unit_of_rank(r)[1] - unit_of_rank(r)[0] for r in range(world)]
    m = max(sizes)
    pad = torch.zeros((m,) + tuple(local.shape[1:]), dtype=local.dtype, device=device or local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    out = torch.cat([p[:sizes[r]] for r, p in enumerate(parts)], dim=0)
    assert out.shape[0] == n_units_total
    return out
