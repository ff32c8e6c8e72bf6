"""Benchmark of the HiLS attention forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole path over one batch of synthetic input
already resident in HBM: landmark summary (a) -> chunk scoring + top-K (b) ->
sparse prefill attention with fusion (c) -> one decode step at full length
(d).  Prints ONE JSON line (rank 0).  The default run also times, in the same
process, the batch-8 GQA decode step and the 7B-shaped GQA prefill (the line's
"extra").  For N > 1 (torchrun) the ranks split one problem: rank r takes a
contiguous range of (batch, kv head) groups of a prefill, or of the sequences
of a decode batch (chunk_wise_sparse_b200/partition.py), and runs the same C
ABI calls on its slice; no collective runs on the data path (strong scaling:
the job is the whole workload, its time the max over ranks).

--impl reference times the fp64 CPU oracle (the reference arm of this
method: there is no other implementation to run) on a bounded sample of the
same workload.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from chunk_wise_sparse_b200.inputs import WORKLOADS, generate, sample_rows  # noqa: E402

DEFAULT_WORKLOAD = "prefill-512k-h16-d64"
METRIC = "HiLS prefill tokens/s (landmark summary + top-K selection + sparse attention, with one decode step)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=j["hbm_gbs"], bf16_tflops=j["bf16_tflops"],
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained", j["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# The sources each recorded kernel is compiled from.
KERNEL_SOURCES = {"select": ["select_tc.cuh", "sm100.cuh", "common.cuh"],
                  "decode": ["decode.cuh", "attend_simt.cuh", "common.cuh"]}


def code_only(text):
    """C/CUDA source without its comments and blank space: what the compiler sees."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernels_sha256(kernel):
    """Hash of a kernel's CUDA sources (code only, comments ignored), to tell
    whether recorded counters still apply."""
    h = hashlib.sha256()
    src = os.path.join(ROOT, "chunk_wise_sparse_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        h.update(name.encode())
        with open(os.path.join(src, name), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()


def recorded_traffic(kernel, rows):
    """DRAM bytes per launch of `kernel` from the committed ncu record (per
    query row, scaled to `rows`), or None when there is none or the kernel
    sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    if kernel not in j.get("per_row_bytes", {}) or j.get("sources_sha256", {}).get(kernel) != kernels_sha256(kernel):
        return None
    return float(j["per_row_bytes"][kernel]) * rows


def recorded_step_traffic(kernel, workload):
    """DRAM bytes per step of `kernel` (all its launches in one step) on
    `workload` from the committed ncu record, or None when there is none or
    the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    key = f"{kernel}:{workload}"
    if key not in j.get("per_step_bytes", {}) or j.get("sources_sha256", {}).get(kernel) != kernels_sha256(kernel):
        return None
    return float(j["per_step_bytes"][key])


def useful_work(w):
    """Algorithmic work of one step: 2d FLOPs per (row, candidate chunk) for
    the scoring, 4d per (row, attended key) for the attention, and the bytes
    the summary must move (keys, landmark queries in; k', b' and the scoring
    operand out)."""
    B, Hq, Hkv, N, d, C, K = w.B, w.Hq, w.Hkv, w.N, w.d, w.C, w.K
    nc = N // C
    wc = max(1, w.window // C)                      # chunks of the local window
    i = np.arange(N, dtype=np.int64)
    own = i // C
    n_cand = np.maximum(0, own - (wc - 1))          # candidate chunks of each row
    keys = np.minimum(K, n_cand) * C + (i - n_cand * C) + 1
    flops_score = 2 * d * Hq * B * C * int(np.maximum(0, np.arange(nc) - (wc - 1)).sum())
    flops_attn = 4 * d * Hq * B * int(keys.sum())
    bytes_summary = B * Hkv * nc * (C * d * 2 + d * 2 + 4 * d + 4 + 2 * (d + 16))
    return dict(flops_score=flops_score, flops_attn=flops_attn, bytes_summary=bytes_summary)


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""
    FIELDS = "clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, index):
        self.index, self.proc, self.out = index, None, None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for _, _, r in rows for k, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def cpu_oracle_sample(w, inp, budget_s=15.0, info=None):
    """Time the fp64 oracle (as it stands) on a bounded sample of the workload:
    the summaries of a head subset plus sampled prefill rows.  Returns
    (tokens/s, description, threads); `info` (a dict) gets the rows and the
    seconds the sample took."""
    from oracle.oracle import Oracle, Rows, max_threads, qcal
    o = Oracle.for_workload(w)
    if w.qcal:
        from chunk_wise_sparse_b200.inputs import qcal_weights
        wt = qcal_weights(w.Hq, w.d, w.qcal, seed=w.seed, dtype=w.dtype)
    # summaries: all chunks of one (b, kv head)
    one = Oracle(1, w.G, 1, w.N, w.d, w.C, w.K, w.window)
    t0 = time.perf_counter()
    kp1, bp1 = one.summary(inp.k_f32[:1, :1], inp.lq_f32[:1, :1])
    t_sum_head = time.perf_counter() - t0
    t_summary = t_sum_head * w.B * w.Hkv
    kp = np.zeros((w.B, w.Hkv, w.nc, w.d))
    bp = np.zeros((w.B, w.Hkv, w.nc))
    kp[0, 0], bp[0, 0] = kp1[0, 0], bp1[0, 0]
    # rows of head 0 spread over the sequence
    n = 64
    elapsed, done = 0.0, 0
    rng = np.random.default_rng(w.seed + 2000)
    while elapsed < budget_s and done < w.N:
        pos = np.sort(rng.choice(w.N, size=n, replace=False))
        rows = Rows(np.zeros(n), np.zeros(n), pos, inp.q_f32[0, 0, pos] if w.kind != "decode" else
                    np.repeat(inp.q_f32[:1, 0], n, axis=0))
        t0 = time.perf_counter()
        if w.qcal:
            qs = qcal(rows.q, rows.hq, wt.w_down_f32, wt.w_up_f32).astype(np.float32)
            ids, _, _ = o.select(kp, bp, Rows(rows.b, rows.hq, rows.pos, qs))
            o.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids, qscore=qs)
        else:
            ids, _, _ = o.select(kp, bp, rows)
            o.attend(inp.k_f32, inp.v_f32, kp, bp, rows, ids)
        elapsed += time.perf_counter() - t0
        done += n
        n = min(2 * n, 4096)
    t_per_row = elapsed / done
    t_token = t_summary / w.N + t_per_row * w.Hq * w.B
    if info is not None:
        info.update(rows=done, row_seconds=elapsed, summary_seconds=t_sum_head)
    desc = (f"fp64 oracle: summaries of 1 of {w.B * w.Hkv} (b, kv head) slabs ({t_sum_head:.2f} s, scaled), "
            f"select+attend of {done} sampled rows of head 0 ({elapsed:.1f} s); tokens/s = 1 / (summary "
            f"time per token + row time x {w.B * w.Hq} rows per token)")
    return 1.0 / t_token, desc, max_threads()


def cpu_oracle_decode(w, inp, budget_s=15.0):
    """Time the fp64 oracle (as it stands) on the decode step of the workload.
    The landmark summaries are setup, untimed, as on the GPU side; the timed
    part is the decode step (scores, top-K, sparse attention) of one sequence
    with all its query heads, repeated for about `budget_s` seconds and scaled
    to the batch (the sequences are independent and equally long).  Returns
    (us/step, description, threads)."""
    from oracle.oracle import Oracle, max_threads
    one = Oracle(1, w.Hq, w.Hkv, w.N, w.d, w.C, w.K, w.window)
    kp, bp = one.summary(inp.k_f32[:1], inp.lq_f32[:1])
    q, kc, vc = inp.q_f32[:1], np.ascontiguousarray(inp.k_f32[:1]), np.ascontiguousarray(inp.v_f32[:1])
    seq = np.array([w.N], np.int32)
    reps, elapsed = 0, 0.0
    while reps == 0 or elapsed < budget_s:
        t0 = time.perf_counter()
        one.decode(q, kc, vc, kp, bp, seq)
        elapsed += time.perf_counter() - t0
        reps += 1
    us = elapsed / reps * w.B * 1e6
    desc = (f"fp64 oracle: the decode step of 1 of {w.B} sequences (all {w.Hq} query heads, {w.N} cached "
            f"tokens), {reps} repetitions in {elapsed:.1f} s, scaled to the batch; summaries built beforehand, "
            f"untimed" + ("; contiguous cache (paging changes only the addresses)" if w.paged else ""))
    return us, desc, max_threads()


def cpu_oracle_backward(w, inp):
    """Time the fp64 oracle (as it stands) on the backward of one (b, kv head)
    slab of the workload -- its G query heads, every row -- for the oracle's
    own selection (setup, untimed) and a seeded output gradient, scaled to the
    B x Hkv independent slabs.  Returns (tokens/s, description, threads)."""
    from oracle.oracle import Oracle, Rows, max_threads
    # a causal prefix of at most 32K tokens is a whole problem of its own;
    # past the first chunks a row's cost does not grow with its position
    n = min(w.N, 32768)
    one = Oracle(1, w.G, 1, n, w.d, w.C, w.K, w.window)
    Q, Kt, Vt, LQ = (np.ascontiguousarray(a[:1, :w.G, :rows] if name == "q" else a[:1, :1, :rows])
                     for name, a, rows in (("q", inp.q_f32, n), ("k", inp.k_f32, n), ("v", inp.v_f32, n),
                                           ("lq", inp.lq_f32, n // w.C)))
    kp, bp = one.summary(Kt, LQ)
    ids, _, _ = one.select(kp, bp, Rows.from_prefill(Q, np.arange(w.G * n)))
    dO = np.random.default_rng(w.seed + 3000).standard_normal(Q.shape).astype(np.float32)
    t0 = time.perf_counter()
    one.backward(Q, Kt, Vt, LQ, ids.reshape(1, w.G, n, w.K), dO)
    t_slab = time.perf_counter() - t0
    tokens_per_s = n / (t_slab * w.Hkv)   # B*N tokens over B*Hkv slabs of N/n such prefixes each
    desc = (f"fp64 oracle: backward of the first {n} tokens of 1 of {w.B * w.Hkv} (b, kv head) slabs "
            f"({w.G} query heads) in {t_slab:.1f} s, scaled to the whole job; selection and summaries "
            f"beforehand, untimed")
    return tokens_per_s, desc, max_threads()


def run_reference(args, w, rank):
    """The reference arm: the fp64 oracle as it stands, on the host cores, each
    step a bounded sample of the workload (about --ref-budget seconds of rows),
    extrapolated to the whole workload for `value`.  steps / ms_per_step are
    the sample steps actually run and their wall time."""
    if rank != 0:
        return
    inp = generate(w)
    for _ in range(args.warmup):
        cpu_oracle_sample(w, inp, budget_s=2.0)
    vals, walls, infos = [], [], []
    for _ in range(args.steps):
        info = {}
        t0 = time.perf_counter()
        v, desc, threads = cpu_oracle_sample(w, inp, budget_s=args.ref_budget, info=info)
        walls.append(time.perf_counter() - t0)
        vals.append(v)
        infos.append(info)
    value = float(np.mean(vals))
    ms_step = 1e3 * float(np.mean(walls))
    full_ms = 1e3 * w.B * w.N / value          # the whole workload at the sampled rate
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args.gpus),
            "extrapolated": True,
            "extrapolation": {"sampled_rows_per_step": int(np.mean([i["rows"] for i in infos])),
                              "sampled_row_seconds_per_step": float(np.mean([i["row_seconds"] for i in infos])),
                              "workload_ms_at_sampled_rate": full_ms, "scale_factor": full_ms / ms_step,
                              "note": "each step times a bounded sample; value is the sampled rate applied to "
                                      "the whole workload"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own tokens_per_rank per step."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


L2_BYTES = 126 << 20


def inputs_exceed_l2(w):
    """Q, K and V each larger than the 126 MB L2 (else the bench flushes L2)."""
    eb = 2 if w.dtype == "bf16" else 4
    q_rows = w.B * w.Hq * (1 if w.kind == "decode" else w.N)
    return min(q_rows * w.d * eb, w.B * w.Hkv * w.N * w.d * eb) > L2_BYTES or \
        (w.kind == "decode" and w.B * w.Hkv * w.N * w.d * eb > L2_BYTES)


def workload_config(w, n_gpus):
    l2 = ("inputs larger than L2 (K and V caches each larger than 126 MB); no flush" if w.kind == "decode" else
          "inputs larger than L2 (Q, K, V are each larger than 126 MB); no flush") if inputs_exceed_l2(w) else \
        "inputs smaller than L2: a 256 MB buffer is written before every step, outside the kernel events, " \
        "and ms_per_step is the sum of the kernel events"
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "N": w.N, "C": w.C, "K": w.K,
            "window": w.window, "qcal_rank": w.qcal, "needles": w.needles, "seed": w.seed,
            "parallelism": ("1 GPU" if n_gpus == 1 else
                            f"{n_gpus} GPUs, one problem split by " +
                            ("sequence" if w.kind == "decode" else "(batch, kv head) group") +
                            ", no collective on the data path"), "l2": l2}


def rank_slices(w, world, rank):
    """The sub-problems rank runs: its (b, kv head) groups of a prefill as
    runs of consecutive kv heads (each one independent problem of batch 1),
    or its sequences of a decode batch.  One rank: the whole workload."""
    from chunk_wise_sparse_b200.partition import decode_slice, prefill_slices
    if world == 1:
        return [None]
    if w.kind == "decode":
        b_lo, b_hi = decode_slice(w.B, world, rank)
        return [("b", b_lo, b_hi)] if b_hi > b_lo else []
    return [("h", s.b, s.h_lo, s.h_hi) for s in prefill_slices(w.B, w.Hkv, world, rank)]


def slice_inputs(w, inp, sl):
    """(workload, inputs) of one sub-problem of rank_slices: views of the host
    arrays of the groups or sequences it covers (no arithmetic)."""
    import dataclasses
    from chunk_wise_sparse_b200.inputs import Inputs
    if sl is None:
        return w, inp
    if sl[0] == "b":
        _, b0, b1 = sl
        cut = {n: lambda a, b0=b0, b1=b1: None if a is None else a[b0:b1] for n in ("q", "k", "v", "lq")}
        ws = dataclasses.replace(w, B=b1 - b0)
    else:
        _, b, h0, h1 = sl
        G = w.G
        cut = {"q": lambda a: None if a is None else a[b:b + 1, h0 * G:h1 * G]}
        for n in ("k", "v", "lq"):
            cut[n] = lambda a: None if a is None else a[b:b + 1, h0:h1]
        ws = dataclasses.replace(w, B=1, Hq=(h1 - h0) * G, Hkv=h1 - h0)
    kw = {}
    for n in ("q", "k", "v", "lq"):
        kw[n + "_f32"] = np.ascontiguousarray(cut[n](getattr(inp, n + "_f32")))
        bits = getattr(inp, n + "_bits")
        kw[n + "_bits"] = None if bits is None else np.ascontiguousarray(cut[n](bits))
    return ws, Inputs(ws, kw["q_f32"], kw["k_f32"], kw["v_f32"], kw["lq_f32"], inp.needle_chunks, inp.needle_blocks,
                      kw["q_bits"], kw["k_bits"], kw["v_bits"], kw["lq_bits"])


class PrefillSlice:
    """Device buffers and C ABI calls of one prefill sub-problem (the whole
    workload on one rank, or a rank's run of (b, kv head) groups)."""

    def __init__(self, w, inp, dev, hils):
        import torch
        self.w, self.inp, self.dev, self.h = w, inp, dev, hils
        self.q, self.k, self.v, self.lq = (self.to_dev(n) for n in ("q", "k", "v", "lq"))
        B, Hq, Hkv, N, d, K = w.B, w.Hq, w.Hkv, w.N, w.d, w.K
        self.dims = hils.dims_for(self.q, self.k, K, w.window)
        self.summ = hils.Summary(self.dims, dev)
        self.ids = torch.empty((B, Hq, N, K), dtype=torch.int32, device=dev)
        self.scores = torch.empty((B, Hq, N, K), dtype=torch.float32, device=dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        self.qd = self.q[:, :, -1, :].contiguous()
        self.seq = torch.full((B,), N, dtype=torch.int32, device=dev)
        self.ddims = hils.make_dims(B, Hq, Hkv, d, N, K, self.q.dtype, window=w.window)
        self.ws = torch.empty((hils.hils_decode_workspace_bytes(self.ddims),), dtype=torch.uint8, device=dev)
        self.pws = hils.prefill_workspace(self.dims, dev)
        self.od = torch.empty_like(self.qd)
        self.ids_d = torch.empty((B, Hq, K), dtype=torch.int32, device=dev)
        self.sc_d = torch.empty((B, Hq, K), dtype=torch.float32, device=dev)
        self.use_qcal = w.qcal > 0
        if self.use_qcal:
            # Q-Cal projections (random init, resident like model weights); the
            # prefill scores with q^, the decode step with the calibrated last row
            from chunk_wise_sparse_b200.inputs import qcal_weights
            wt = qcal_weights(Hq, d, w.qcal, seed=w.seed, dtype=w.dtype)
            if wt.w_down_bits is not None:
                self.wd = torch.from_numpy(wt.w_down_bits.view(np.int16)).to(dev).view(torch.bfloat16)
                self.wu = torch.from_numpy(wt.w_up_bits.view(np.int16)).to(dev).view(torch.bfloat16)
            else:
                self.wd, self.wu = torch.from_numpy(wt.w_down_f32).to(dev), torch.from_numpy(wt.w_up_f32).to(dev)
            self.q_hat, self.qd_hat = torch.empty_like(self.q), torch.empty_like(self.qd)
            self.cdims = hils.make_dims(B, Hq, Hq, d, 64, 1, self.q.dtype)
        self.cur = {"q": self.q, "k": self.k, "v": self.v, "lq": self.lq, "qd": self.qd}

    def to_dev(self, name):
        import torch
        bits = getattr(self.inp, name + "_bits")
        if bits is not None:
            return torch.from_numpy(bits.view(np.int16)).to(self.dev).view(torch.bfloat16)
        return torch.from_numpy(getattr(self.inp, name + "_f32")).to(self.dev)

    # the phases of one step, each one C ABI call (two for Q-Cal)
    def summary(self, st):
        t = self.cur
        self.h.hils_landmark_summary(self.dims, t["k"], t["lq"], 0, self.w.N // 64, self.summ.kprime,
                                     self.summ.bprime, self.summ.kprime_mma, st)

    def qcal(self, st):
        t = self.cur
        self.h.hils_query_calibrate(self.cdims, t["q"], self.w.N, self.wd, self.wu, self.w.qcal, self.q_hat, st)
        self.h.hils_query_calibrate(self.cdims, t["qd"], 1, self.wd, self.wu, self.w.qcal, self.qd_hat, st)

    def select(self, st):
        t, s = self.cur, self.summ
        self.h.hils_select(self.dims, self.q_hat if self.use_qcal else t["q"], s.kprime, s.bprime, s.kprime_mma,
                           None, 0, self.ids, self.scores, st)

    def prefill(self, st):
        t, s = self.cur, self.summ
        self.h.hils_attn_prefill(self.dims, t["q"], t["k"], t["v"], s.kprime, s.bprime, s.kprime_mma, self.ids,
                                 self.scores, self.o, self.lse, self.pws, stream=st)

    def decode(self, st):
        t, s = self.cur, self.summ
        if self.use_qcal:
            self.h.hils_attn_decode_qcal(self.ddims, t["qd"], self.qd_hat, t["k"], t["v"], None, 0, s.kprime,
                                         s.bprime, s.kprime_mma, self.seq, self.od, self.ids_d, self.sc_d, self.ws,
                                         stream=st)
        else:
            self.h.hils_attn_decode(self.ddims, t["qd"], t["k"], t["v"], s.kprime, s.bprime, s.kprime_mma, self.seq,
                                    self.od, self.ids_d, self.sc_d, self.ws, stream=st)


def run_ours(args, w, rank, world, local_rank):
    """One prefill step (summary, [Q-Cal,] select, prefill, one decode step at
    full length) per iteration.  With N ranks, rank r runs the step on its own
    (b, kv head) groups only (partition.prefill_slices); the job is the whole
    workload, its time the max over ranks.  Returns the JSON line (rank 0)."""
    import torch
    import torch.distributed as dist
    from chunk_wise_sparse_b200 import hils

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hils.lib()
    inp = generate(w)
    parts = [PrefillSlice(*slice_inputs(w, inp, sl), dev, hils) for sl in rank_slices(w, world, rank)]
    B, Hq, Hkv, N, d, K = w.B, w.Hq, w.Hkv, w.N, w.d, w.K
    stream = torch.cuda.current_stream()
    flush = None if inputs_exceed_l2(w) else torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    use_qcal = w.qcal > 0
    names = ["summary"] + (["qcal"] if use_qcal else []) + ["select", "prefill", "decode"]
    n_ev = len(names) + 1

    def step(ev=None):
        if flush is not None:
            flush.fill_(1)
        if ev: ev[0].record(stream)
        for j, name in enumerate(names):
            for pt in parts:
                getattr(pt, name)(stream)
            if ev: ev[j + 1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hils.hils_get_status() != 0:
        raise RuntimeError("device status error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    launches0 = hils.hils_kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    launches = hils.hils_kernel_launches() - launches0
    clk = clocks.stop()
    status = hils.hils_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} ({hils.strerror(status)}) during the timed steps")
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(n_ev - 1)] for e in evs])   # ms per kernel
    ms_step = total_ms / args.steps
    if flush is not None:
        ms_step = max_over_ranks(float(per.sum(axis=1).mean()), world, dev)
    value = B * N / (ms_step / 1e3)    # the whole job's tokens, all ranks together

    # end to end through the public API: every step copies its inputs from
    # pinned host memory and reads its outputs back.  Two device input sets:
    # step i+1's inputs are copied (on a copy stream) while step i computes.
    e2e = None
    if not args.no_e2e:
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        h2d = d2h = 0
        for pt in parts:
            host = {n: getattr(pt.inp, n + "_bits") if getattr(pt.inp, n + "_bits") is not None else
                    getattr(pt.inp, n + "_f32") for n in ("q", "k", "v", "lq")}
            pt.pinned = {n: torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).pin_memory()
                         for n, a in host.items()}
            pt.sets = [{"q": pt.q, "k": pt.k, "v": pt.v, "lq": pt.lq, "qd": pt.qd},
                       {"q": torch.empty_like(pt.q), "k": torch.empty_like(pt.k), "v": torch.empty_like(pt.v),
                        "lq": torch.empty_like(pt.lq), "qd": torch.empty_like(pt.qd)}]
            pt.o_host = torch.empty(pt.o.shape, dtype=pt.o.dtype).pin_memory()
            pt.od_host = torch.empty(pt.od.shape, dtype=pt.od.dtype).pin_memory()
            h2d += sum(t.numel() * t.element_size() for t in pt.pinned.values())
            d2h += pt.o_host.numel() * pt.o_host.element_size() + pt.od_host.numel() * pt.od_host.element_size()

        def h2d_into(k):
            for pt in parts:
                for n, src in pt.pinned.items():
                    t = pt.sets[k][n]
                    t.view(torch.int16 if t.dtype == torch.bfloat16 else t.dtype).copy_(src, non_blocking=True)

        def run_e2e(n_steps):
            for ev in done:
                ev.record(stream)
            copy_stream.wait_stream(stream)
            with torch.cuda.stream(copy_stream):
                h2d_into(0)
                copied[0].record(copy_stream)
            for i in range(n_steps):
                cur, nxt = i % 2, (i + 1) % 2
                if i + 1 < n_steps:
                    copy_stream.wait_event(done[nxt])   # the step that last read set nxt is done
                    with torch.cuda.stream(copy_stream):
                        h2d_into(nxt)
                        copied[nxt].record(copy_stream)
                stream.wait_event(copied[cur])
                for pt in parts:
                    pt.cur = pt.sets[cur]
                    pt.cur["qd"].copy_(pt.cur["q"][:, :, -1, :])   # the decode query is the step's last prefill row
                step()
                for pt in parts:
                    pt.o_host.copy_(pt.o, non_blocking=True)
                    pt.od_host.copy_(pt.od, non_blocking=True)
                done[cur].record(stream)
            for pt in parts:
                pt.cur = pt.sets[0]

        run_e2e(2)
        torch.cuda.synchronize()
        n_e2e = max(2, min(args.steps, 8))
        if world > 1:
            dist.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        run_e2e(n_e2e)
        a1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a0.elapsed_time(a1) / n_e2e, world, dev)
        e2e = {"value": B * N / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "overlap": "step i+1's host-to-device copies run on a copy stream during step i"}
        if world > 1:
            e2e["bytes_note"] = "h2d / d2h bytes of rank 0's slice"
    if rank != 0:
        return None

    # the work and the kernel fractions are those of rank 0's share of the job
    w0 = parts[0].w if len(parts) == 1 else w
    work = useful_work(w0)
    if len(parts) > 1:
        work = {key: sum(useful_work(pt.w)[key] for pt in parts) for key in work}
    peaks = load_peaks()
    avg = per.mean(axis=0)
    kernels_ms = {n: float(a) for n, a in zip(names, avg)}
    dom = names[int(np.argmax(avg))]
    rows0 = sum(pt.w.B * pt.w.Hq * N for pt in parts)
    if dom in ("select", "prefill"):
        fl = work["flops_score"] if dom == "select" else work["flops_attn"]
        ach = fl / (kernels_ms[dom] / 1e3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                "traffic": recorded_traffic(dom, rows0),
                "peak_source": peaks["source"] + " bf16 dense burst"}
    else:
        by = work["bytes_summary"]
        ach = by / (kernels_ms[dom] / 1e3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": None, "peak_source": peaks["source"] + " copy"}
    bc_flops = work["flops_score"] + work["flops_attn"]
    bc_ms = kernels_ms["select"] + kernels_ms["prefill"]
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp32",
        "data": f"synthetic: i.i.d. N(0,1) Q/K/V/landmark queries, {w.needles} planted needle chunks, seed {w.seed}",
        "config": workload_config(w, world),
        "kernels_ms": kernels_ms,
        "kernels_ms_per_step": per.round(4).tolist(),
        "decode_us_per_step": 1e3 * kernels_ms["decode"],
        "prefill_bc_tflops_useful": bc_flops / (bc_ms / 1e3) / 1e12,
        "prefill_bc_frac_of_bf16_peak": bc_flops / (bc_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
        "prefill_bc_frac_of_bf16_sustained": bc_flops / (bc_ms / 1e3) / 1e12 / peaks["bf16_tflops_sustained"],
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": clk,
        "e2e": e2e,
    }
    if world > 1:
        line["rank0_share"] = {"slices": [list(sl) for sl in rank_slices(w, world, 0)],
                               "note": "kernels_ms, roofline and the (b)+(c) fraction are rank 0's share"}
    if use_qcal:
        eb = 2 if w.dtype == "bf16" else 4
        qb = sum(2 * pt.w.B * pt.w.Hq * (N + 1) * d * eb for pt in parts)   # q read and q^ written
        line["qcal"] = {"rank": w.qcal, "ms": kernels_ms["qcal"], "bytes": qb,
                        "gbs": qb / (kernels_ms["qcal"] / 1e3) / 1e9,
                        "frac_of_hbm": qb / (kernels_ms["qcal"] / 1e3) / 1e9 / peaks["hbm_gbs"]}
    if not args.no_cpu_baseline and world == 1:
        v, desc, threads = cpu_oracle_sample(w, inp, budget_s=args.ref_budget)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc}
    return line


def decode_selected_bytes(ids, w):
    """Distinct K/V bytes a decode step must read at full length: per (b, kv
    head) the union of the G heads' kept chunks plus the local window's chunks,
    64 keys x d elements x (K, V)."""
    B, Hq, K = ids.shape
    n_win = min(max(1, w.window // w.C), w.N // w.C)
    elem = 2 if w.dtype == "bf16" else 4
    total = 0
    for b in range(B):
        for h in range(w.Hkv):
            sel = ids[b, h * w.G:(h + 1) * w.G].reshape(-1)
            n_union = len(np.unique(sel[sel >= 0])) + n_win
            total += n_union * w.C * w.d * elem * 2
    return total


def run_backward(args, w, rank, world, local_rank):
    """One backward step (gradients of q, k, v, lq for the forward's
    selection) per iteration, after one untimed forward."""
    import torch
    from chunk_wise_sparse_b200 import hils

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = generate(w)

    def to_dev(name):
        bits = getattr(inp, name + "_bits")
        if bits is not None:
            return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(getattr(inp, name + "_f32")).to(dev)

    q, k, v, lq = (to_dev(n) for n in ("q", "k", "v", "lq"))
    B, Hq, Hkv, N, d, K = w.B, w.Hq, w.Hkv, w.N, w.d, w.K
    o, aux = hils.prefill(q, k, v, lq, K, return_all=True, window=w.window)
    torch.cuda.synchronize()
    d_o = torch.randn(q.shape, device=dev, generator=torch.Generator(device=dev).manual_seed(w.seed)).to(q.dtype)
    dims = hils.dims_for(q, k, K, w.window)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk = torch.empty((B, Hq, N, d), **f32), torch.empty((B, Hkv, N, d), **f32)
    dv, dlq = torch.empty((B, Hkv, N, d), **f32), torch.empty((B, Hkv, N // 64, d), **f32)
    ws = torch.empty((hils.hils_attn_backward_workspace_bytes(dims),), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    flush = None if inputs_exceed_l2(w) else torch.empty((256 << 20,), dtype=torch.uint8, device=dev)

    def step():
        hils.hils_attn_backward(dims, q, None, k, v, lq, aux["summary"].kprime, aux["ids"], aux["scores"],
                                aux["lse_own"], o, d_o, dq, None, dk, dv, dlq, ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hils.hils_get_status() != 0:
        raise RuntimeError("device status error during warm-up")
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    launches0 = hils.hils_kernel_launches()
    ms = []
    for _ in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    launches = hils.hils_kernel_launches() - launches0
    clk = clocks.stop()
    if hils.hils_get_status() != 0:
        raise RuntimeError("device status error during the timed steps")
    if world > 1:
        dist.barrier()
    ms_step = max_over_ranks(float(np.mean(ms)), world, dev)
    if rank != 0:
        return
    # algorithmic work: per attended key 10d flops (the logits and <dO, v_j>
    # again, dq, dk, dv), per key of a summary 10d more
    wc = max(1, w.window // w.C)
    i = np.arange(N, dtype=np.int64)
    n_cand = np.maximum(0, i // w.C - (wc - 1))
    keys = np.minimum(K, n_cand) * w.C + (i - n_cand * w.C) + 1
    flops = 10 * d * Hq * B * int(keys.sum()) + 10 * d * B * Hkv * N
    props = torch.cuda.get_device_properties(dev)
    max_mhz = (clk or {}).get("sm_max_mhz") or 1965.0
    ach = flops / (ms_step / 1e3) / 1e12
    if w.dtype == "bf16":
        # bf16: the selected chunks' products (most of the flops) run on the
        # tensor cores, the window branch and the summaries on CUDA cores
        peaks = load_peaks()
        bound = "tensor"
        peak = peaks["bf16_tflops"]
        psrc = f"{peaks['source']} bf16 dense burst"
    else:
        # fp32: every backward kernel runs on CUDA cores
        bound = "alu"
        peak = props.multi_processor_count * 128 * 2 * max_mhz * 1e6 / 1e12   # fp32 FMA lanes x 2 flops x clock
        psrc = f"{props.multi_processor_count} SMs x 128 fp32 lanes x 2 x {max_mhz:.0f} MHz"
    line = {
        "metric": "HiLS backward tokens/s (gradients of q, k, v, lq for a fixed selection)",
        "value": job_throughput(world, B * N, ms_step), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 (fp32 sums)" if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": workload_config(w, world),
        "roofline": {"kernel": "backward (whole call)", "bound": bound, "achieved": ach, "peak": peak,
                     "unit": "TFLOP/s", "frac": ach / peak, "traffic": None, "peak_source": psrc},
        "gpu_launches": int(launches), "clocks": clk, "e2e": None,
    }
    if not args.no_cpu_baseline and world == 1:
        v_cpu, desc, threads = cpu_oracle_backward(w, inp)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": desc}
    print(json.dumps(line), flush=True)


def run_decode(args, w, rank, world, local_rank):
    """One decode step per step for every sequence of the batch; the landmark
    summaries of the cache are built in the untimed setup.  L2 is flushed
    between steps (the compressed keys fit in L2)."""
    import torch
    from chunk_wise_sparse_b200 import hils

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hils.lib()
    w_job = w
    sl = rank_slices(w, world, rank)
    if not sl:
        raise RuntimeError(f"rank {rank}: no sequence of the batch of {w.B} to decode")
    w, inp = slice_inputs(w_job, generate(w_job), sl[0])   # this rank's sequences

    def to_dev(name):
        bits = getattr(inp, name + "_bits")
        if bits is not None:
            return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(getattr(inp, name + "_f32")).to(dev)

    q, k, v, lq = (to_dev(n) for n in ("q", "k", "v", "lq"))
    B, Hq, Hkv, N, d, K = w.B, w.Hq, w.Hkv, w.N, w.d, w.K
    dims = hils.make_dims(B, Hq, Hkv, d, N, K, q.dtype, window=w.window)
    if w.paged:
        # the cache in chunk pages of a pool, in a seeded random order (setup, untimed)
        from chunk_wise_sparse_b200.inputs import page_table
        table, n_pages = page_table(w)
        nc = N // 64
        idx = torch.from_numpy(table.reshape(-1).astype(np.int64)).to(dev)

        def paginate(t):
            pool = torch.empty((n_pages, Hkv, 64, d), dtype=t.dtype, device=dev)
            pool[idx] = t.view(B, Hkv, nc, 64, d).permute(0, 2, 1, 3, 4).reshape(B * nc, Hkv, 64, d)
            return pool

        k, v = paginate(k), paginate(v)
        tab = torch.from_numpy(table).to(dev)
        summ = hils.Summary(dims, dev)
        hils.hils_landmark_summary_paged(dims, k, tab, n_pages, lq, 0, nc, summ.kprime, summ.bprime, summ.kprime_mma)
    else:
        summ = hils.landmark_summary(k, lq, K)
    seq = torch.full((B,), N, dtype=torch.int32, device=dev)
    ws = torch.empty((hils.hils_decode_workspace_bytes(dims),), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    ids = torch.empty((B, Hq, K), dtype=torch.int32, device=dev)
    sc = torch.empty((B, Hq, K), dtype=torch.float32, device=dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        if w.paged:
            hils.hils_attn_decode_paged(dims, q, k, v, tab, n_pages, summ.kprime, summ.bprime, summ.kprime_mma, seq,
                                        o, ids, sc, ws, stream=stream)
        else:
            hils.hils_attn_decode(dims, q, k, v, summ.kprime, summ.bprime, summ.kprime_mma, seq, o, ids, sc, ws,
                                  stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hils.hils_get_status() != 0:
        raise RuntimeError("device status error during warm-up")
    times = []
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    clocks.start()
    time.sleep(0.3)
    launches0 = hils.hils_kernel_launches()
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    launches = hils.hils_kernel_launches() - launches0
    clk = clocks.stop()
    status = hils.hils_get_status()
    if status != 0:
        raise RuntimeError(f"device status {status} during the timed steps")
    us = 1e3 * max_over_ranks(float(np.median(times)), world, dev)
    # the median over 100 more flushed steps, after the timed ones
    more = []
    for _ in range(100):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        torch.cuda.synchronize()
        more.append(e0.elapsed_time(e1))
    if hils.hils_get_status() != 0:
        raise RuntimeError("device status error during the extra steps")
    us_100 = 1e3 * max_over_ranks(float(np.median(more)), world, dev)
    # end to end: every step copies the new queries and the sequence lengths in
    # from pinned host memory and reads the outputs back (the KV cache and its
    # summaries stay resident, as in a serving loop)
    e2e = None
    if not args.no_e2e:
        q_host = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        q_host.copy_(q)
        seq_host = torch.empty(seq.shape, dtype=seq.dtype).pin_memory()
        seq_host.copy_(seq)
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = q_host.numel() * q_host.element_size() + seq_host.numel() * seq_host.element_size()
        d2h = o_host.numel() * o_host.element_size()

        def e2e_step():
            q.copy_(q_host, non_blocking=True)
            seq.copy_(seq_host, non_blocking=True)
            step()
            o_host.copy_(o, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(5, args.steps)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e_us = 1e3 * max_over_ranks(a0.elapsed_time(a1) / n_e2e, world, dev)
        e2e = {"value": e_us, "unit": "us/step", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": "steps back to back, no L2 flush between them"}
    if rank != 0:
        return None
    sel_bytes = decode_selected_bytes(ids.cpu().numpy(), w)
    kp_bytes = B * Hkv * w.nc * (d + 16) * 2
    peaks = load_peaks()
    gbs = sel_bytes / (us / 1e6) / 1e9
    all_gbs = (sel_bytes + kp_bytes) / (us / 1e6) / 1e9
    line = {
        "metric": "HiLS decode us/step (one new token per sequence: scoring, top-K, sparse attention)",
        "value": us, "unit": "us/step", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "fp32",
        "data": f"synthetic: i.i.d. N(0,1), seed {w.seed}" + (", KV cache in chunk pages (random order)" if w.paged else ""),
        "config": dict(workload_config(w_job, world), l2="256 MiB buffer written between steps (L2 flush)"),
        "roofline": {"kernel": "decode step", "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "traffic": recorded_step_traffic("decode", w.name),
                     "bytes": "selected-KV (union of kept chunks + local window chunks per (b, kv head))",
                     "selected_kv_bytes": sel_bytes, "all_bytes_gbs": all_gbs},
        "gpu_launches": int(launches),
        "clocks": clk,
        "e2e": e2e,
        "median_us_of_100_more_steps": us_100,
    }
    if world > 1:
        line["rank0_share"] = {"sequences": list(sl[0][1:]),
                               "note": "the roofline bytes and the e2e copies are rank 0's sequences"}
    if not args.no_cpu_baseline and world == 1:
        v_cpu, desc, threads = cpu_oracle_decode(w, inp, budget_s=args.ref_budget)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "us/step", "cores": threads, "kind": "oracle",
                                "sample": desc}
    return line


# Workloads the default run also times, each in the same process after the
# headline workload, reported under "extra": the batch-8 GQA decode step and
# the 7B-shaped GQA prefill.
EXTRA_WORKLOADS = ("decode-128k-b8-gqa4-d128", "prefill-128k-gqa4-d128")
EXTRA_KEYS = ("value", "unit", "steps", "warmup", "ms_per_step", "higher_is_better", "kernels_ms",
              "decode_us_per_step", "prefill_bc_tflops_useful", "prefill_bc_frac_of_bf16_peak", "roofline",
              "gpu_launches", "clocks", "e2e", "median_us_of_100_more_steps", "config", "rank0_share")


def run_extra(args, name, rank, world, local_rank):
    import copy
    import torch
    w = WORKLOADS[name]
    a = copy.copy(args)
    a.no_cpu_baseline = True
    if w.kind == "decode":
        a.steps, a.warmup = max(args.steps, 50), max(args.warmup, 5)
        line = run_decode(a, w, rank, world, local_rank)
    else:
        a.no_e2e = True
        line = run_ours(a, w, rank, world, local_rank)
    torch.cuda.empty_cache()
    return None if line is None else {k: line[k] for k in EXTRA_KEYS if k in line}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=None, choices=list(WORKLOADS),
                    help=f"default {DEFAULT_WORKLOAD}, plus the extra workloads {', '.join(EXTRA_WORKLOADS)}")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="time the headline workload only")
    ap.add_argument("--ref-budget", type=float, default=15.0, help="seconds of oracle work per sample")
    ap.add_argument("--backward", action="store_true", help="time the backward pass of a prefill workload")
    args = ap.parse_args()
    extras = args.workload is None and not args.no_extras and not args.backward
    w = WORKLOADS[args.workload or DEFAULT_WORKLOAD]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.backward:
            run_backward(args, w, rank, world, local_rank)
            return
        line = (run_decode if w.kind == "decode" else run_ours)(args, w, rank, world, local_rank)
        if extras:
            ex = {name: run_extra(args, name, rank, world, local_rank) for name in EXTRA_WORKLOADS}
            if line is not None:
                line["extra"] = ex
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
