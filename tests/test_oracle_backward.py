"""Pins of the oracle's backward pass (gradients of <dO, O> for a fixed
selection; the AI Trends article, section "방법론", states that the chunk
score is part of the forward attention, so the loss gradient reaches the
landmark queries and the Q-Cal adapter through it).

The backward is pinned to things other than itself: torch autograd of an
independent fp64 statement of the forward (whose output is first checked
against the oracle's forward), central finite differences of the oracle's
forward, the dense causal attention it reduces to when the window covers the
sequence, and invariants of the forward (each row's fusion weights sum to 1,
so the value gradients sum to the output gradients; a common shift of all
keys of a kv head leaves the output unchanged, so their gradients sum to 0).
CPU only.
"""
import math

import numpy as np
import pytest
import torch

from oracle.oracle import Oracle, Rows


def rand(rng, *shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def case(seed, B=1, Hq=2, Hkv=1, N=512, d=16, C=64, K=3, W=0, qs=False):
    rng = np.random.default_rng(seed)
    t = dict(Q=rand(rng, B, Hq, N, d), K=rand(rng, B, Hkv, N, d), V=rand(rng, B, Hkv, N, d),
             LQ=rand(rng, B, Hkv, N // C, d, scale=1.5), dO=rand(rng, B, Hq, N, d))
    t["Qs"] = (t["Q"] + rand(rng, B, Hq, N, d, scale=0.5)) if qs else None
    o = Oracle(B, Hq, Hkv, N, d, C, K, W)
    kp, bp = o.summary(t["K"], t["LQ"])
    rows = Rows.from_prefill(t["Q"] if t["Qs"] is None else t["Qs"], np.arange(B * Hq * N))
    ids, _, _ = o.select(kp, bp, rows)
    t["ids"] = ids.reshape(B, Hq, N, K)
    return o, t


def torch_forward(Q, Kt, V, LQ, ids, C, W, Qs=None):
    """The forward for fixed ids, written with torch ops in fp64: summaries by
    a softmax over each chunk, scores, a softmax inside each selected chunk and
    over the causal window, and a softmax over the branch scores."""
    B, Hq, N, d = Q.shape
    Hkv = Kt.shape[1]
    G = Hq // Hkv
    nc = N // C
    tau = 1.0 / math.sqrt(d)
    Kc = Kt.reshape(B, Hkv, nc, C, d)
    pl = torch.softmax(tau * torch.einsum("bhcd,bhcjd->bhcj", LQ, Kc), dim=-1)
    kp = torch.einsum("bhcj,bhcjd->bhcd", pl, Kc)
    bp = -(pl * torch.log(pl)).sum(-1)
    wc = max(1, W // C)
    out = torch.zeros_like(Q)
    Qs = Q if Qs is None else Qs
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            for i in range(N):
                q, qs = Q[b, hq, i], Qs[b, hq, i]
                us, os_ = [], []
                for c in ids[b, hq, i]:
                    c = int(c)
                    if c < 0:
                        continue
                    p = torch.softmax(tau * Kt[b, h, c * C:(c + 1) * C] @ q, 0)
                    os_.append(p @ V[b, h, c * C:(c + 1) * C])
                    us.append(tau * (qs @ kp[b, h, c]) + bp[b, h, c])
                w0 = max(0, (i // C - (wc - 1)) * C)
                z = tau * Kt[b, h, w0:i + 1] @ q
                us.append(torch.logsumexp(z, 0))
                os_.append(torch.softmax(z, 0) @ V[b, h, w0:i + 1])
                a = torch.softmax(torch.stack(us), 0)
                out[b, hq, i] = (a[:, None] * torch.stack(os_)).sum(0)
    return out


@pytest.mark.parametrize("W,qs", [(0, False), (192, False), (0, True)])
def test_pin_backward_equals_autograd_of_an_independent_forward(W, qs):
    o, t = case(3, W=W, qs=qs, N=384)
    g = o.backward(t["Q"], t["K"], t["V"], t["LQ"], t["ids"], t["dO"], Qs=t["Qs"])
    T = {n: torch.tensor(t[n], dtype=torch.float64, requires_grad=True) for n in ("Q", "K", "V", "LQ")}
    Ts = torch.tensor(t["Qs"], dtype=torch.float64, requires_grad=True) if qs else None
    out = torch_forward(T["Q"], T["K"], T["V"], T["LQ"], t["ids"], 64, W, Ts)
    # the restatement computes the oracle's forward
    kp, bp = o.summary(t["K"], t["LQ"])
    rows = Rows.from_prefill(t["Q"], np.arange(t["Q"].shape[0] * t["Q"].shape[1] * t["Q"].shape[2]))
    O_or, _ = o.attend(t["K"], t["V"], kp, bp, rows, t["ids"].reshape(len(rows), -1),
                       qscore=None if not qs else t["Qs"].reshape(len(rows), -1))
    assert np.max(np.abs(out.detach().numpy().reshape(len(rows), -1) - O_or)) < 1e-12
    loss = (out * torch.tensor(t["dO"], dtype=torch.float64)).sum()
    wrt = [T["Q"], T["K"], T["V"], T["LQ"]] + ([Ts] if qs else [])
    grads = torch.autograd.grad(loss, wrt)
    names = ["dQ", "dK", "dV", "dLQ"] + (["dQs"] if qs else [])
    for n, gr in zip(names, grads):
        ref = gr.numpy()
        assert np.max(np.abs(g[n] - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref))), n


def test_pin_backward_matches_finite_differences():
    o, t = case(5, W=128, Hq=2, N=320, d=8)
    g = o.backward(t["Q"], t["K"], t["V"], t["LQ"], t["ids"], t["dO"])
    B, Hq, N, d = t["Q"].shape
    rows = Rows.from_prefill(t["Q"], np.arange(B * Hq * N))
    ids = t["ids"].reshape(len(rows), -1)

    def loss(Q, K, V, LQ):
        kp, bp = o.summary(K, LQ)
        O, _ = o.attend(K, V, kp, bp, Rows.from_prefill(Q, np.arange(B * Hq * N)), ids)
        return float((O * t["dO"].reshape(len(rows), -1).astype(np.float64)).sum())

    rng = np.random.default_rng(9)
    for name, key in (("Q", "dQ"), ("K", "dK"), ("V", "dV"), ("LQ", "dLQ")):
        for _ in range(4):
            arr = t[name]
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            h = 1e-2
            ap, am = arr.copy(), arr.copy()
            ap[idx] += h
            am[idx] -= h
            args = {n: t[n] for n in ("Q", "K", "V", "LQ")}
            fd = (loss(**{**args, name: ap}) - loss(**{**args, name: am})) / float(ap[idx] - am[idx])
            assert abs(fd - g[key][idx]) <= 2e-5 * max(1.0, abs(fd)), (name, idx, fd, g[key][idx])


def test_pin_window_over_everything_is_dense_attention_backward():
    """No candidates: the gradients are those of dense causal softmax
    attention (torch autograd of the textbook formula) and the landmark
    queries get none."""
    o, t = case(7, W=512, N=512, Hq=2, Hkv=1)
    assert np.all(t["ids"] == -1)
    g = o.backward(t["Q"], t["K"], t["V"], t["LQ"], t["ids"], t["dO"])
    Q = torch.tensor(t["Q"], dtype=torch.float64, requires_grad=True)
    Kt = torch.tensor(t["K"], dtype=torch.float64, requires_grad=True)
    V = torch.tensor(t["V"], dtype=torch.float64, requires_grad=True)
    N, d = Q.shape[2], Q.shape[3]
    s = Q @ Kt.expand(-1, 2, -1, -1).transpose(-1, -2) / math.sqrt(d)
    s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    out = torch.softmax(s, -1) @ V.expand(-1, 2, -1, -1)
    gq, gk, gv = torch.autograd.grad((out * torch.tensor(t["dO"], dtype=torch.float64)).sum(), [Q, Kt, V])
    for mine, ref in ((g["dQ"], gq), (g["dK"], gk), (g["dV"], gv)):
        assert np.max(np.abs(mine - ref.numpy())) < 1e-10
    assert np.all(g["dLQ"] == 0)


def test_value_gradients_sum_to_the_output_gradients():
    """Every row's weights over all the keys it attends sum to 1, so the sum
    of dV over the keys of a kv head is the sum of dO over its query heads."""
    o, t = case(11, W=192, Hq=4, Hkv=2, N=448, K=4)
    g = o.backward(t["Q"], t["K"], t["V"], t["LQ"], t["ids"], t["dO"])
    B, Hq, N, d = t["Q"].shape
    dOg = t["dO"].astype(np.float64).reshape(B, 2, 2, N, d).sum(axis=(2, 3))
    assert np.max(np.abs(g["dV"].sum(axis=2) - dOg)) < 1e-9


def test_shifting_all_keys_changes_nothing():
    """Adding one vector to every key of a kv head shifts all of a row's
    logits and branch scores (summaries included) by the same amount, so the
    output does not move: the key gradients of each kv head sum to zero."""
    o, t = case(13, W=128, Hq=2, N=384, K=3, qs=False)
    g = o.backward(t["Q"], t["K"], t["V"], t["LQ"], t["ids"], t["dO"])
    assert np.max(np.abs(g["dK"].sum(axis=2))) < 1e-9
    assert np.max(np.abs(g["dK"])) > 1e-2
