"""The seeded input generator: determinism, bf16 rounding, needle placement."""
import numpy as np
import torch

from chunk_wise_sparse_b200.inputs import (QUERY_BLOCK, WORKLOADS, custom, generate, round_bf16_bits,
                                           bf16_bits_to_f32, sample_rows)


def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 100000),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0], np.float32)])
    x = x.astype(np.float32)
    ours = round_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generator_rounding_matches_numpy_rne():
    """The generator's bf16 conversion equals an independent numpy RNE."""
    w = custom(B=1, Hq=1, Hkv=1, d=64, N=4096, K=4, seed=9, dtype="bf16")
    inp = generate(w)
    from chunk_wise_sparse_b200.inputs import _normal
    assert np.array_equal(inp.v_bits, round_bf16_bits(_normal((1, 1, 4096, 64), 9, 2)))


def test_generation_is_deterministic():
    w = custom(B=1, Hq=2, Hkv=1, d=32, N=2048, K=4, seed=7, dtype="bf16", needles=3, needle_mode="random")
    a, b = generate(w), generate(w)
    for n in ("q_bits", "k_bits", "v_bits", "lq_bits"):
        assert np.array_equal(getattr(a, n), getattr(b, n))
    assert np.array_equal(a.needle_chunks, b.needle_chunks)


def test_needles_lie_before_their_block_and_shift_keys():
    w = custom(B=2, Hq=4, Hkv=2, d=64, N=4096, K=4, seed=3, dtype="fp32", needles=5, needle_mode="random")
    inp = generate(w)
    assert len(set(inp.needle_chunks.tolist())) == 5
    for c, blk in zip(inp.needle_chunks, inp.needle_blocks):
        assert (c + 1) * w.C <= blk * QUERY_BLOCK
    # the needle chunk keys carry a 1.5 * unit-vector shift: their mean moves
    from chunk_wise_sparse_b200.inputs import _normal
    k0 = _normal((w.B, w.Hkv, w.N, w.d), w.seed, 1)
    for c in inp.needle_chunks:
        delta = (inp.k_f32 - k0)[:, :, c * w.C:(c + 1) * w.C]
        assert np.allclose(np.linalg.norm(delta.mean(axis=2), axis=-1), 1.5, atol=1e-5)
    mask = np.ones(w.nc, bool); mask[inp.needle_chunks] = False
    assert np.array_equal(inp.k_f32.reshape(w.B, w.Hkv, w.nc, w.C, w.d)[:, :, mask],
                          k0.reshape(w.B, w.Hkv, w.nc, w.C, w.d)[:, :, mask])


def test_per_block_needles_tiny_workload():
    w = WORKLOADS["tiny-fp32-1k"]
    inp = generate(w)
    assert list(inp.needle_blocks) == [1, 2, 3]
    for c, blk in zip(inp.needle_chunks, inp.needle_blocks):
        assert (c + 1) * w.C <= blk * QUERY_BLOCK
    assert inp.q_bits is None and inp.q_f32.dtype == np.float32


def test_sample_rows():
    w = WORKLOADS["prefill-128k-gqa4-d128"]
    r = sample_rows(w)
    assert len(r) == 4096 and len(np.unique(r)) == 4096 and np.all(np.diff(r) > 0)
    assert r.max() < w.B * w.Hq * w.N
    assert np.array_equal(sample_rows(WORKLOADS["tiny-fp32-1k"]), np.arange(1024))
