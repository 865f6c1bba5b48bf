"""The seeded input generator (workloads.py), on the CPU: its bf16 rounding
against torch's, and the recipes as stated in its docstring."""
import numpy as np
import torch

from quantization_aware_attention_nvfp4_b200 import workloads as W


def test_bf16_rounding_matches_torch_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(1e3),
        # exact halfway cases between neighbouring bf16 values, both parities
        (np.arange(1, 4096, dtype=np.uint32) << np.uint32(15)).view(np.float32),
        np.array([0.0, -0.0, 1e-45, -3.4e38, 3.3e38], np.float32),
    ])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(W.f32_to_bf16_bits(x), want)
    assert np.array_equal(W.bf16_bits_to_f32(want), torch.from_numpy(want.view(np.int16)).view(
        torch.bfloat16).float().numpy())


def test_each_head_regenerates_on_its_own():
    w = W.custom(2, 3, 40, 56, 32, seed_index=7)
    full = W.tensor_bits(w, "k")
    assert full.shape == (2, 3, 56, 32)
    assert np.array_equal(W.head_bits(w, "k", 1, 2), full[1, 2])
    # different heads and tensors draw different streams
    assert not np.array_equal(full[0, 0], full[0, 1])
    assert not np.array_equal(W.head_bits(w, "q", 0, 0)[:40], W.head_bits(w, "k", 0, 0)[:40])


def test_outlier_channels_shared_by_q_and_k():
    w = W.get("outlier_channels_4096")
    for h in (0, 5):
        q, k = (np.abs(W.head_f32(w, t, 0, h)) for t in ("q", "k"))
        top_q = set(np.argsort(q.mean(0))[-4:])
        top_k = set(np.argsort(k.mean(0))[-4:])
        assert top_q == top_k  # the same 4 channels, x20
        rest = np.setdiff1d(np.arange(w.D), list(top_q))
        assert q[:, list(top_q)].mean() > 10 * q[:, rest].mean()
    v = np.abs(W.head_f32(w, "v", 0, 0))
    assert v.mean(0).max() < 1.2  # V is plain N(0, 1)


def test_per_head_scales_and_token_outliers():
    w = W.get("scaled_heads_16384")
    base = W.custom(1, 1, w.Lq, w.Lk, w.D, seed_index=w.index)  # same streams, recipe "normal"
    for t in ("q", "k", "v", "do"):
        x, x0 = W.head_f32(w, t, 1, 4), W.head_f32(base, t, 1, 4)
        nz = x0 != 0
        s = x[nz] / x0[nz]
        assert np.allclose(s, s[0], rtol=1e-6) and 0.5 <= s[0] <= 2.0
    w = W.get("large_40h_75600")
    x = W.head_f32(w, "v", 0, 3)[:, :8]
    plain = W.head_f32(W.custom(1, 40, w.Lq, w.Lk, w.D, seed_index=w.index), "v", 0, 3)[:, :8]
    scaled_rows = np.flatnonzero(np.any(x != plain, axis=1))
    assert len(scaled_rows) == round(0.01 * w.Lk)
    assert np.allclose(x[scaled_rows], 8 * plain[scaled_rows])
    do = W.head_f32(w, "do", 0, 3)[:, :8]
    assert np.array_equal(do, W.head_f32(W.custom(1, 40, w.Lq, w.Lk, w.D, seed_index=w.index), "do", 0, 3)[:, :8])
