"""Seeded input generator: determinism, rounding and the stated distributions."""
import numpy as np
import torch

from selective_state_space_32_b200 import workloads as W


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 1e-40, 3e38],
                                 dtype=np.float32)])
    ours = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(W.bf16_bits_to_f32(ours),
                          torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generate_is_deterministic_and_block_invariant():
    a = W.generate(2, 40, 24, 16, "bf16", 0.1, 0.32, seed=7, block=1 << 20)
    b = W.generate(2, 40, 24, 16, "bf16", 0.1, 0.32, seed=7, block=97)
    for k in ("u", "delta", "A", "B", "C", "h0"):
        assert np.array_equal(a[k], b[k]), k
    c = W.generate(2, 40, 24, 16, "bf16", 0.1, 0.32, seed=8)
    assert not np.array_equal(a["u"], c["u"])


def test_shapes_and_distributions():
    g = W.generate(2, 512, 64, 16, "f32", 0.0, 0.0, seed=3)
    assert g["u"].shape == (2, 512, 64) and g["u"].dtype == np.float32
    assert g["B"].shape == (2, 512, 16) and g["A"].shape == (64, 16) and g["h0"] is None
    assert np.array_equal(g["A"], -np.arange(1, 17, dtype=np.float32)[None].repeat(64, 0))
    d = g["delta"]
    assert d.min() > 0
    # median delta per channel sits inside the [1e-3, 1e-1] initialisation range
    med = np.median(d.reshape(-1, 64), axis=0)
    assert med.min() > 5e-4 and med.max() < 0.2
    assert abs(g["u"].std() - 1.0) < 0.05


def test_reset_tokens():
    L = 1000
    g = W.generate(2, L, 8, 16, "f32", 0.0, 0.32, seed=4)
    big = g["delta"] > 2.5          # reset tokens: delta + 3
    # every channel of a reset position is bumped; exactly round(0.32 L) positions per row
    per_pos = big.all(axis=2)
    assert np.array_equal(per_pos, big.any(axis=2))
    assert list(per_pos.sum(axis=1)) == [320, 320]
    assert g["delta"][~big].max() < 0.05


def test_workload_table():
    w = W.WORKLOADS["mamba130m_f32"]
    assert (w.B, w.L, w.D, w.N, w.dtype) == (8, 2048, 1536, 16, "f32")
    assert w.algorithmic_bytes() == 304971776
    assert W.WORKLOADS["mamba1p4b_bf16"].algorithmic_bytes() == 405012480
    assert W.WORKLOADS["longseq_bf16"].algorithmic_bytes() == 1619394560
    assert W.WORKLOADS["zoh_n64_bf16"].algorithmic_bytes() == 529793024


def test_fused_generator_matches_the_unfused_recipe():
    # same seed: u, B, C, h0 identical; softplus(raw delta + bias) is the unfused delta
    # up to the fp32 rounding of the raw value and of the bias
    a = W.generate(2, 40, 24, 16, "f32", 0.1, seed=77)
    b = W.generate(2, 40, 24, 16, "f32", 0.1, seed=77, fused=True)
    for k in ("u", "B", "C", "h0", "A"):
        assert np.array_equal(a[k], b[k]), k
    s = b["delta"].astype(np.float64) + b["delta_bias"].astype(np.float64)[None, None, :]
    eff = np.maximum(s, 0.0) + np.log1p(np.exp(-np.abs(s)))
    assert np.allclose(eff, a["delta"], rtol=2e-6, atol=0)
    assert b["z"].shape == (2, 40, 24) and b["delta_bias"].dtype == np.float32
    assert a["z"] is None and a["delta_bias"] is None
    w = W.WORKLOADS["mamba130m_fused_f32"]
    assert w.algorithmic_bytes() == W.WORKLOADS["mamba130m_f32"].algorithmic_bytes() + 4 * 8 * 2048 * 1536 + 4 * 1536
