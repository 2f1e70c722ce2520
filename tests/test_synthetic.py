"""The seeded input generators produce what the input recipe states: the
same tensor for the same key, the stated distributions, exactly the stated
number of outliers, a unit-norm steering vector and the workload shapes."""
import numpy as np
import torch

import synthetic


def test_same_key_same_tensor_and_keys_differ():
    a = synthetic.weight("t/W", 64, 128)
    assert torch.equal(a, synthetic.weight("t/W", 64, 128))
    assert not torch.equal(a, synthetic.weight("t/W2", 64, 128))
    assert not torch.equal(a, synthetic.weight("t/W", 64, 128, base=1))
    assert a.dtype == torch.float16 and a.shape == (64, 128)


def test_weight_distribution_and_exact_outlier_count():
    N, K = 1536, 1536
    w = synthetic.weight("t/dist", N, K).float()
    assert abs(w.mean().item()) < 2e-4 and abs(w.std().item() - 0.02) < 2e-4
    wo = synthetic.weight("t/dist", N, K, outlier_frac=0.001).float()
    changed = (wo != w)
    assert int(changed.sum()) == round(0.001 * N * K)          # exactly the stated count
    assert abs(wo[changed].std().item() - 0.2) < 0.02           # redrawn from N(0, 0.2^2)


def test_activation_outlier_channels():
    M, K = 64, 1536
    x = synthetic.activation("t/act", M, K).float()
    xo = synthetic.activation("t/act", M, K, outlier_channel_frac=0.01).float()
    ratio = (xo / x.masked_fill(x == 0, 1)).abs()
    cols = (ratio > 10).all(dim=0)
    assert int(cols.sum()) == round(0.01 * K)                    # 15 of 1536 channels, every row
    assert torch.allclose(xo[:, cols], (x[:, cols] * 20).half().float(), rtol=1e-3)
    assert torch.equal(xo[:, ~cols], x[:, ~cols])


def test_steer_vector_unit_norm_fp32():
    v = synthetic.replay_steer()
    assert v.dtype == torch.float32 and v.shape == (1536,)
    assert abs(float(np.linalg.norm(v.double().numpy())) - 1.0) < 1e-6


def test_workload_shapes():
    assert [(n, k, nn) for n, k, nn in synthetic.D1536] == [
        ("qkv", 1536, 4608), ("out", 1536, 1536), ("up", 1536, 6144), ("down", 6144, 1536)]
    assert [(n, k, nn) for n, k, nn in synthetic.D1024] == [
        ("qkv", 1024, 3072), ("out", 1024, 1024), ("up", 1024, 4096), ("down", 4096, 1024)]
    assert (synthetic.REPLAY_BLOCKS, synthetic.REPLAY_STEPS, synthetic.REPLAY_M) == (24, 8, 432)
    W, X = synthetic.w8a8_d1536("down", 432)
    assert W.shape == (1536, 6144) and X.shape == (432, 6144)
    t = synthetic.tiny_q8()
    assert t["W"].shape == (256, 256) and t["X"].shape == (64, 256) and t["bias"].shape == (256,)
