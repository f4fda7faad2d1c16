"""The seeded input generator: determinism, subsets, bf16 rounding, shapes."""
import numpy as np
import torch

import dbst_synth as S


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, -0.0, 65504.0, 1e-30], np.float32)])
    ours = S.bf16_bits_from_f32(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(S.f32_from_bf16_bits(ours),
                                  torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_generator_is_deterministic_and_subsets_match():
    w = S.workload("small")
    q1, k1, v1 = S.make_qkv(w)
    q2, k2, v2 = S.make_qkv(w, heads=range(3, 6))
    assert q1.shape == (w.B, w.H, w.N, w.D) and q1.dtype == np.uint16
    np.testing.assert_array_equal(q1[:, 3:6], q2)
    np.testing.assert_array_equal(k1[:, 3:6], k2)
    np.testing.assert_array_equal(v1[:, 3:6], v2)
    q3, _, _ = S.make_qkv(w)
    np.testing.assert_array_equal(q1, q3)


def test_workload_geometry():
    for w in S.WORKLOADS:
        assert w.blk == 64
        assert all(g % t == 0 for g, t in zip(w.grid, w.tile))
        assert w.NB * 64 == w.N
    assert S.workload("wan").NB == 588 and S.workload("wan").N == 37632
    assert S.workload("hunyuan").NB == 2040 and S.workload("hunyuan").N == 130560
    assert S.workload("sweep").NB == 256
    assert S.workload("wan_2x4x8").NB == 616 and S.workload("wan_2x4x8").N == 39424


def test_field_statistics():
    w = S.workload("tiny")
    q, k, v = S.make_qkv(w)
    qf, kf, vf = (S.f32_from_bf16_bits(a).astype(np.float64) for a in (q, k, v))
    assert abs(vf.mean()) < 0.05 and abs(vf.std() - 1.0) < 0.05
    # q and k share the smooth field: strongly correlated, not identical
    c = np.corrcoef(qf.ravel(), kf.ravel())[0, 1]
    expect = w.alpha**2 * w.f_rms**2 / (w.alpha**2 * w.f_rms**2 + w.beta**2)
    assert abs(c - expect) < 0.05
