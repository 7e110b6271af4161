"""The seeded input generator: published SplitMix64 vectors, stream layout, torch twin."""
import numpy as np
import torch

from qi21_synth import gen, configs


def test_splitmix64_published_vector():
    # SplitMix64 from state 0: the first three outputs as published with the
    # reference implementation (Vigna, splitmix64.c).
    got = [int(v) for v in gen.uniform_u64(0, 0, 3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert gen.splitmix64_mix(gen.GOLDEN_GAMMA) == 0xE220A8397B1DCDAF


def test_normal_is_counter_based_and_chunk_invariant():
    a = gen.normal(7, "x", (1000,))
    b = gen.normal(7, "x", (1000,), chunk=37)
    np.testing.assert_array_equal(a, b)
    c = gen.normal(7, "y", (1000,))
    assert not np.array_equal(a, c)
    assert abs(a.mean()) < 0.15 and abs(a.std() - 1.0) < 0.1
    big = gen.normal(3, "z", (200000,))
    assert abs(big.mean()) < 0.01 and abs(big.std() - 1.0) < 0.01


def test_torch_twin_matches_numpy():
    a = gen.normal(1234, "L0.w_q", (3, 1001), std=0.02)
    t = gen.normal_torch(1234, "L0.w_q", (3, 1001), std=0.02, chunk=777).numpy()
    np.testing.assert_allclose(t, a, rtol=0, atol=1e-17)


def test_bf16_rounding_matches_torch():
    x = gen.normal(5, "r", (4096,), std=0.02)
    ours = configs.round_to(x, "bfloat16")
    ref = torch.from_numpy(x).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_workload_sizes():
    w = configs.make_workload("full")
    assert (w.n_prefix, w.n_target) == (4608, 4096)
    w = configs.make_workload("large")
    assert (w.n_prefix, w.n_target) == (33792, 16384)
    w = configs.make_workload("toy")
    assert (w.n_prefix, w.n_target) == (7, 4)
