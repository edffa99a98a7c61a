"""The seeded input generator: distribution, counter addressing and dtype rounding."""
import numpy as np
import pytest
import scipy.stats
import torch

import synth


def test_standard_normal():
    a = synth.fill_host(1_000_000, 0, 3, 0, 1.0, synth.F32).astype(np.float64)
    assert abs(a.mean()) < 5e-3
    assert abs(a.var() - 1.0) < 5e-3
    assert abs(scipy.stats.skew(a)) < 1e-2
    assert abs(scipy.stats.kurtosis(a)) < 2e-2
    assert scipy.stats.kstest(a[:200_000], "norm").pvalue > 1e-3


def test_counter_addressing():
    full = synth.fill_host(50_000, 4, 5, 0, 0.5, synth.F32)
    part = synth.fill_host(1000, 4, 5, 20_000, 0.5, synth.F32)
    assert np.array_equal(full[20_000:21_000], part)
    # thread count does not change the bits
    assert np.array_equal(full, synth.fill_host(50_000, 4, 5, 0, 0.5, synth.F32, nthreads=1))


def test_streams_differ():
    a = synth.fill_host(4096, 0, 3, 0, 1.0, synth.F32)
    b = synth.fill_host(4096, 0, 4, 0, 1.0, synth.F32)
    c = synth.fill_host(4096, 1, 3, 0, 1.0, synth.F32)
    assert np.mean(a == b) < 0.01 and np.mean(a == c) < 0.01
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.06


def test_bf16_is_round_to_nearest_even_of_the_f32_draw():
    f = synth.fill_host(100_000, 2, 7, 0, 0.02, synth.F32)
    b = synth.fill_host(100_000, 2, 7, 0, 0.02, synth.BF16)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, ref)


@pytest.mark.parametrize("which", ["router", "gate", "up", "down"])
def test_tensor_std(which):
    shape = synth.OLMOE
    t = synth.bf16_bits_to_f32(synth.host_tensor(shape, which, 0 if which != "router" else None))
    want = {"router": 0.02, "gate": shape.hidden ** -0.5, "up": shape.hidden ** -0.5,
            "down": shape.inter ** -0.5}[which]
    assert abs(t.astype(np.float64).std() / want - 1) < 0.01


def test_expert_slices_are_independent_of_the_rest():
    shape = synth.TINY
    whole = synth.host_tensor(shape, "up")
    assert np.array_equal(whole[3], synth.host_tensor(shape, "up", 3))
