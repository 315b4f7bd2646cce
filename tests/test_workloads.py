"""The seeded input generator: determinism, distributions, bf16 rounding."""
import math

import numpy as np
import torch

import workloads as wl


def test_generator_is_deterministic_and_keyed_by_name():
    a = wl.normal(7, "q", (1000,))
    b = wl.normal(7, "q", (1000,))
    c = wl.normal(7, "k", (1000,))
    d = wl.normal(8, "q", (1000,))
    np.testing.assert_array_equal(a, b)
    assert not np.allclose(a, c) and not np.allclose(a, d)
    # a prefix of a longer draw is the shorter draw
    np.testing.assert_array_equal(wl.normal(7, "q", (2000,))[:1000], a)


def test_splitmix64_reference_values():
    # splitmix64 with state 0: the published first outputs of the generator
    z = wl.splitmix64(np.uint64(0), 3)
    assert [int(x) for x in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_distributions():
    x = wl.normal(3, "x", (200000,), std=0.5)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 0.5) < 0.01
    u = wl.uniform(3, "u", (200000,), 0.0, math.log(16))
    assert u.min() > 0 and u.max() < math.log(16) and abs(u.mean() - math.log(16) / 2) < 0.01


def test_bf16_rounding_matches_torch():
    x = wl.normal(1, "r", (50000,), std=3.0)
    x[:4] = [0.0, -0.0, 1e-40, 65504.0]
    ours = wl.to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = wl.round_bf16(x)
    np.testing.assert_array_equal(back, torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().double().numpy())


def test_scan_inputs_shapes():
    cfg = wl.PREFILL_PYTHIA
    inp = wl.scan_inputs(cfg, B=1, L=64)
    assert inp["q"].shape == (1, 64, 8, 256) and inp["v"].shape == (1, 64, 8, 256)
    assert inp["W_q"].shape == (128, 256) and inp["dt"].shape == (1, 64, 8)
    assert inp["A_log"].shape == (8,)
    # values are already bf16-representable
    np.testing.assert_array_equal(wl.round_bf16(inp["q"]), inp["q"])


def test_sub_blocks_equal_slices_of_the_full_draw():
    # contiguous sub-blocks (drawn pair by pair over a flat range) and strided
    # ones (drawn element by element) both equal the same slice of the full array
    shape = (6, 70, 4, 64)
    full = wl.normal(9, "v", shape, std=0.5)
    np.testing.assert_array_equal(wl.normal(9, "v", shape, std=0.5, index=(slice(1, 5),)), full[1:5])
    np.testing.assert_array_equal(wl.normal(9, "v", shape, std=0.5, index=(3, slice(7, 60))), full[3, 7:60])
    np.testing.assert_array_equal(wl.normal(9, "v", shape, std=0.5, index=(slice(0, 6, 2),)), full[0:6:2])
    np.testing.assert_array_equal(wl.normal(9, "v", shape, std=0.5, index=(-1,)), full[-1])
    u = wl.uniform(9, "a", shape)
    np.testing.assert_array_equal(wl.uniform(9, "a", shape, index=(slice(2, 4),)), u[2:4])
