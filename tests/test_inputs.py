"""The seeded input generator: published splitmix64 values, determinism, moments."""
import math

import torch

from routed_grouped_gemm_softmax_b200.inputs import (CONFIGS, gaussian_tensor, make_inputs,
                                                     splitmix64, zipf_bias)


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0: the first outputs of Vigna's reference implementation
    z = splitmix64(0, 0, 3)
    got = [int(v) & ((1 << 64) - 1) for v in z]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_streams_are_counter_based_and_deterministic():
    a = gaussian_tensor(3, "x", (1000,), 1.0)
    b = gaussian_tensor(3, "x", (1000,), 1.0, chunk=97)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    c = gaussian_tensor(3, "router_w", (1000,), 1.0)
    assert not torch.equal(a, c)


def test_normal_moments():
    v = gaussian_tensor(11, "x", (1 << 20,), 2.0, out_dtype=torch.float32).double()
    assert abs(v.mean().item()) < 0.01
    assert abs(v.std().item() - 2.0) < 0.01
    assert abs(((v / 2) ** 4).mean().item() - 3.0) < 0.05


def test_shapes_and_bias():
    inp = make_inputs(CONFIGS["tiny"])
    assert inp.x.shape == (64, 256) and inp.router_w.shape == (256, 8)
    assert inp.w_gate.shape == (8, 512, 256) and inp.w_down.shape == (8, 256, 512)
    b = zipf_bias(64, 1.2)
    p = torch.exp(b.double())
    assert abs(p.sum().item() - 1) < 1e-6 and abs(p[0].item() - 0.2925) < 1e-3
    assert math.isclose(float(b[0] - b[1]), 1.2 * math.log(2), rel_tol=1e-5)
