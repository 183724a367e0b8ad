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


def test_mx_weights_match_the_oracle_quantiser():
    # the MX weight recipe (e2m1 codes, one e8m0 scale per 32 values) gives the same codes
    # and scales as the oracle's MX quantiser, on random rows of many magnitudes, an
    # all-zero block, one huge value and exact powers of two; and the workload
    # generator draws the same master values as the bf16 weights
    import numpy as np

    import oracle
    from routed_grouped_gemm_softmax_b200.inputs import make_mx_weights, quantize_blocks_mx_e2m1

    rng = np.random.default_rng(0)
    w = torch.tensor(rng.standard_normal((2, 8, 128)).astype(np.float32)) * 10.0 ** torch.tensor(
        rng.uniform(-3, 3, (2, 8, 1)).astype(np.float32))
    w[0, 0, :32] = 0.0
    w[1, 1, 5] = 1.0e4
    w[1, 2, :] = torch.tensor(np.ldexp(1.0, np.arange(-60, 68)).astype(np.float32))
    q, x = quantize_blocks_mx_e2m1(w)
    qo, xo = oracle.get().mx_quantize_rows(w.reshape(-1, 128).numpy(), 1)
    assert np.array_equal(q.reshape(-1, 128).numpy(), qo)
    assert np.array_equal(x.reshape(-1, 4).numpy(), xo)

    cfg = CONFIGS["fp8"].replace(E=2, H=128, I=64, T=4, seed=6)
    mw = make_mx_weights(cfg)
    master = make_inputs(cfg).w_gate.float()
    q2, x2 = quantize_blocks_mx_e2m1(master)
    assert torch.equal(mw["w_gate_q"], q2) and torch.equal(mw["w_gate_x"], x2)
