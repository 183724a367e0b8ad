"""The certified router's error bound, on the CPU, against the oracle's exact values.

The bound the router uses for |fp32 chain - tensor-core logit| is, per (t, e),
  d = eps * |x_t| * |w_e| (+ a few ulps of |logit|),
  eps = (H + 256 + H/64 + slices) * u * 1.01,   u = 2^-24,
where H*u bounds the fp32 fma chain's own rounding (recursive summation: each of
the H steps rounds once, so the error is at most H*u*sum_h |x_h w_he| to first
order), 256*u covers each 64-term tensor-core block accumulated within 4 ulps,
(H/64 + slices)*u the fp32 sums of the blocks and of the K slices, and
sum_h |x_h w_he| <= |x_t| |w_e| by Cauchy-Schwarz.  These tests check each piece
against the oracle's fp64 logits: the chain stays inside its own first term, and a
simulated tensor-core evaluation (each 64-term block's exact sum rounded to fp32,
then fp32 sums) stays inside the whole bound.
"""
import numpy as np
import torch

import oracle
from routed_grouped_gemm_softmax_b200.inputs import CONFIGS, make_inputs

U = 2.0 ** -24


def _bf16_to_f64(t):
    return t.float().double().numpy()


def _case(cfg, adversarial=False):
    inp = make_inputs(cfg, device="cpu", weights=False)
    x, rw = inp.x, inp.router_w
    if adversarial:
        # heavy cancellation: x_h * w_he of alternating sign and large magnitude, so
        # |sum| << sum |x_h w_he| and the relative error of the logit is large
        xs = x.float()
        xs[:, 1::2] = -xs[:, 0::2]
        x = (xs * 64).to(torch.bfloat16)
        rw = (rw.float() * 64).to(torch.bfloat16)
    return x, rw, inp.bias


def _bound_parts(x64, w64, H, slices):
    abs_sum = np.abs(x64) @ np.abs(w64)                       # sum_h |x_h w_he|
    cs = np.linalg.norm(x64, axis=1)[:, None] * np.linalg.norm(w64, axis=0)[None, :]
    eps = (H * U + 256 * U + (H / 64 + slices) * U) * 1.01
    return abs_sum, cs, eps


def _simulated_tensor_core(x64, w64, slices):
    """Each 64-wide K block summed exactly and rounded to fp32 (within the 4-ulp
    assumption), the blocks of a slice summed in fp32 in K order, then the slices."""
    T, H = x64.shape
    nb = H // 64
    per = (nb + slices - 1) // slices
    total = np.zeros((T, w64.shape[1]), np.float32)
    for s in range(slices):
        acc = np.zeros_like(total)
        for b in range(s * per, min(nb, (s + 1) * per)):
            blk = (x64[:, 64 * b:64 * b + 64] @ w64[64 * b:64 * b + 64, :]).astype(np.float32)
            acc = (acc + blk).astype(np.float32)
        total = (total + acc).astype(np.float32)
    return total.astype(np.float64)


def _check(cfg, adversarial, slices):
    x, rw, bias = _case(cfg, adversarial)
    _, _, l32, l64 = oracle.get().route(x, rw, None, cfg.top_k, want_logits=True)
    x64, w64 = _bf16_to_f64(x), _bf16_to_f64(rw)
    H = cfg.H
    abs_sum, cs, eps = _bound_parts(x64, w64, H, slices)
    # Cauchy-Schwarz
    assert np.all(abs_sum <= cs * (1 + 1e-12))
    # the fp32 chain within H*u*sum|x_h w_he| of the exact value
    chain_err = np.abs(l32.astype(np.float64) - l64)
    assert np.all(chain_err <= H * U * abs_sum + 1e-300), float((chain_err / (H * U * abs_sum + 1e-300)).max())
    # a simulated tensor-core value within the whole bound of the chain
    d = eps * cs * 1.001 ** 2 + np.abs(l32.astype(np.float64)) * 4.8e-7 + 1e-30
    tc = _simulated_tensor_core(x64, w64, slices)
    gap = np.abs(tc - l32.astype(np.float64))
    assert np.all(gap <= d), float((gap / d).max())
    return float((chain_err / (eps * cs)).max()), float((gap / d).max())


def test_bound_covers_chain_and_blocked_sums_prefill_shape():
    cfg = CONFIGS["prefill"].replace(name="bnd", T=48, seed=51)
    r_chain, r_tc = _check(cfg, adversarial=False, slices=4)
    assert r_chain < 0.1 and r_tc < 0.5   # typical inputs sit far inside the bound


def test_bound_covers_heavy_cancellation():
    cfg = CONFIGS["prefill"].replace(name="bnd_adv", T=40, H=1024, E=64, seed=52)
    _check(cfg, adversarial=True, slices=8)


def test_bound_is_tight_enough_to_matter():
    # The bound must not be so loose that the tensor-core filter excludes nothing: at
    # the prefill shape (k = 8 of 256) the experts whose upper bound reaches the k-th
    # largest lower bound -- the ones whose chain is evaluated -- stay close to k.
    cfg = CONFIGS["prefill"].replace(name="bnd_t", T=32, seed=53)
    x, rw, _ = _case(cfg)
    x64, w64 = _bf16_to_f64(x), _bf16_to_f64(rw)
    _, cs, eps = _bound_parts(x64, w64, cfg.H, 4)
    lt = x64 @ w64
    d = eps * cs * 1.001 ** 2
    tau = -np.sort(-(lt - d), axis=1)[:, cfg.top_k - 1:cfg.top_k]
    cand = (lt + d >= tau).sum(axis=1)
    assert cand.min() >= cfg.top_k and cand.mean() <= cfg.top_k + 2, cand.mean()
