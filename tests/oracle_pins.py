"""Pins of the CPU oracle to facts outside itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises ``AssertionError`` when the
oracle disagrees with brute force, a closed form, an invariant or a library
routine.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on copies of the oracle with a planted
mistake and requires every mistake to be caught by at least one pin.

Definition pinned (vLLM fused-MoE page, section 02): top-k routing by router
logits, softmax-normalised gating over the chosen k, a gate/up/down SwiGLU FFN
per expert, and the gate-weighted sum of the k expert outputs.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch
import torch.nn.functional as F

from routed_grouped_gemm_softmax_b200.inputs import CONFIGS, make_inputs


def _bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().double().numpy()


def tiny_inputs(**kw):
    cfg = CONFIGS["tiny"].replace(**kw)
    return make_inputs(cfg)


# ------------------------------------------------------------------ router

def pin_logits_vs_fp64_matmul(orc):
    """fp32 FMA-chain logits agree with an fp64 numpy matmul within the chain's
    forward error bound (n*u*sum|x*w|), and the oracle's own fp64 logits agree with
    numpy's to 1e-12 relative.  A transposed/dropped/shifted term breaks this."""
    for bias_on in (False, True):
        inp = tiny_inputs(zipf_s=1.2 if bias_on else None)
        idx, gate, l32, l64 = orc.route(inp.x, inp.router_w, inp.bias, 2, want_logits=True)
        X, W = _f64(inp.x), _f64(inp.router_w)
        ref = X @ W
        if inp.bias is not None:
            ref = ref + inp.bias.double().numpy()[None, :]
        mag = np.abs(X) @ np.abs(W)
        H = X.shape[1]
        bound = (H + 2) * 2.0 ** -24 * (mag + (np.abs(inp.bias.double().numpy())[None, :]
                                               if inp.bias is not None else 0.0)) + 1e-30
        assert np.all(np.abs(l32.astype(np.float64) - ref) <= bound), "fp32 logits off the bound"
        assert np.allclose(l64, ref, rtol=1e-12, atol=1e-12), "fp64 logits differ from matmul"


def pin_logit_chain_order(orc):
    """Closed form of the fixed evaluation order: with x = [1, 2^-12, 2^-12] and
    w = [1, 2^-12, 2^-12] the chain fma over h ascending gives 1 + 2^-24 -> 1
    (tie to even) twice, i.e. exactly 1.0f; summing the small terms first would
    give 1 + 2^-23.  Integer-valued inputs give the exact integer dot product."""
    s = 2.0 ** -12
    x = _bf16([[1.0, s, s]])
    w = _bf16([[1.0, 0.0], [s, 0.0], [s, 0.0]])
    _, _, l32, _ = orc.route(x, w, None, 1, want_logits=True)
    assert l32[0, 0] == np.float32(1.0), l32[0, 0]
    x = _bf16([[3, -2, 5, 7]])
    w = _bf16([[1, 2], [4, -3], [-1, 2], [2, 1]])
    _, _, l32, _ = orc.route(x, w, None, 2, want_logits=True)
    assert l32[0, 0] == 3 - 8 - 5 + 14 and l32[0, 1] == 6 + 6 + 10 + 7, l32


def pin_topk_brute_force(orc):
    """Tiny: the selected k equal the first k of a library sort by (-logit, e), and no
    other k-subset has a larger logit sum (brute-force enumeration of all subsets)."""
    inp = tiny_inputs()
    for k in (1, 2, 3, 8):
        idx, _, l32, _ = orc.route(inp.x, inp.router_w, None, k, want_logits=True)
        E = l32.shape[1]
        for t in range(l32.shape[0]):
            order = sorted(range(E), key=lambda e: (-float(l32[t, e]), e))
            assert list(idx[t]) == order[:k], (t, idx[t], order[:k])
            best = max(sum(float(l32[t, e]) for e in c) for c in itertools.combinations(range(E), k))
            assert sum(float(l32[t, e]) for e in idx[t]) == best


def pin_ties_lower_index(orc):
    """Equal logits go to the lower expert index: router_w = 0 gives experts 0..k-1
    with gates 1/k; a bias with exact ties [0,1,0,1,1] picks [1,3,4,0,2]."""
    inp = tiny_inputs()
    z = torch.zeros_like(inp.router_w)
    for k in (1, 3, 8):
        idx, gate = orc.route(inp.x, z, None, k)
        assert np.all(idx == np.arange(k)[None, :])
        assert np.all(gate == 1.0 / k) if k in (1, 8) else np.allclose(gate, 1.0 / k, rtol=0, atol=1e-15)
    x = _bf16(np.ones((2, 4)))
    w = _bf16(np.zeros((4, 5)))
    bias = torch.tensor([0.0, 1.0, 0.0, 1.0, 1.0])
    idx, _ = orc.route(x, w, bias, 5)
    assert np.all(idx == np.array([1, 3, 4, 0, 2])[None, :]), idx


def pin_gates(orc):
    """Gates sum to 1; k=1 gives exactly 1; k=2 matches the closed form
    1/(1+exp(l1-l0)); and softmax over all E renormalised over the chosen k
    (scipy) equals the softmax over the chosen k."""
    from scipy.special import softmax
    inp = tiny_inputs()
    idx, gate = orc.route(inp.x, inp.router_w, None, 1)
    assert np.all(gate == 1.0)
    idx, gate, l32, _ = orc.route(inp.x, inp.router_w, None, 2, want_logits=True)
    l = l32.astype(np.float64)
    for t in range(l.shape[0]):
        d = l[t, idx[t, 1]] - l[t, idx[t, 0]]
        assert abs(gate[t, 0] - 1.0 / (1.0 + math.exp(d))) <= 1e-15
    for k in (3, 5):
        idx, gate, l32, _ = orc.route(inp.x, inp.router_w, None, k, want_logits=True)
        assert np.all(np.abs(gate.sum(1) - 1.0) <= 1e-12)
        p = softmax(l32.astype(np.float64), axis=1)
        sel = np.take_along_axis(p, idx.astype(np.int64), 1)
        assert np.allclose(gate, sel / sel.sum(1, keepdims=True), rtol=1e-12, atol=0)


def pin_bias_enters_logits(orc):
    """A per-expert bias shifts every token's logit by exactly bias[e] (up to the one
    fp32 rounding of the final add): with a huge bias on expert 5 every token picks 5 first."""
    inp = tiny_inputs()
    b = torch.zeros(8)
    b[5] = 1000.0
    idx, _, l32, _ = orc.route(inp.x, inp.router_w, b, 2, want_logits=True)
    _, _, l0, _ = orc.route(inp.x, inp.router_w, None, 2, want_logits=True)
    assert np.all(idx[:, 0] == 5)
    assert np.all(l32[:, 5] == (l0[:, 5] + np.float32(1000.0)))
    assert np.all(np.delete(l32, 5, 1) == np.delete(l0, 5, 1))


# ----------------------------------------------------------------- permute

def _check_permute(idx, E, p, bm=128):
    fl = np.asarray(idx).reshape(-1)
    A = fl.size
    s2f, f2s, off = p["sorted_to_flat"], p["flat_to_sorted"], p["offsets"]
    assert off[0] == 0 and off[E] == A and np.all(np.diff(off) >= 0)
    assert np.array_equal(np.diff(off), np.bincount(fl, minlength=E))
    assert np.array_equal(np.sort(s2f), np.arange(A)), "not a bijection"
    assert np.array_equal(s2f[f2s], np.arange(A)) and np.array_equal(f2s[s2f], np.arange(A))
    assert np.array_equal(s2f, np.argsort(fl, kind="stable")), "not the stable sort"
    tiles = [(e, off[e] + r, min(bm, off[e + 1] - off[e] - r))
             for e in range(E) for r in range(0, off[e + 1] - off[e], bm)]
    assert p["num_tiles"] == len(tiles)
    assert [tuple(int(v) for v in row) for row in p["tile_list"]] == tiles


def pin_permute(orc):
    """Bijection + inverse, offsets = cumulative bincount, order = numpy's stable
    argsort, tile list = closed form; on skewed, empty and single-expert routings."""
    rng = np.random.default_rng(7)
    cases = [(rng.integers(0, 8, size=(64, 2)), 8),
             (rng.integers(0, 256, size=(512, 8)), 256),
             (np.zeros((300, 1), np.int64), 4),                   # one expert holds all
             (np.minimum(rng.zipf(1.5, size=(1000, 3)) - 1, 15), 16),
             (np.zeros((0, 2), np.int64), 8)]                     # empty
    for bm in (128, 7):
        for idx, E in cases:
            p = orc.permute(idx, E, bm=bm)
            _check_permute(idx, E, p, bm)


# ------------------------------------------------------------- expert FFN

def _dense_reference(inp, idx, gate):
    """Brute force: every expert on every token (numpy fp64 matmuls), masked by a
    dense [T,E] gate matrix that is zero for experts a token did not pick."""
    X = _f64(inp.x)
    Wg, Wu, Wd = _f64(inp.w_gate), _f64(inp.w_up), _f64(inp.w_down)
    T, E = X.shape[0], Wg.shape[0]
    G = np.zeros((T, E))
    for t in range(T):
        for j in range(idx.shape[1]):
            G[t, idx[t, j]] += gate[t, j]
    out = np.zeros_like(X)
    for e in range(E):
        g = X @ Wg[e].T
        u = X @ Wu[e].T
        a = (g / (1.0 + np.exp(-g))) * u
        out += G[:, e:e + 1] * (a @ Wd[e].T)
    return out


def pin_ffn_dense_brute_force(orc):
    """Tiny: the per-token sparse evaluation equals the dense all-experts evaluation."""
    for k in (1, 2, 5):
        inp = tiny_inputs(T=24)
        idx, gate = orc.route(inp.x, inp.router_w, None, k)
        out = orc.combine_ffn(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down)
        ref = _dense_reference(inp, idx, gate)
        assert np.allclose(out, ref, rtol=1e-11, atol=1e-12), np.abs(out - ref).max()


def pin_topk_all_uniform_is_mean(orc):
    """top_k = E with router_w = 0 (uniform gates 1/E): out = mean_e FFN_e(x) (torch fp64)."""
    inp = tiny_inputs(T=16)
    z = torch.zeros_like(inp.router_w)
    out, idx, gate = orc.forward(inp.x, z, None, inp.w_gate, inp.w_up, inp.w_down, top_k=8)
    x = inp.x.double()
    ys = []
    for e in range(8):
        a = F.silu(x @ inp.w_gate[e].double().T) * (x @ inp.w_up[e].double().T)
        ys.append(a @ inp.w_down[e].double().T)
    ref = torch.stack(ys).mean(0).numpy()
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12), np.abs(out - ref).max()


def pin_identical_experts(orc):
    """All experts identical: out = FFN(x) whatever the routing (gates sum to 1)."""
    inp = tiny_inputs(T=16)
    wg = inp.w_gate[:1].expand_as(inp.w_gate).contiguous()
    wu = inp.w_up[:1].expand_as(inp.w_up).contiguous()
    wd = inp.w_down[:1].expand_as(inp.w_down).contiguous()
    out, _, _ = orc.forward(inp.x, inp.router_w, None, wg, wu, wd, top_k=3)
    x = inp.x.double()
    ref = ((F.silu(x @ wg[0].double().T) * (x @ wu[0].double().T)) @ wd[0].double().T).numpy()
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12)


def pin_single_expert_is_swiglu_mlp(orc):
    """E = 1, k = 1: the layer is a textbook SwiGLU MLP (torch fp64 silu and matmuls)."""
    inp = tiny_inputs(T=12, E=1)
    out, idx, gate = orc.forward(inp.x, inp.router_w, None, inp.w_gate, inp.w_up, inp.w_down, top_k=1)
    assert np.all(idx == 0) and np.all(gate == 1.0)
    x = inp.x.double()
    ref = ((F.silu(x @ inp.w_gate[0].double().T) * (x @ inp.w_up[0].double().T))
           @ inp.w_down[0].double().T).numpy()
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12)


def pin_linear_in_down_proj(orc):
    """Doubling W_down (exact in bf16) doubles the output exactly."""
    inp = tiny_inputs(T=8)
    idx, gate = orc.route(inp.x, inp.router_w, None, 2)
    a = orc.combine_ffn(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down)
    b = orc.combine_ffn(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down * 2)
    assert np.array_equal(b, 2 * a)


def pin_worked_example(orc):
    """Hand-derived example: x = [1, 2]; router columns give logits (1, 2, 1.5) so the
    top-2 is (1, 2) with gates (1/(1+e^-0.5), 1/(1+e^0.5)); with I = 1,
      expert 1: g = 1, u = 2, a = 2 silu(1), y = a * (1, -1)
      expert 2: g = 2, u = 3, a = 3 silu(2), y = a * (0.5, 2)."""
    x = _bf16([[1.0, 2.0]])
    rw = _bf16([[1.0, 0.0, 0.5], [0.0, 1.0, 0.5]])
    wg = _bf16([[[0.0, 0.0]], [[1.0, 0.0]], [[0.0, 1.0]]])
    wu = _bf16([[[0.0, 0.0]], [[0.0, 1.0]], [[1.0, 1.0]]])
    wd = _bf16([[[0.0], [0.0]], [[1.0], [-1.0]], [[0.5], [2.0]]])
    out, idx, gate = orc.forward(x, rw, None, wg, wu, wd, top_k=2)
    assert list(idx[0]) == [1, 2]
    g0, g1 = 1.0 / (1.0 + math.exp(-0.5)), 1.0 / (1.0 + math.exp(0.5))
    assert abs(gate[0, 0] - g0) < 1e-15 and abs(gate[0, 1] - g1) < 1e-15
    silu = lambda v: v / (1.0 + math.exp(-v))
    a1, a2 = 2.0 * silu(1.0), 3.0 * silu(2.0)
    ref = [g0 * a1 + g1 * 0.5 * a2, -g0 * a1 + g1 * 2.0 * a2]
    assert np.allclose(out[0], ref, rtol=1e-14, atol=0), (out[0], ref)


ALL_PINS = [pin_logits_vs_fp64_matmul, pin_logit_chain_order, pin_topk_brute_force,
            pin_ties_lower_index, pin_gates, pin_bias_enters_logits, pin_permute,
            pin_ffn_dense_brute_force, pin_topk_all_uniform_is_mean, pin_identical_experts,
            pin_single_expert_is_swiglu_mlp, pin_linear_in_down_proj, pin_worked_example]


# ------------------------------------------------------------- FP8 variant

def _e4m3_torch(v):
    """Library rounding: torch's float8_e4m3fn cast (values already in +-448)."""
    return torch.as_tensor(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_e4m3_codes_vs_torch(orc):
    """Decoding every finite code matches torch's float8_e4m3fn -> float; encoding matches
    torch's cast on random values, on every exact midpoint between neighbouring codes
    (ties to even) and on the subnormal range."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    dec = orc.e4m3_decode(codes)
    ref = torch.as_tensor(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(dec, ref)
    pos = np.sort(np.unique(np.abs(dec)))
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(3)
    vals = np.concatenate([mids, -mids, pos, -pos, rng.uniform(-448, 448, 5000),
                           rng.uniform(-0.02, 0.02, 2000), [0.0, -0.0, 448.0, -448.0]]).astype(np.float32)
    assert np.array_equal(orc.e4m3_encode(vals), _e4m3_torch(vals))


def pin_quantize_rows(orc):
    """Row/128-group quantiser: scale = amax/448 in fp32, codes = e4m3(clamp(v/s)) (torch
    cast as the rounding routine), round-trip error within half an e4m3 step, a zero
    group gives scale 1 and zero codes."""
    rng = np.random.default_rng(5)
    a = torch.as_tensor(rng.standard_normal((6, 384)).astype(np.float32)).to(torch.bfloat16)
    a[2, 128:256] = 0.0
    a[4, :] *= 1e-3
    q, s = orc.quantize_rows(a)
    f = a.float().view(6, 3, 128)
    amax = f.abs().amax(-1)
    s_ref = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    assert np.array_equal(s, s_ref.numpy())
    r = (f / s_ref[..., None]).clamp(-448, 448)
    assert np.array_equal(q, _e4m3_torch(r.reshape(6, 384).numpy()))
    assert np.all(q[2, 128:256] == 0) and s[2, 1] == 1.0
    deq = torch.as_tensor(q).view(torch.float8_e4m3fn).double().view(6, 3, 128) * torch.as_tensor(s).double()[..., None]
    err = (deq - f.double()).abs()
    assert torch.all(err <= (f.double().abs() * 2.0 ** -4 + torch.as_tensor(s).double()[..., None] * 2.0 ** -10))


def _fp8_case(E=3, H=256, I=256, T=10, k=2, seed=9):
    from routed_grouped_gemm_softmax_b200.inputs import make_fp8_weights
    cfg = CONFIGS["fp8"].replace(E=E, H=H, I=I, T=T, top_k=k, seed=seed)
    inp = make_inputs(cfg, weights=False)
    return cfg, inp, make_fp8_weights(cfg)


def _fp8_dense_reference(inp, w, idx, gate):
    """Brute force: dequantise every weight to fp64 (torch float8 -> float), quantise x and
    h with torch casts, run dense fp64 matmuls for every expert, mask by the gates."""
    def deq(q, s):
        E, N, K = q.shape
        v = q.view(torch.float8_e4m3fn).double().view(E, N // 128, 128, K // 128, 128)
        return (v * s.double()[:, :, None, :, None]).view(E, N, K)

    def quant_rows(m32):  # m32: fp32 [R, K] -> dequantised fp64 [R, K]
        R, K = m32.shape
        g = m32.view(R, K // 128, 128)
        amax = g.abs().amax(-1)
        s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
        qq = (g / s[..., None]).clamp(-448, 448).to(torch.float8_e4m3fn)
        return (qq.double() * s.double()[..., None]).view(R, K)

    Wg, Wu, Wd = deq(w["w_gate_q"], w["w_gate_s"]), deq(w["w_up_q"], w["w_up_s"]), deq(w["w_down_q"], w["w_down_s"])
    X = quant_rows(inp.x.float())
    T, E = X.shape[0], Wg.shape[0]
    G = torch.zeros(T, E, dtype=torch.float64)
    for t in range(T):
        for j in range(idx.shape[1]):
            G[t, int(idx[t, j])] += float(gate[t, j])
    out = torch.zeros(T, X.shape[1], dtype=torch.float64)
    for e in range(E):
        h = (F.silu(X @ Wg[e].T) * (X @ Wu[e].T)).float()
        out += G[:, e:e + 1] * (quant_rows(h) @ Wd[e].T)
    return out.numpy()


def pin_fp8_ffn_dense_brute_force(orc):
    """FP8 layer: the oracle's blockwise sums equal the dense dequantise-then-matmul
    evaluation (torch casts for every quantisation decision) on a small case."""
    cfg, inp, w = _fp8_case()
    idx, gate = orc.route(inp.x, inp.router_w, None, cfg.top_k)
    out = orc.combine_ffn_fp8(inp.x, idx, gate, w["w_gate_q"], w["w_gate_s"], w["w_up_q"], w["w_up_s"],
                              w["w_down_q"], w["w_down_s"])
    ref = _fp8_dense_reference(inp, w, idx, gate)
    assert np.allclose(out, ref, rtol=1e-9, atol=1e-12), np.abs(out - ref).max()


def pin_fp8_close_to_unquantised(orc):
    """The fp8 layer approximates the unquantised layer on the same master weights
    (bf16 copies): relative L2 error of a few percent, far below 1."""
    cfg, inp, w = _fp8_case(T=16)
    full = make_inputs(cfg)
    idx, gate = orc.route(inp.x, inp.router_w, None, cfg.top_k)
    a = orc.combine_ffn_fp8(inp.x, idx, gate, w["w_gate_q"], w["w_gate_s"], w["w_up_q"], w["w_up_s"],
                            w["w_down_q"], w["w_down_s"])
    b = orc.combine_ffn(inp.x, idx, gate, full.w_gate.to(torch.bfloat16), full.w_up.to(torch.bfloat16),
                        full.w_down.to(torch.bfloat16))
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-3 < rel < 0.08, rel


ALL_PINS += [pin_e4m3_codes_vs_torch, pin_quantize_rows, pin_fp8_ffn_dense_brute_force,
             pin_fp8_close_to_unquantised]


# ------------------------------------------------------------- shared expert

def pin_shared_expert_is_swiglu_mlp(orc):
    """A shared expert (every token, weight 1) is a textbook SwiGLU MLP: torch fp64
    silu(x Wg^T) * (x Wu^T), then Wd, on all tokens and on a subset in any order.
    Its intermediate size differs from the routed experts' so that a mixed-up
    shape or transposed operand cannot pass.  With the weights of routed expert e
    it equals the layer restricted to expert e with gate 1."""
    inp = tiny_inputs(T=12)
    H, I_s = inp.x.shape[1], 192
    g = torch.Generator().manual_seed(7)
    wg = (torch.randn(I_s, H, generator=g, dtype=torch.float64) / H ** 0.5).to(torch.bfloat16)
    wu = (torch.randn(I_s, H, generator=g, dtype=torch.float64) / H ** 0.5).to(torch.bfloat16)
    wd = (torch.randn(H, I_s, generator=g, dtype=torch.float64) / I_s ** 0.5).to(torch.bfloat16)
    out = orc.shared_ffn(inp.x, wg, wu, wd)
    X = inp.x.double()
    ref = (F.silu(X @ wg.double().T) * (X @ wu.double().T)) @ wd.double().T
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    sub = orc.shared_ffn(inp.x, wg, wu, wd, tokens=[5, 2, 11])
    assert np.array_equal(sub, out[[5, 2, 11]])
    e = 3
    T = inp.x.shape[0]
    one = orc.combine_ffn(inp.x, np.full((T, 1), e, np.int32), np.ones((T, 1)), inp.w_gate, inp.w_up, inp.w_down)
    same = orc.shared_ffn(inp.x, inp.w_gate[e], inp.w_up[e], inp.w_down[e])
    assert np.allclose(same, one, rtol=1e-13, atol=1e-13)


ALL_PINS += [pin_shared_expert_is_swiglu_mlp]


# --------------------------------------------- MX variant (FP4 weights, FP8 acts)

E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # the e2m1 magnitudes, OCP MX v1.0 table


def _e4m3_mags():
    """The 127 finite non-negative e4m3 magnitudes, decoded by torch's float8_e4m3fn."""
    return torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def _rne_code(v, mags, sign_bit):
    """Nearest magnitude by brute force; a tie goes to the even code."""
    a = abs(float(v))
    d = np.abs(np.asarray(mags) - a)
    near = np.flatnonzero(d == d.min())
    c = int(near[0]) if near.size == 1 else int([n for n in near if n % 2 == 0][0])
    return c | ((1 << sign_bit) if (v < 0 and c != 0) else 0)


def _mx_quant_ref(row, fmt):
    """Reference MX quantisation of one row (numpy): per 32 values, X = floor(log2 amax)
    - emax (np.frexp), elements round-to-nearest-even of v / 2^X, clamped."""
    mags, sb, emax, vmax = (_e4m3_mags(), 7, 8, 448.0) if fmt == 0 else (E2M1_MAGS, 3, 2, 6.0)
    row = np.asarray(row, dtype=np.float32).astype(np.float64)
    q = np.zeros(row.size, np.uint8)
    xs = np.zeros(row.size // 32, np.uint8)
    for b in range(row.size // 32):
        blk = row[b * 32:(b + 1) * 32]
        amax = np.abs(blk).max()
        if amax == 0.0:
            xs[b] = 127
            continue
        X = int(np.clip(np.frexp(amax)[1] - 1 - emax, -127, 127))
        xs[b] = X + 127
        r = np.clip(np.ldexp(blk, -X), -vmax, vmax)
        q[b * 32:(b + 1) * 32] = [_rne_code(v, mags, sb) for v in r]
    return q, xs


def _mx_dequant(q, xs, fmt):
    mags = _e4m3_mags() if fmt == 0 else np.asarray(E2M1_MAGS)
    sb = 7 if fmt == 0 else 3
    q = np.asarray(q, dtype=np.int64)
    mag = mags[q & ((1 << sb) - 1)] * np.where(q >> sb, -1.0, 1.0)
    sc = np.ldexp(1.0, np.repeat(np.asarray(xs, dtype=np.int64) - 127, 32, axis=-1))
    return mag * sc


def pin_e2m1_codes(orc):
    """e2m1 decoding is the OCP table; encoding is the nearest code with ties to the even
    code, on random values, every midpoint between neighbours, and past the largest."""
    codes = np.arange(16, dtype=np.uint8)
    ref = np.array(E2M1_MAGS + [-m for m in E2M1_MAGS])
    assert np.array_equal(orc.e2m1_decode(codes), ref)
    vals = list(np.random.default_rng(3).uniform(-6.5, 6.5, 500).astype(np.float32))
    vals += [(a + b) / 2 for a, b in zip(E2M1_MAGS, E2M1_MAGS[1:])] + [-0.75, -2.5, 6.0, 7.0, -9.0]
    got = orc.e2m1_encode(np.asarray(vals, np.float32))
    assert [int(c) for c in got] == [_rne_code(v, E2M1_MAGS, 3) for v in vals]


def pin_mx_quantize_rows(orc):
    """MX quantisation of both element formats equals the reference on random rows of
    many magnitudes, an all-zero block, a block with one huge value and exact powers of two."""
    rng = np.random.default_rng(4)
    rows = [rng.standard_normal(64) * 10.0 ** rng.uniform(-3, 3) for _ in range(6)]
    special = np.zeros(64)
    special[32:] = rng.standard_normal(32)
    special[40] = 3.0e4
    rows += [special, np.ldexp(1.0, np.arange(-20, 44))]
    a = np.asarray(rows, dtype=np.float32)
    for fmt in (0, 1):
        q, xs = orc.mx_quantize_rows(a, fmt)
        for r in range(a.shape[0]):
            qr, xr = _mx_quant_ref(a[r], fmt)
            assert np.array_equal(xs[r], xr), (fmt, r)
            assert np.array_equal(q[r], qr), (fmt, r)
        assert list(xs[6][:1]) == [127] and not q[6][:32].any()   # the all-zero block


def _mx_case():
    rng = np.random.default_rng(5)
    T, H, I, E, k = 6, 64, 96, 3, 2
    x = torch.as_tensor(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16)
    master = {n: rng.standard_normal((E,) + s).astype(np.float32) / np.sqrt(s[1])
              for n, s in (("w_gate", (I, H)), ("w_up", (I, H)), ("w_down", (H, I)))}
    w = {}
    for n, m in master.items():
        E_, N, K = m.shape
        qs = [_mx_quant_ref(m[e, r], 1) for e in range(E_) for r in range(N)]
        w[n + "_q"] = np.stack([a for a, _ in qs]).reshape(E_, N, K)
        w[n + "_x"] = np.stack([b for _, b in qs]).reshape(E_, N, K // 32)
    idx = np.array([[0, 1], [2, 0], [1, 2], [0, 2], [2, 1], [1, 0]], np.int32)
    gate = rng.uniform(0.1, 1.0, (T, k))
    gate /= gate.sum(1, keepdims=True)
    return x, master, w, idx, gate


def pin_mx_ffn_dense_brute_force(orc):
    """The MX layer equals a dense evaluation: every quantisation by the reference, the
    codes dequantised, then fp64 matmuls, SwiGLU (torch silu), h rounded to fp32."""
    x, _, w, idx, gate = _mx_case()
    out = orc.combine_ffn_mx(x, idx, gate, w["w_gate_q"], w["w_gate_x"], w["w_up_q"], w["w_up_x"],
                             w["w_down_q"], w["w_down_x"])
    deq = {n: _mx_dequant(w[n + "_q"], w[n + "_x"], 1) for n in ("w_gate", "w_up", "w_down")}
    X = x.float().numpy()
    ref = np.zeros(out.shape)
    for t in range(X.shape[0]):
        qx, sx = _mx_quant_ref(X[t], 0)
        xd = _mx_dequant(qx, sx, 0)
        for j in range(idx.shape[1]):
            e = idx[t, j]
            g, u = deq["w_gate"][e] @ xd, deq["w_up"][e] @ xd
            h = (F.silu(torch.as_tensor(g)) * torch.as_tensor(u)).numpy().astype(np.float32)
            qh, sh = _mx_quant_ref(h, 0)
            ref[t] += gate[t, j] * (deq["w_down"][e] @ _mx_dequant(qh, sh, 0))
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-12), np.abs(out - ref).max()


def pin_mx_close_to_unquantised(orc):
    """With FP4 weights and FP8 activations the layer stays near the unquantised layer
    on the same master weights (rel-L2 well below 1: no dropped scale or factor 2^k)."""
    x, master, w, idx, gate = _mx_case()
    out = orc.combine_ffn_mx(x, idx, gate, w["w_gate_q"], w["w_gate_x"], w["w_up_q"], w["w_up_x"],
                             w["w_down_q"], w["w_down_x"])
    ref = orc.combine_ffn(x, idx, gate, *[torch.as_tensor(master[n]).to(torch.bfloat16)
                                          for n in ("w_gate", "w_up", "w_down")])
    r = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert r < 0.3, r


ALL_PINS += [pin_e2m1_codes, pin_mx_quantize_rows, pin_mx_ffn_dense_brute_force, pin_mx_close_to_unquantised]
